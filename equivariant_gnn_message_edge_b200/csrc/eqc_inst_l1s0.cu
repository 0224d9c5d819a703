// Kernel instances for L_in = 1, L_sh = 0.
#define EQC_LIN 1
#define EQC_LSH 0
#include "eqc_inst.cuh"

// Kernel instances for L_in = 0, L_sh = 1.
#define EQC_LIN 0
#define EQC_LSH 1
#include "eqc_inst.cuh"

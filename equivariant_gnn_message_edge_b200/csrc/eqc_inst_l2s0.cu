// Kernel instances for L_in = 2, L_sh = 0.
#define EQC_LIN 2
#define EQC_LSH 0
#include "eqc_inst.cuh"

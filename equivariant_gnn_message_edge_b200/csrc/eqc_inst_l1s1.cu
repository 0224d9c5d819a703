// Kernel instances for L_in = 1, L_sh = 1.
#define EQC_LIN 1
#define EQC_LSH 1
#include "eqc_inst.cuh"

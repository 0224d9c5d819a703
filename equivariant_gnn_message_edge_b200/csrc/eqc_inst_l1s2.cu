// Kernel instances for L_in = 1, L_sh = 2.
#define EQC_LIN 1
#define EQC_LSH 2
#include "eqc_inst.cuh"

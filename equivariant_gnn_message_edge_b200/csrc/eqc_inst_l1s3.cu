// Kernel instances for L_in = 1, L_sh = 3.
#define EQC_LIN 1
#define EQC_LSH 3
#include "eqc_inst.cuh"

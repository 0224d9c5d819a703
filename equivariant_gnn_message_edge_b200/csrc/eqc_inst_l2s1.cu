// Kernel instances for L_in = 2, L_sh = 1.
#define EQC_LIN 2
#define EQC_LSH 1
#include "eqc_inst.cuh"

// Kernel instances for L_in = 3, L_sh = 2.
#define EQC_LIN 3
#define EQC_LSH 2
#include "eqc_inst.cuh"

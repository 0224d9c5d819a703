// Kernel instances for L_in = 3, L_sh = 0.
#define EQC_LIN 3
#define EQC_LSH 0
#include "eqc_inst.cuh"

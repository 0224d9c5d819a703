// Kernel instances for L_in = 2, L_sh = 3.
#define EQC_LIN 2
#define EQC_LSH 3
#include "eqc_inst.cuh"

// Kernel instances for L_in = 0, L_sh = 2.
#define EQC_LIN 0
#define EQC_LSH 2
#include "eqc_inst.cuh"

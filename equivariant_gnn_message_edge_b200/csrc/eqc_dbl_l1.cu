// Double-backward kernel instances for L_in = 1.
#define EQC_LIN 1
#include "eqc_dbl_inst.cuh"

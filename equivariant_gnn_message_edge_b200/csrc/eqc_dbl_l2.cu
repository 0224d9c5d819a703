// Double-backward kernel instances for L_in = 2.
#define EQC_LIN 2
#include "eqc_dbl_inst.cuh"

// Double-backward kernel instances for L_in = 0.
#define EQC_LIN 0
#include "eqc_dbl_inst.cuh"

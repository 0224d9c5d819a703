// Double-backward kernel instances for L_in = 3.
#define EQC_LIN 3
#include "eqc_dbl_inst.cuh"

// Kernel instances for both-parity outputs, L_in = 2.
#define EQC_MODE 1
#define EQC_LIN 2
#include "eqc_inst_modes.cuh"

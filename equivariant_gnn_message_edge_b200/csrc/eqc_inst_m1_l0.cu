// Kernel instances for both-parity outputs, L_in = 0.
#define EQC_MODE 1
#define EQC_LIN 0
#include "eqc_inst_modes.cuh"

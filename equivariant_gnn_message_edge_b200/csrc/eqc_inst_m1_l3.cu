// Kernel instances for both-parity outputs, L_in = 3.
#define EQC_MODE 1
#define EQC_LIN 3
#include "eqc_inst_modes.cuh"

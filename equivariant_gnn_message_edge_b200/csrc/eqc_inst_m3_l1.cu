// Kernel instances for both-parity per-path outputs, L_in = 1.
#define EQC_MODE 3
#define EQC_LIN 1
#include "eqc_inst_modes.cuh"

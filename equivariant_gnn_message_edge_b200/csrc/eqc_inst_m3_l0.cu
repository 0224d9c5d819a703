// Kernel instances for both-parity per-path outputs, L_in = 0.
#define EQC_MODE 3
#define EQC_LIN 0
#include "eqc_inst_modes.cuh"

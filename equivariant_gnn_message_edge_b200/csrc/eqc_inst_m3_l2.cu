// Kernel instances for both-parity per-path outputs, L_in = 2.
#define EQC_MODE 3
#define EQC_LIN 2
#include "eqc_inst_modes.cuh"

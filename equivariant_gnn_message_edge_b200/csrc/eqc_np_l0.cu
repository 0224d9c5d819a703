// Node-local product kernel instances for L_u = 0.
#define EQC_LIN 0
#include "eqc_nodeprod_inst.cuh"

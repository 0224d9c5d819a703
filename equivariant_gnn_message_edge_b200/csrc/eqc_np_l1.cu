// Node-local product kernel instances for L_u = 1.
#define EQC_LIN 1
#include "eqc_nodeprod_inst.cuh"

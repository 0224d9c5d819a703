// Node-local product kernel instances for L_u = 3.
#define EQC_LIN 3
#include "eqc_nodeprod_inst.cuh"

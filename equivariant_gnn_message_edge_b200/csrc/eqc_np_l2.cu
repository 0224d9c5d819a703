// Node-local product kernel instances for L_u = 2.
#define EQC_LIN 2
#include "eqc_nodeprod_inst.cuh"

// Instances for one (L_in, L_sh): every L_out in 0..3 and VEC in {2, 4}.
// Included by the eqc_inst_l<L_in>s<L_sh>.cu files with EQC_LIN / EQC_LSH set.
#include "eqc_launch.cuh"

#ifndef EQC_LIN
#error "EQC_LIN must be defined"
#endif

namespace eqc {

#ifndef EQC_VEC_SMALL
#define EQC_VEC_SMALL 2
#endif
#define EQC_PAIR(LOUT) {Launch<Cfg<EQC_LIN, EQC_LSH, LOUT, EQC_VEC_SMALL>>::make(), Launch<Cfg<EQC_LIN, EQC_LSH, LOUT, 4>>::make()}
#define EQC_NAME2(a, b) instances_l##a##_s##b
#define EQC_NAME(a, b) EQC_NAME2(a, b)

const KernelSet* EQC_NAME(EQC_LIN, EQC_LSH)(int lout, int vec) {
    static const KernelSet table[4][2] = {EQC_PAIR(0), EQC_PAIR(1), EQC_PAIR(2), EQC_PAIR(3)};
    if (lout < 0 || lout > 3) return nullptr;
    if (vec == 2) return &table[lout][0];
    if (vec == 4) return &table[lout][1];
    return nullptr;
}

}  // namespace eqc

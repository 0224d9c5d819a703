// Instances for one (L_in, L_sh): every L_out in 0..3 and channel vector
// widths 1, 2 and 4 (tiles of 32, 64 and 128 channels).  Width 1 is compiled
// only where an l = 3 block makes the unrolled per-edge code large (there the
// narrower tile halves the code a warp runs and measured faster on B200);
// elsewhere its slot holds the width-2 kernels.
// Included by the eqc_inst_l<L_in>s<L_sh>.cu files with EQC_LIN / EQC_LSH set.
#include "eqc_launch.cuh"

#ifndef EQC_LIN
#error "EQC_LIN must be defined"
#endif

namespace eqc {

constexpr int narrow_vec(int lin, int lsh, int lout) { return (lin == 3 || lsh == 3 || lout == 3) ? 1 : 2; }

#define EQC_TRIPLE(LOUT)                                                     \
    {Launch<Cfg<EQC_LIN, EQC_LSH, LOUT, narrow_vec(EQC_LIN, EQC_LSH, LOUT)>>::make(), \
     Launch<Cfg<EQC_LIN, EQC_LSH, LOUT, 2>>::make(), Launch<Cfg<EQC_LIN, EQC_LSH, LOUT, 4>>::make()}
#define EQC_NAME2(a, b) instances_l##a##_s##b
#define EQC_NAME(a, b) EQC_NAME2(a, b)

const KernelSet* EQC_NAME(EQC_LIN, EQC_LSH)(int lout, int vec) {
    static const KernelSet table[4][3] = {EQC_TRIPLE(0), EQC_TRIPLE(1), EQC_TRIPLE(2), EQC_TRIPLE(3)};
    if (lout < 0 || lout > 3) return nullptr;
    if (vec == 1) return &table[lout][0];
    if (vec == 2) return &table[lout][1];
    if (vec == 4) return &table[lout][2];
    return nullptr;
}

}  // namespace eqc

// Instances of the output variants for one (mode, L_in): L_sh and L_out in
// 1..3, one channel width each (1 where an l = 3 block is present, else 2).
// Included by the eqc_inst_m<mode>_l<L_in>.cu files with EQC_MODE / EQC_LIN set.
#include "eqc_launch.cuh"

#if !defined(EQC_MODE) || !defined(EQC_LIN)
#error "EQC_MODE and EQC_LIN must be defined"
#endif

namespace eqc {

#define EQC_MI(LSH, LOUT) Launch<Cfg<EQC_LIN, LSH, LOUT, mode_vec(EQC_LIN, LSH, LOUT), EQC_MODE>>::make()
#define EQC_MROW(LSH) {EQC_MI(LSH, 1), EQC_MI(LSH, 2), EQC_MI(LSH, 3)}
#define EQC_MNAME2(m, a) instances_m##m##_l##a
#define EQC_MNAME(m, a) EQC_MNAME2(m, a)

const KernelSet* EQC_MNAME(EQC_MODE, EQC_LIN)(int lsh, int lout) {
    static const KernelSet table[3][3] = {EQC_MROW(1), EQC_MROW(2), EQC_MROW(3)};
    if (lsh < 1 || lsh > 3 || lout < 1 || lout > 3) return nullptr;
    return &table[lsh - 1][lout - 1];
}

}  // namespace eqc

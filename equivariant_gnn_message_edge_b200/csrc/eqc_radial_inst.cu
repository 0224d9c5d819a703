// Instances of the convolution with on-chip radial weights: natural-parity
// prefixes with L_in = L_sh = L_out in 1..3 and the (1, 2, 2) setting
// (0e+1o -> 0e+1o+2e).
#include "eqc_radial_launch.cuh"

namespace eqc {
namespace radial {

static const RadConvSet kSets[] = {
    RadLaunch<1, 1, 1>::make(),
    RadLaunch<1, 2, 2>::make(),
    RadLaunch<2, 2, 2>::make(),
    RadLaunch<3, 3, 3>::make(),
};

const RadConvSet* find_radial_conv(int lin, int lsh, int lout) {
    for (const RadConvSet& s : kSets)
        if (s.lin == lin && s.lsh == lsh && s.lout == lout) return &s;
    return nullptr;
}

}  // namespace radial
}  // namespace eqc

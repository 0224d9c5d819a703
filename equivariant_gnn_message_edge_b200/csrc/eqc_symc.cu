// Launchers and the instance table of the symmetric contraction (every
// L_A, L_out in 0..3): the forward at 64-channel tiles, the backward at
// 32-channel tiles (its per-species weight-gradient partials live in shared
// memory, one row of the tile's channels per species and weight).
#include <cuda_runtime.h>

#include "eqc_symc.cuh"
#include "eqc_symc.h"

namespace eqc {

void count_launch();

template <int LA, int LOUT>
struct SymLaunch {
    using KF = SymCfg<LA, LOUT, 2>;
    using KB = SymCfg<LA, LOUT, 1>;
    static int blocks(int N) {
        const int need = (N + kSymWarps - 1) / kSymWarps;
        return need < 148 ? (need > 0 ? need : 1) : 148;
    }
    static size_t workspace(int N, int C, int S) {
        return (size_t)blocks(N) * kSymWarps * S * KB::NW * C * sizeof(float);
    }
    static cudaError_t fwd(const SymParams& prm, cudaStream_t st) {
        const int need = (prm.N + kSymWarps - 1) / kSymWarps;
        const dim3 grid(need < 2 * 148 ? need : 2 * 148, (prm.C + KF::TILE_C - 1) / KF::TILE_C);
        eqconv_symc_fwd_kernel<KF><<<grid, kSymWarps * 32, 0, st>>>(prm);
        count_launch();
        return cudaGetLastError();
    }
    static cudaError_t bwd(const SymParams& prm_in, float* dW1, float* dW2, cudaStream_t st) {
        SymParams prm = prm_in;
        const dim3 grid(blocks(prm.N), (prm.C + KB::TILE_C - 1) / KB::TILE_C);
        prm.warps = (int)grid.x * kSymWarps;
        const int smem = kSymWarps * prm.S * KB::NW * KB::TILE_C * (int)sizeof(float);
        static bool done[64] = {};
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        if (dev >= 0 && dev < 64 && !done[dev]) {
            err = cudaFuncSetAttribute(eqconv_symc_bwd_kernel<KB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSymWarps * kSymMaxSpecies * KB::NW * KB::TILE_C * (int)sizeof(float));
            if (err != cudaSuccess) return err;
            done[dev] = true;
        }
        eqconv_symc_bwd_kernel<KB><<<grid, kSymWarps * 32, smem, st>>>(prm);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        const int64_t total = (int64_t)prm.S * KB::NW * prm.C;
        eqconv_symc_dw_reduce<KB><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(prm.dw_part, prm.warps, prm.S,
                                                                                  prm.C, dW1, dW2);
        count_launch();
        return cudaGetLastError();
    }
    static constexpr SymKernelSet make() {
        SymKernelSet k{LA, LOUT, KF::NP, KF::NW, KF::L1N, KF::D_A, KF::D_OUT, {}, &workspace, &fwd, &bwd};
        for (int q = 0; q < KF::NP; ++q) {
            k.paths[q][0] = KF::PL.l1[q];
            k.paths[q][1] = KF::PL.l2[q];
            k.paths[q][2] = KF::PL.l3[q];
        }
        return k;
    }
};

#define EQC_SROW(LA) SymLaunch<LA, 0>::make(), SymLaunch<LA, 1>::make(), SymLaunch<LA, 2>::make(), SymLaunch<LA, 3>::make()

const SymKernelSet* find_symc(int la, int lout) {
    static const SymKernelSet table[16] = {EQC_SROW(0), EQC_SROW(1), EQC_SROW(2), EQC_SROW(3)};
    if (la < 0 || la > 3 || lout < 0 || lout > 3) return nullptr;
    return &table[la * 4 + lout];
}

}  // namespace eqc

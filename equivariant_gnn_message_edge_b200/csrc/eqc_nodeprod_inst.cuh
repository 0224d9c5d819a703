// Host-side launchers of the node-local product for one kernel instance, and
// the instance table for one L_u (every L_v and L_out in 0..3; summed and
// per-path outputs; channel width 1 where an l = 3 block is present, else 2).
// Included by the eqc_np_l<L_u>.cu files with EQC_LIN set.
#pragma once

#include "eqc_launch.cuh"
#include "eqc_nodeprod.cuh"

#ifndef EQC_LIN
#error "EQC_LIN must be defined"
#endif

namespace eqc {

template <class K>
struct NpLaunch {
    // two CTAs of 4 warps per SM keep enough rows in flight to stream HBM;
    // a fixed grid makes each warp's dw partial cover a fixed node set
    static int blocks(int N) {
        const int need = (N + kNpWarps - 1) / kNpWarps;
        return need < 2 * 148 ? (need > 0 ? need : 1) : 2 * 148;
    }
    static cudaError_t fwd(const NpParams& prm_in, cudaStream_t st) {
        NpParams prm = prm_in;
        const dim3 grid(blocks(prm.N), (prm.C + K::TILE_C - 1) / K::TILE_C);
        eqconv_np_fwd_kernel<K><<<grid, kNpWarps * 32, 0, st>>>(prm);
        count_launch();
        return cudaGetLastError();
    }
    static cudaError_t bwd(const NpParams& prm_in, cudaStream_t st) {
        NpParams prm = prm_in;
        const dim3 grid(blocks(prm.N), (prm.C + K::TILE_C - 1) / K::TILE_C);
        prm.warps = (int)grid.x * kNpWarps;
        eqconv_np_bwd_kernel<K><<<grid, kNpWarps * 32, 0, st>>>(prm);
        count_launch();
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess || !prm.dw) return err;
        const int PC = K::NP * prm.C;
        eqconv_np_dw_reduce<><<<(PC + 127) / 128, 128, 0, st>>>(prm.dw_part, prm.warps, PC, prm.dw);
        count_launch();
        return cudaGetLastError();
    }
    static constexpr NpKernelSet make() { return NpKernelSet{K::LIN, K::LSH, K::LOUT, K::VEC, K::MODE, &fwd, &bwd}; }
};

#define EQC_NI(LSH, LOUT, MODE) NpLaunch<Cfg<EQC_LIN, LSH, LOUT, mode_vec(EQC_LIN, LSH, LOUT), MODE>>::make()
#define EQC_NROW(LSH, MODE) {EQC_NI(LSH, 0, MODE), EQC_NI(LSH, 1, MODE), EQC_NI(LSH, 2, MODE), EQC_NI(LSH, 3, MODE)}
#define EQC_NTAB(MODE) {EQC_NROW(0, MODE), EQC_NROW(1, MODE), EQC_NROW(2, MODE), EQC_NROW(3, MODE)}
#define EQC_NNAME2(a) np_instances_l##a
#define EQC_NNAME(a) EQC_NNAME2(a)

const NpKernelSet* EQC_NNAME(EQC_LIN)(int lsh, int lout, bool per_path) {
    static const NpKernelSet table[2][4][4] = {EQC_NTAB(0), EQC_NTAB(kModePerPath)};
    if (lsh < 0 || lsh > 3 || lout < 0 || lout > 3) return nullptr;
    return &table[per_path ? 1 : 0][lsh][lout];
}

}  // namespace eqc

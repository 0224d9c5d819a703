// Host-side launchers for one kernel instance (irreps L_in, L_sh, L_out and
// channel vector width VEC), collected into a KernelSet that the C ABI
// dispatches through.
#pragma once

#include <cuda_runtime.h>

#include "eqc_conv.cuh"
#include "eqc_dispatch.h"

namespace eqc {

void count_launch();

// One-time (per kernel, per device) opt-in above the 48 KB shared-memory default;
// `done` must be distinct for every kernel.
template <class Kern>
static cudaError_t ensure_smem(Kern kern, int bytes, bool (&done)[64]) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (bytes <= 48 * 1024 || dev >= 64 || done[dev]) return cudaSuccess;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err == cudaSuccess) done[dev] = true;
    return err;
}

template <class K>
struct Launch {
    static cudaError_t fwd(const FwdParams& prm_in, int tiles, int bands, cudaStream_t st) {
        FwdParams prm = prm_in;
        auto kern = eqconv_fwd_kernel<K>;
        static bool done[64] = {};
        constexpr int W = FwdShape<K>::WARPS;
        constexpr int smem = W * FwdShape<K>::L::BYTES;
        cudaError_t err = ensure_smem(kern, smem, done);
        if (err != cudaSuccess) return err;
        // with no edges the weight map is never read: give it a valid stand-in
        CUtensorMap tw, tx;
        if (!encode_rows_map(&tw, prm.E > 0 ? (const void*)prm.w : (const void*)prm.x,
                             prm.E > 0 ? (uint64_t)prm.E : (uint64_t)prm.N, prm.E > 0 ? K::NP : K::D_IN, prm.C,
                             K::TILE_C) ||
            !encode_rows_map(&tx, prm.x, (uint64_t)prm.N, K::D_IN, prm.C, K::TILE_C))
            return cudaErrorInvalidValue;
        dim3 grid((prm.N + W - 1) / W, tiles);
        for (int b = 0; b < bands; ++b) {
            prm.band_lo = (int)((int64_t)prm.N * b / bands);
            prm.band_hi = (int)((int64_t)prm.N * (b + 1) / bands);
            prm.accumulate = b > 0;
            kern<<<grid, W * 32, smem, st>>>(prm, tw, tx);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        return cudaSuccess;
    }
    template <bool DET, bool FUSED>
    static cudaError_t bwd_one(const BwdParams& prm_in, int bands, cudaStream_t st) {
        BwdParams prm = prm_in;
        auto kern = eqconv_bwd_kernel<K, DET, FUSED>;
        if constexpr (DET && !FUSED && K::VEC == 4) kern = eqconv_bwd_tiles_kernel<K>;
        static bool done[64] = {};
        constexpr int W = BwdShape<K, DET>::WARPS;
        constexpr int smem = W * BwdShape<K, DET>::L::BYTES;
        cudaError_t err = ensure_smem(kern, smem, done);
        if (err != cudaSuccess) return err;
        CUtensorMap tw, tg;
        const float* g = DET ? prm.gy : prm.x;
        if (!encode_rows_map(&tw, prm.w, (uint64_t)prm.E, K::NP, prm.C, K::TILE_C) ||
            !encode_rows_map(&tg, g, (uint64_t)prm.N, DET ? K::D_OUT : K::D_IN, prm.C, K::TILE_C))
            return cudaErrorInvalidValue;
        dim3 grid((prm.N + W - 1) / W, prm.T);
        for (int b = 0; b < bands; ++b) {
            prm.band_lo = (int)((int64_t)prm.N * b / bands);
            prm.band_hi = (int)((int64_t)prm.N * (b + 1) / bands);
            prm.accumulate = b > 0;
            kern<<<grid, W * 32, smem, st>>>(prm, tw, tg);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        return cudaSuccess;
    }
    static cudaError_t bwd(const BwdParams& prm, bool det, bool fused, int bands, cudaStream_t st) {
        if (det) return fused ? bwd_one<true, true>(prm, bands, st) : bwd_one<true, false>(prm, bands, st);
        return fused ? bwd_one<false, true>(prm, bands, st) : bwd_one<false, false>(prm, bands, st);
    }
    static constexpr KernelSet make() {
        return KernelSet{K::LIN, K::LSH, K::LOUT, K::VEC, K::MODE, K::TILE_C, K::G, &fwd, &bwd};
    }
};

}  // namespace eqc

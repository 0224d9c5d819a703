// Host-side launcher of the double backward for one kernel instance, and the
// instance table for one L_in (every L_sh and L_out in 0..3, natural-parity
// summed outputs, channel width 1 where an l = 3 block is present, else 2).
// Included by the eqc_dbl_l<L_in>.cu files with EQC_LIN set.
#pragma once

#include "eqc_dbl.cuh"
#include "eqc_launch.cuh"

#ifndef EQC_LIN
#error "EQC_LIN must be defined"
#endif

namespace eqc {

template <class K>
struct DblLaunch {
    static cudaError_t run(const DblParams& prm, const DblParams& send_prm, cudaStream_t st) {
        using LR = DblRing<K, true>;
        using LS = DblRing<K, false>;
        auto recv = eqconv_dbl_recv_kernel<K>;
        auto send = eqconv_dbl_send_kernel<K>;
        static bool done_recv[64] = {}, done_send[64] = {};
        cudaError_t err = ensure_smem(recv, LR::SMEM, done_recv);
        if (err == cudaSuccess) err = ensure_smem(send, LS::SMEM, done_send);
        if (err != cudaSuccess) return err;
        if (prm.N > 0) {
            // with no edges the edge maps are never read: give them a valid stand-in
            const bool edges = prm.E > 0;
            const void* wb = edges ? (const void*)prm.w : (const void*)prm.x;
            const void* bb = edges ? (const void*)prm.b : (const void*)prm.x;
            const uint64_t ne = edges ? (uint64_t)prm.E : (uint64_t)prm.N;
            const int nr = edges ? K::NP : K::D_IN;
            CUtensorMap tw, tb, tx, ta, tg;
            if (!encode_rows_map(&tw, wb, ne, nr, prm.C, K::TILE_C) ||
                !encode_rows_map(&tb, bb, ne, nr, prm.C, K::TILE_C) ||
                !encode_rows_map(&tx, prm.x, (uint64_t)prm.N, K::D_IN, prm.C, K::TILE_C) ||
                !encode_rows_map(&ta, prm.a, (uint64_t)prm.N, K::D_IN, prm.C, K::TILE_C) ||
                !encode_rows_map(&tg, prm.gy, (uint64_t)prm.N, K::D_OUT, prm.C, K::TILE_C))
                return cudaErrorInvalidValue;
            recv<<<dim3((prm.N + LR::WARPS - 1) / LR::WARPS, prm.T), LR::WARPS * 32, LR::SMEM, st>>>(prm, tw, tb, tx,
                                                                                                  ta);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
            send<<<dim3((prm.N + LS::WARPS - 1) / LS::WARPS, prm.T), LS::WARPS * 32, LS::SMEM, st>>>(send_prm, tw, tb,
                                                                                                  tg);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        if (prm.E > 0) {
            eqconv_dbl_r_epilogue<K::LSH><<<(prm.E + 255) / 256, 256, 0, st>>>(prm.part, prm.T, prm.r, prm.q, prm.g_r,
                                                                               prm.E);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        return cudaSuccess;
    }
    static constexpr DblKernelSet make() { return DblKernelSet{K::LIN, K::LSH, K::LOUT, K::VEC, K::TILE_C, K::G, &run}; }
};

#ifndef EQC_DBL_VEC
#define EQC_DBL_VEC 0   // channel width of every instance (0: 1 where an l = 3 block is present, else 2)
#endif
constexpr int dbl_vec(int lin, int lsh, int lout) { return EQC_DBL_VEC > 0 ? EQC_DBL_VEC : mode_vec(lin, lsh, lout); }

#define EQC_DI(LSH, LOUT) DblLaunch<Cfg<EQC_LIN, LSH, LOUT, dbl_vec(EQC_LIN, LSH, LOUT)>>::make()
#define EQC_DROW(LSH) {EQC_DI(LSH, 0), EQC_DI(LSH, 1), EQC_DI(LSH, 2), EQC_DI(LSH, 3)}
#define EQC_DNAME2(a) dbl_instances_l##a
#define EQC_DNAME(a) EQC_DNAME2(a)

const DblKernelSet* EQC_DNAME(EQC_LIN)(int lsh, int lout) {
    static const DblKernelSet table[4][4] = {EQC_DROW(0), EQC_DROW(1), EQC_DROW(2), EQC_DROW(3)};
    if (lsh < 0 || lsh > 3 || lout < 0 || lout > 3) return nullptr;
    return &table[lsh][lout];
}

}  // namespace eqc

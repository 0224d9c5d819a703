// Launchers of the convolution with on-chip radial weights for one
// (L_in, L_sh, L_out); included by the instantiation units.
#pragma once

#include <cuda_runtime.h>

#include "eqc_dispatch.h"
#include "eqc_radial.h"
#include "eqc_radial_bwd.cuh"
#include "eqc_radial_conv.cuh"
#include "eqc_radial_conv.h"

namespace eqc {

void count_launch();

namespace radial {

bool encode_f16_rows(CUtensorMap* map, const void* base, uint64_t rows, int box_rows);

template <int LIN, int LSH, int LOUT>
struct RadLaunch {
    using KS = Cfg<LIN, LSH, LOUT, 1, 0>;               // summed natural-parity layout
    using KP = Cfg<LIN, LSH, LOUT, 1, kModePerPath>;    // per-path blocks (the kernel's own output)

    static size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

    // radial workspace (W3 split, h2 by receiver position, per-edge factors)
    // followed by the per-path output blocks when the plan sums paths
    static size_t fwd_workspace(int N, int E, int C, bool per_path) {
        const size_t rad = up256(workspace_bytes(E, KP::NP * C));
        return rad + (per_path ? 0 : up256((size_t)N * KP::D_OUT * C * sizeof(float)));
    }

    static cudaError_t fwd(const RadFwdArgs& a, cudaStream_t st) {
        using S = RadFwdSmem<KP>;
        const int PC = KP::NP * a.C;
        const Workspace ws = carve(a.workspace, a.E, PC);
        float* y_pp = a.per_path ? a.y
                                 : reinterpret_cast<float*>(static_cast<char*>(a.workspace) +
                                                            up256(workspace_bytes(a.E, PC)));
        cudaError_t err = prepare(ws, a.r, a.recv_perm, a.E, a.W1, a.W2, a.W3, a.NB, a.rc, PC, st, nullptr,
                                  a.senders, a.receivers);
        if (err != cudaSuccess) return err;
        if (a.E > 0) {
            CUtensorMap ma_hi, ma_lo, mh_hi, mh_lo, mx;
            if (!encode_f16_rows(&ma_hi, ws.a_hi, (uint64_t)PC, 32) ||
                !encode_f16_rows(&ma_lo, ws.a_lo, (uint64_t)PC, 32) ||
                !encode_f16_rows(&mh_hi, ws.h_hi, (uint64_t)a.E, kEdgeTile) ||
                !encode_f16_rows(&mh_lo, ws.h_lo, (uint64_t)a.E, kEdgeTile) ||
                !encode_rows_map(&mx, a.x, (uint64_t)a.N, KP::D_IN, a.C, kSlice))
                return cudaErrorInvalidValue;
            static bool attr_done[64] = {};
            int dev = 0;
            if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
            if (dev >= 0 && dev < 64 && !attr_done[dev]) {
                err = cudaFuncSetAttribute(radial_conv_fwd_kernel<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           S::BYTES);
                if (err != cudaSuccess) return err;
                attr_done[dev] = true;
            }
            const int slices = a.C / kSlice, groups = (KP::NP + kGroupPaths - 1) / kGroupPaths;
            // about 4 waves of two CTAs per SM
            const long long want = 148LL * 2 * 4;
            int npc = (int)(((long long)a.N * slices * groups + want - 1) / want);
            if (npc < 1) npc = 1;
            RadFwdParams prm{a.x, a.recv_ptr, ws.rec, ws.ids, y_pp, a.N, a.C, a.E, npc, a.status};
            const dim3 grid((a.N + npc - 1) / npc, slices, groups);
            radial_conv_fwd_kernel<KP><<<grid, kConvThreads, S::BYTES, st>>>(prm, ma_hi, ma_lo, mh_hi, mh_lo, mx);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        } else {
            // no edges: every output row is zero
            const size_t bytes = (size_t)a.N * KP::D_OUT * a.C * sizeof(float);
            if ((err = cudaMemsetAsync(y_pp, 0, bytes, st)) != cudaSuccess) return err;
        }
        if (!a.per_path) {
            const int64_t total = (int64_t)a.N * KS::D_OUT * (a.C / 4);
            radial_sum_paths_kernel<KS, KP><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(y_pp, a.y, a.N, a.C);
            count_launch();
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        return cudaSuccess;
    }

    // ------------------------------------------------------------ backward

    static int bwd_slices(int C) { return C / kSlice; }
    static constexpr int bwd_groups() { return (KP::NP + kBwdGroupPaths - 1) / kBwdGroupPaths; }
    static int bwd_nodes_per_cta(int N, int C) {
        const long long want = 148LL * 2 * 4;   // about 4 waves of two CTAs per SM
        const int npc = (int)(((long long)N * bwd_slices(C) * bwd_groups() + want - 1) / want);
        return npc < 1 ? 1 : npc;
    }
    static constexpr int kEpiChunks = 16;   // 64-position chunks per epilogue CTA
    static int epi_ctas(int E) { return (E + kEpiTile * kEpiChunks - 1) / (kEpiTile * kEpiChunks); }

    struct BwdWs {
        Workspace rad;
        float* dx_pp;
        float* gy_part;
        float* gd_part;
        float* gw3_part;
        float* gw2_part;
        float* gw1_part;
        size_t bytes;
    };
    static BwdWs bwd_carve(void* ws, int N, int E, int C) {
        using R = BwdRows<KP>;
        BwdWs b{};
        const int PC = KP::NP * C;
        char* p = static_cast<char*>(ws);
        b.rad = carve(ws, E, PC);
        p += up256(workspace_bytes(E, PC));
        const int slices = bwd_slices(C), sg = slices * bwd_groups();
        const int ranges = (N + bwd_nodes_per_cta(N, C) - 1) / bwd_nodes_per_cta(N, C);
        b.dx_pp = reinterpret_cast<float*>(p);
        p += up256((size_t)N * R::DX_PP * C * 4);
        b.gy_part = reinterpret_cast<float*>(p);
        p += up256((size_t)E * slices * R::SD2 * 4);
        b.gd_part = reinterpret_cast<float*>(p);
        p += up256((size_t)sg * E * kH * 4);
        b.gw3_part = reinterpret_cast<float*>(p);
        p += up256((size_t)(ranges > 0 ? ranges : 1) * PC * kH * 4);
        b.gw2_part = reinterpret_cast<float*>(p);
        p += up256((size_t)(epi_ctas(E) > 0 ? epi_ctas(E) : 1) * kH * kH * 4);
        b.gw1_part = reinterpret_cast<float*>(p);
        p += up256((size_t)(epi_ctas(E) > 0 ? epi_ctas(E) : 1) * kMaxBasis * kH * 4);
        b.bytes = (size_t)(p - static_cast<char*>(ws));
        return b;
    }
    static size_t bwd_workspace(int N, int E, int C) { return bwd_carve(nullptr, N, E, C).bytes; }

    template <class KG>   // KG: the Cfg of gy's layout (summed or per-path)
    static cudaError_t bwd_impl(const RadBwdArgs& a, cudaStream_t st) {
        using S = RadBwdSmem<KG>;
        const int PC = KP::NP * a.C;
        const BwdWs b = bwd_carve(a.workspace, a.N, a.E, a.C);
        float* scal = b.rad.inv_scale;     // [0] 2^-sA, [1..3] maxima bits
        unsigned* sbits = reinterpret_cast<unsigned*>(scal);
        cudaError_t err;
        if (a.E == 0) {   // no edges: every gradient is zero
            if ((err = cudaMemsetAsync(a.dx, 0, (size_t)a.N * KP::D_IN * a.C * 4, st)) != cudaSuccess) return err;
            if ((err = cudaMemsetAsync(a.gW1, 0, (size_t)a.NB * kH * 4, st)) != cudaSuccess) return err;
            if ((err = cudaMemsetAsync(a.gW2, 0, (size_t)kH * kH * 4, st)) != cudaSuccess) return err;
            return cudaMemsetAsync(a.gW3, 0, (size_t)kH * PC * 4, st);
        }
        if ((err = cudaMemsetAsync(sbits + 1, 0, 3 * sizeof(unsigned), st)) != cudaSuccess) return err;
        const int64_t nx4 = (int64_t)a.N * KP::D_IN * a.C / 4, ng4 = (int64_t)a.N * KG::D_OUT * a.C / 4;
        radial_absmax_kernel<<<296, 256, 0, st>>>(a.x, nx4, sbits + 1);
        count_launch();
        radial_absmax_kernel<<<296, 256, 0, st>>>(a.gy, ng4, sbits + 2);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        err = prepare(b.rad, a.r, a.send_perm, a.E, a.W1, a.W2, a.W3, a.NB, a.rc, PC, st, sbits + 3, a.receivers,
                      a.senders);
        if (err != cudaSuccess) return err;
        CUtensorMap ma_hi, ma_lo, mh_hi, mh_lo, mg;
        if (!encode_f16_rows(&ma_hi, b.rad.a_hi, (uint64_t)PC, 32) ||
            !encode_f16_rows(&ma_lo, b.rad.a_lo, (uint64_t)PC, 32) ||
            !encode_f16_rows(&mh_hi, b.rad.h_hi, (uint64_t)a.E, kEdgeTile) ||
            !encode_f16_rows(&mh_lo, b.rad.h_lo, (uint64_t)a.E, kEdgeTile) ||
            !encode_rows_map(&mg, a.gy, (uint64_t)a.N, KG::D_OUT, a.C, kSlice))
            return cudaErrorInvalidValue;
        static bool attr_done[64] = {};
        int dev = 0;
        if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
        if (dev >= 0 && dev < 64 && !attr_done[dev]) {
            err = cudaFuncSetAttribute(radial_conv_bwd_kernel<KG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       S::BYTES);
            if (err != cudaSuccess) return err;
            err = cudaFuncSetAttribute(radial_bwd_epilogue_kernel<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kEpiSmemBytes);
            if (err != cudaSuccess) return err;
            attr_done[dev] = true;
        }
        const int slices = bwd_slices(a.C), groups = bwd_groups(), npc = bwd_nodes_per_cta(a.N, a.C);
        const int ranges = (a.N + npc - 1) / npc;
        RadBwdParams prm{a.x, a.gy, a.send_ptr, b.rad.rec, b.rad.ids, scal, b.dx_pp, b.gy_part, b.gd_part,
                         b.gw3_part, a.N, a.C, a.E, npc, a.status};
        radial_conv_bwd_kernel<KG><<<dim3(ranges, slices, groups), kBwdThreads, S::BYTES, st>>>(prm, ma_hi, ma_lo,
                                                                                               mh_hi, mh_lo, mg);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        const int64_t ndx = (int64_t)a.N * KP::D_IN * (a.C / 4);
        radial_sum_dx_kernel<KP><<<(unsigned)((ndx + 255) / 256), 256, 0, st>>>(b.dx_pp, a.dx, a.N, a.C);
        count_launch();
        const int ne = epi_ctas(a.E);
        radial_bwd_epilogue_kernel<KP><<<ne, kEpiThreads, kEpiSmemBytes, st>>>(a.r, a.send_perm, a.E, a.W1, a.W2, a.NB, a.rc,
                                                                   scal, b.rad.zscale, b.gy_part, slices, b.gd_part,
                                                                   slices * groups, kEpiChunks, a.dr, b.gw1_part,
                                                                   b.gw2_part);
        count_launch();
        radial_sum_parts_kernel<<<(kH * kH + 255) / 256, 256, 0, st>>>(b.gw2_part, ne, (int64_t)kH * kH,
                                                                      (int64_t)kH * kH, a.gW2);
        count_launch();
        radial_sum_parts_kernel<<<(a.NB * kH + 255) / 256, 256, 0, st>>>(b.gw1_part, ne, (int64_t)kMaxBasis * kH,
                                                                        (int64_t)a.NB * kH, a.gW1);
        count_launch();
        radial_sum_gw3_kernel<<<(unsigned)(((int64_t)PC * kH + 255) / 256), 256, 0, st>>>(b.gw3_part, ranges, PC,
                                                                                          scal, a.gW3);
        count_launch();
        return cudaGetLastError();
    }

    static cudaError_t bwd(const RadBwdArgs& a, cudaStream_t st) {
        return a.per_path ? bwd_impl<KP>(a, st) : bwd_impl<KS>(a, st);
    }

    static constexpr RadConvSet make() {
        return RadConvSet{LIN, LSH, LOUT, KP::NP, KP::D_OUT, &fwd_workspace, &fwd, &bwd_workspace, &bwd};
    }
};

}  // namespace radial
}  // namespace eqc

// Launchers of the convolution with on-chip radial weights for one
// (L_in, L_sh, L_out); included by the instantiation units.
#pragma once

#include <cuda_runtime.h>

#include "eqc_dispatch.h"
#include "eqc_radial.h"
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
        cudaError_t err = prepare(ws, a.r, a.recv_perm, a.E, a.W1, a.W2, a.W3, a.NB, a.rc, PC, st);
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
            // about 4 waves of one CTA per SM
            const long long want = 148LL * 4;
            int npc = (int)(((long long)a.N * slices * groups + want - 1) / want);
            if (npc < 1) npc = 1;
            RadFwdParams prm{a.x, a.r, a.recv_ptr, a.recv_perm, a.senders, ws.uscale, y_pp, a.N, a.C, a.E, npc,
                             a.status};
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

    static constexpr RadConvSet make() { return RadConvSet{LIN, LSH, LOUT, KP::NP, KP::D_OUT, &fwd_workspace, &fwd}; }
};

}  // namespace radial
}  // namespace eqc

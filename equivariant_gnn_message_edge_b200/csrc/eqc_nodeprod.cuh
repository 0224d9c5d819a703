// Node-local channel-diagonal tensor product, forward and backward (device
// code).
//
// FlashCart (arXiv 2610.06409) §5, App. B and App. D: the correlation ladder
// builds higher-order features by repeated pairwise products at each atom;
// each step couples same-index channels of two node features along the
// admissible paths and keeps every path's output or sums weighted paths.
// For u [N][D_u][C], v [N][D_v][C] and weights w [P][C] (none: all ones):
//   y[i, o3(p)+m3, c] = sum_p w[p,c] sum_{m1,m2} C_p[m1,m2,m3] u[i,l1 m1,c] v[i,l2 m2,c]
//   du[i, l1 m1, c]   = sum_p w[p,c] sum_{m2,m3} C_p v[i,l2 m2,c] gy[i,o3+m3,c]
//   dv[i, l2 m2, c]   = sum_p w[p,c] sum_{m1,m3} C_p u[i,l1 m1,c] gy[i,o3+m3,c]
//   dw[p, c]          = sum_i sum C_p u v gy
// The paths are those of the convolution with L_sh = L_v (v's irreps are a
// natural-parity prefix, like the harmonics), so Cfg<L_u, L_v, L_out, VEC,
// MODE> and its compile-time CG serve both ops.
//
// One warp = one channel tile of one node at a time; warps walk the nodes
// with a fixed grid stride, so each warp's dw partial covers a fixed node
// set and the final sum over warps (in warp order) is bitwise reproducible.
// The op streams u, v and y (gy, du, dv) once: it is HBM-bound at l <= 2.
#pragma once

#include "eqc_conv.cuh"

namespace eqc {

struct NpParams {
    const float* u;
    const float* v;
    const float* w;       // [P][C] or null (all ones)
    const float* gy;
    float* y;
    float* du;
    float* dv;
    float* dw_part;       // [warps][P][C] partials of dw
    float* dw;            // [P][C]
    int N, C, warps;      // warps = gridDim.x * warps per CTA
};

constexpr int kNpWarps = 4;

template <int V, int R>
__device__ __forceinline__ void np_load(float (&d)[R][V], const float* base, int C, bool on) {
#pragma unroll
    for (int k = 0; k < R; ++k) {
        if (on) {
            ld_stream<V>(d[k], base + (size_t)k * C, policy_evict_first());
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) d[k][v] = 0.f;
        }
    }
}

template <class K>
__device__ __forceinline__ void np_weights(float (&wv)[K::NP][K::VEC], const float* w, int C, int c, bool on) {
#pragma unroll
    for (int p = 0; p < K::NP; ++p)
#pragma unroll
        for (int v = 0; v < K::VEC; ++v) wv[p][v] = (w && on) ? w[(size_t)p * C + c + v] : 1.f;
}

template <class K>
__global__ void __launch_bounds__(kNpWarps * 32) eqconv_np_fwd_kernel(const NpParams prm) {
    constexpr int V = K::VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = prm.C, c = blockIdx.y * K::TILE_C + lane * V;
    const bool on = c < C;
    float wv[K::NP][V];
    np_weights<K>(wv, prm.w, C, c, on);
    for (int i = blockIdx.x * kNpWarps + warp; i < prm.N; i += gridDim.x * kNpWarps) {
        float uv[K::D_IN][V], vv[K::D_SH][V], y[K::D_OUT][V];
        np_load<V>(uv, prm.u + (size_t)i * K::D_IN * C + c, C, on);
        np_load<V>(vv, prm.v + (size_t)i * K::D_SH * C + c, C, on);
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d)
#pragma unroll
            for (int q = 0; q < V; ++q) y[d][q] = 0.f;
        static_for<K::NP>([&](auto pc) {
            constexpr int p = EQC_CV(pc);
            constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
            constexpr int o1 = l1 * l1, o2 = l2 * l2, o3 = K::PL.o3[p];
            static_for<2 * l3 + 1>([&](auto m3c) {
                constexpr int m3 = EQC_CV(m3c);
                float t[V];
#pragma unroll
                for (int q = 0; q < V; ++q) t[q] = 0.f;
                static_for<2 * l1 + 1>([&](auto m1c) {
                    constexpr int m1 = EQC_CV(m1c);
                    static_for<2 * l2 + 1>([&](auto m2c) {
                        constexpr int m2 = EQC_CV(m2c);
                        constexpr double cg = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                        if constexpr (cg != 0.0) {
#pragma unroll
                            for (int q = 0; q < V; ++q)
                                t[q] = fmaf((float)cg * uv[o1 + m1][q], vv[o2 + m2][q], t[q]);
                        }
                    });
                });
#pragma unroll
                for (int q = 0; q < V; ++q) y[o3 + m3][q] = fmaf(wv[p][q], t[q], y[o3 + m3][q]);
            });
        });
        if (on) {
            float* yi = prm.y + (size_t)i * K::D_OUT * C + c;
#pragma unroll
            for (int d = 0; d < K::D_OUT; ++d) st_stream<V>(yi + (size_t)d * C, y[d]);
        }
    }
}

template <class K>
__global__ void __launch_bounds__(kNpWarps * 32) eqconv_np_bwd_kernel(const NpParams prm) {
    constexpr int V = K::VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = prm.C, c = blockIdx.y * K::TILE_C + lane * V;
    const bool on = c < C;
    float wv[K::NP][V], dwa[K::NP][V];
    np_weights<K>(wv, prm.w, C, c, on);
#pragma unroll
    for (int p = 0; p < K::NP; ++p)
#pragma unroll
        for (int q = 0; q < V; ++q) dwa[p][q] = 0.f;
    for (int i = blockIdx.x * kNpWarps + warp; i < prm.N; i += gridDim.x * kNpWarps) {
        float uv[K::D_IN][V], vv[K::D_SH][V], g[K::D_OUT][V], du[K::D_IN][V], dv[K::D_SH][V];
        np_load<V>(uv, prm.u + (size_t)i * K::D_IN * C + c, C, on);
        np_load<V>(vv, prm.v + (size_t)i * K::D_SH * C + c, C, on);
        np_load<V>(g, prm.gy + (size_t)i * K::D_OUT * C + c, C, on);
#pragma unroll
        for (int d = 0; d < K::D_IN; ++d)
#pragma unroll
            for (int q = 0; q < V; ++q) du[d][q] = 0.f;
#pragma unroll
        for (int d = 0; d < K::D_SH; ++d)
#pragma unroll
            for (int q = 0; q < V; ++q) dv[d][q] = 0.f;
        static_for<K::NP>([&](auto pc) {
            constexpr int p = EQC_CV(pc);
            constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
            constexpr int o1 = l1 * l1, o2 = l2 * l2, o3 = K::PL.o3[p];
            float wg[2 * l3 + 1][V];     // w_p gy on the path's output rows
#pragma unroll
            for (int m3 = 0; m3 < 2 * l3 + 1; ++m3)
#pragma unroll
                for (int q = 0; q < V; ++q) wg[m3][q] = wv[p][q] * g[o3 + m3][q];
            float s[V];
#pragma unroll
            for (int q = 0; q < V; ++q) s[q] = 0.f;
            static_for<2 * l1 + 1>([&](auto m1c) {
                constexpr int m1 = EQC_CV(m1c);
                static_for<2 * l2 + 1>([&](auto m2c) {
                    constexpr int m2 = EQC_CV(m2c);
                    static_for<2 * l3 + 1>([&](auto m3c) {
                        constexpr int m3 = EQC_CV(m3c);
                        constexpr double cg = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                        if constexpr (cg != 0.0) {
#pragma unroll
                            for (int q = 0; q < V; ++q) {
                                const float cw = (float)cg * wg[m3][q];
                                du[o1 + m1][q] = fmaf(cw, vv[o2 + m2][q], du[o1 + m1][q]);
                                dv[o2 + m2][q] = fmaf(cw, uv[o1 + m1][q], dv[o2 + m2][q]);
                                const float cu = (float)cg * uv[o1 + m1][q];
                                s[q] = fmaf(cu * vv[o2 + m2][q], g[o3 + m3][q], s[q]);
                            }
                        }
                    });
                });
            });
#pragma unroll
            for (int q = 0; q < V; ++q) dwa[p][q] += s[q];
        });
        if (on) {
            float* di = prm.du + (size_t)i * K::D_IN * C + c;
#pragma unroll
            for (int d = 0; d < K::D_IN; ++d) st_stream<V>(di + (size_t)d * C, du[d]);
            float* dvi = prm.dv + (size_t)i * K::D_SH * C + c;
#pragma unroll
            for (int d = 0; d < K::D_SH; ++d) st_stream<V>(dvi + (size_t)d * C, dv[d]);
        }
    }
    if (prm.dw_part && on) {
        float* pp = prm.dw_part + (size_t)(blockIdx.x * kNpWarps + warp) * K::NP * C + c;
#pragma unroll
        for (int p = 0; p < K::NP; ++p) st_plain<V>(pp + (size_t)p * C, dwa[p]);
    }
}

// dw[p, c] = sum over warps (in order) of the partials; one thread per (p, c).
template <int = 0>
__global__ void eqconv_np_dw_reduce(const float* dw_part, int warps, int PC, float* dw) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= PC) return;
    float s = 0.f;
    for (int j = 0; j < warps; ++j) s += dw_part[(size_t)j * PC + k];
    dw[k] = s;
}

}  // namespace eqc

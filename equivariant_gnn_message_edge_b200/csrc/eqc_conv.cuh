// Fused kernels of the equivariant message-passing convolution (sm_100a).
//
// e3j (arXiv 2609.35099), abstract / Table 1: the convolution of MACE-style
// potentials, forward and backward.  FlashCart (arXiv 2610.06409) §4 and
// App. D: a receiver-sorted forward that gives each program a receiver and a
// channel tile, sums its incoming edges locally and stores each result once
// (no atomics, no per-edge message tensors); a VJP whose shared input
// gradient is either accumulated with atomics (receiver order) or, ordered by
// sender, deterministically; weight gradients stored directly.
//
// Mapping (one warp = one node x one channel tile of 32*VEC channels; each
// lane owns VEC consecutive channels, so every x / w / y row segment is a
// coalesced 512 B (VEC=4) run):
//   * a warp walks its node's edge list in windows of up to 32 edges; lane 0
//     keeps a 2-stage shared-memory ring filled by TMA bulk copies of each
//     edge's rows (w_e and the gathered x_s or gy_i) two edges ahead;
//   * in chunks (Cfg::chunk) lane t evaluates Y(r_e) of edge t and, for the
//     forward, the per-edge coupling matrices
//       A_p[m3][m1] = sum_m2 C_p[m1,m2,m3] Y_{l2 m2}(r_e)        (l2 > 0)
//     with the CG as compile-time immediates (zeros skipped) into shared
//     memory; paths with l2 = 0 have A = identity;
//   * forward:  acc[l3 m3] += w_p * sum_m1 A_p[m3][m1] x[s, l1 m1]
//   * backward (per channel): h[m1][m2] = sum_m3 C_p[m1,m2,m3] gy_i[m3],
//               t[m1] = sum_m2 Y[m2] h = (A_p^T gy_i)[m1],  dw_p = x_s . t,
//               dx_s += w_p t,  gY[l2 m2] += w_p sum_m1 x_s[m1] h
//     (gY summed over the lane's channels, then across the warp by a fixed
//     butterfly; dr = (dY/dr)^T gY).
// Streams (w read, dw written) carry L2 evict-first hints; gathered rows
// (x or gy, reused ~45 times) carry evict-last hints.
#pragma once

#include <cuda.h>

#include <cstdint>
#include <type_traits>
#include <utility>

#include "eqc_sh.cuh"
#include "eqc_tables.h"

// Build-time tuning knobs (defaults are the tuned values).
#ifndef EQC_STAGES
#define EQC_STAGES 2
#endif
#ifndef EQC_CHUNK_SMALL
#define EQC_CHUNK_SMALL 0   // 0: 16 edges at VEC=4, 8 at narrower tiles
#endif
#ifndef EQC_CHUNK_LARGE
#define EQC_CHUNK_LARGE 4   // edges per coupling sub-batch when A is large (l = 3)
#endif
#ifndef EQC_CHUNK_LARGE_ATOMIC
#define EQC_CHUNK_LARGE_ATOMIC 8   // the same for the atomic backward (register-bound, 2 CTAs/SM)
#endif
#ifndef EQC_BWD_H
#define EQC_BWD_H 1         // 1: the backward takes t = A^T g from h = C.g (no coupling matrices)
#endif
#ifndef EQC_CHUNK_BWD_H
#define EQC_CHUNK_BWD_H 0   // edges per harmonics batch of that backward (0: as the coupling batch)
#endif
#ifndef EQC_FWD_PRED
#define EQC_FWD_PRED 1      // 1: predicate the forward row reads at VEC = 4; 2: at every width
#endif

namespace eqc {

#define EQC_CV(x) std::decay_t<decltype(x)>::value

template <class F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
    (f(std::integral_constant<int, Is>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

constexpr int pad_odd4(int n) {
    int m = n < 4 ? 4 : ((n + 3) & ~3);
    if (((m / 4) & 1) == 0) m += 4;
    return m;
}

// MODE: output variant bits (kModeAllParity, kModePerPath; 0 = natural-parity
// outputs summed over paths).
template <int LIN_, int LSH_, int LOUT_, int VEC_, int MODE_ = 0>
struct Cfg {
    static constexpr int LIN = LIN_, LSH = LSH_, LOUT = LOUT_, VEC = VEC_, MODE = MODE_;
    static constexpr PathList PL = make_paths(LIN, LSH, LOUT, MODE);
    static constexpr int NP = PL.n;
    static constexpr int D_IN = (LIN + 1) * (LIN + 1);
    static constexpr int D_SH = (LSH + 1) * (LSH + 1);
    static constexpr int D_OUT = PL.dout;
    static constexpr int G = D_SH - 1;              // dr needs gY for l2 > 0 only
    static constexpr AOffsets AO = make_aoffsets(PL);
    static constexpr int NA = AO.total;
    static constexpr int NA_PAD = pad_odd4(NA);     // row stride; NA_PAD/4 odd: conflict-free STS.128
    // edges whose coupling matrices A sit in shared memory at a time; the
    // atomic backward is held to two CTAs per SM by its registers, so it
    // takes the larger batch, the other kernels gain occupancy from a small one
    static constexpr int chunk(bool atomic_bwd) {
        return NA_PAD > 128 ? (atomic_bwd ? EQC_CHUNK_LARGE_ATOMIC : EQC_CHUNK_LARGE)
                            : (EQC_CHUNK_SMALL > 0 ? EQC_CHUNK_SMALL : (VEC >= 4 ? 16 : 8));
    }
    static constexpr int GS = G | 1;                // gY row stride in shared memory (odd)
    static constexpr int YS = pad_odd4(D_SH);       // harmonics row (backward without coupling matrices)
    static constexpr int A_ROW = NA_PAD > YS ? NA_PAD : YS;   // coupling-batch row stride in shared memory
    static constexpr int TILE_C = 32 * VEC;
    static constexpr int STAGES = EQC_STAGES;       // edges staged ahead per warp (ring depth)
    static_assert(NP > 0, "no admissible path");
};

// ---------------------------------------------------------------- memory ops

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

template <int VEC>
__device__ __forceinline__ void ld_stream(float* d, const float* p, uint64_t pol) {
    if constexpr (VEC == 1) {
        asm("ld.global.nc.L1::no_allocate.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(d[0]) : "l"(p), "l"(pol));
    } else if constexpr (VEC == 4) {
        asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "l"(p), "l"(pol));
    } else {
        asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.f32 {%0,%1}, [%2], %3;"
            : "=f"(d[0]), "=f"(d[1])
            : "l"(p), "l"(pol));
    }
}
template <int VEC>
__device__ __forceinline__ void ld_keep(float* d, const float* p, uint64_t pol) {
    if constexpr (VEC == 1) {
        asm("ld.global.nc.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(d[0]) : "l"(p), "l"(pol));
    } else if constexpr (VEC == 4) {
        asm("ld.global.nc.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "l"(p), "l"(pol));
    } else {
        asm("ld.global.nc.L2::cache_hint.v2.f32 {%0,%1}, [%2], %3;"
            : "=f"(d[0]), "=f"(d[1])
            : "l"(p), "l"(pol));
    }
}
template <int VEC>
__device__ __forceinline__ void st_plain(float* p, const float* v) {
    if constexpr (VEC == 1)
        *p = v[0];
    else if constexpr (VEC == 4)
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}
template <int VEC>
__device__ __forceinline__ void st_stream(float* p, const float* v) {
    if constexpr (VEC == 1)
        __stcs(p, v[0]);
    else if constexpr (VEC == 4)
        __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    else
        __stcs(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
}
template <int VEC>
__device__ __forceinline__ void red_add(float* p, const float* v) {
    if constexpr (VEC == 1)
        atomicAdd(p, v[0]);
    else if constexpr (VEC == 4)
        atomicAdd(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    else
        atomicAdd(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
}

template <int V>
__device__ __forceinline__ void lds_vec(float* d, const float* p) {
    if constexpr (V == 1) {
        d[0] = *p;
    } else if constexpr (V == 4) {
        const float4 t = *reinterpret_cast<const float4*>(p);
        d[0] = t.x;
        d[1] = t.y;
        d[2] = t.z;
        d[3] = t.w;
    } else {
        const float2 t = *reinterpret_cast<const float2*>(p);
        d[0] = t.x;
        d[1] = t.y;
    }
}

// ------------------------------------------------------- per-edge coupling A

template <int L1, int L2, int L3>
constexpr bool cg_row_nonzero(int m1, int m2) {
    for (int m3 = 0; m3 < 2 * L3 + 1; ++m3)
        if (RealCG<L1, L2, L3>::t.v[m1][m2][m3] != 0.0) return true;
    return false;
}

// Arow[AO.off[p] + m3*(2l1+1) + m1] = sum_m2 C_p[m1,m2,m3] Y[l2^2 + m2]
template <class K>
__device__ __forceinline__ void compute_A(const float* Y, float* Arow) {
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        if constexpr (l2 > 0) {
            constexpr int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1, o2 = l2 * l2;
            constexpr int n4 = (d1 * d3 + 3) / 4;
            constexpr int off = K::AO.off[p];
            float a[n4 * 4];
#pragma unroll
            for (int q = d1 * d3; q < n4 * 4; ++q) a[q] = 0.f;
            static_for<d3>([&](auto m3c) {
                static_for<d1>([&](auto m1c) {
                    constexpr int m1 = EQC_CV(m1c), m3 = EQC_CV(m3c);
                    float s = 0.f;
                    static_for<d2>([&](auto m2c) {
                        constexpr int m2 = EQC_CV(m2c);
                        constexpr double c = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                        if constexpr (c != 0.0) s = fmaf((float)c, Y[o2 + m2], s);
                    });
                    a[m3 * d1 + m1] = s;
                });
            });
#pragma unroll
            for (int q = 0; q < n4; ++q)
                reinterpret_cast<float4*>(Arow + off)[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
        }
    });
}

template <int N4>
__device__ __forceinline__ void load_A(const float* src, float* a) {
#pragma unroll
    for (int q = 0; q < N4; ++q) {
        const float4 t = reinterpret_cast<const float4*>(src)[q];
        a[4 * q] = t.x;
        a[4 * q + 1] = t.y;
        a[4 * q + 2] = t.z;
        a[4 * q + 3] = t.w;
    }
}

// ------------------------------------------------------------ forward math

template <class K>
__device__ __forceinline__ void fwd_edge(const float* As, const float (&xv)[K::D_IN][K::VEC],
                                         const float (&wv)[K::NP][K::VEC], float (&acc)[K::D_OUT][K::VEC]) {
    constexpr int V = K::VEC;
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o3 = K::PL.o3[p];
        if constexpr (l2 == 0) {
            static_assert(l1 == l3, "l x 0 -> l");
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) acc[o3 + m][v] = fmaf(wv[p][v], xv[o1 + m][v], acc[o3 + m][v]);
        } else {
            constexpr int n4 = (d1 * d3 + 3) / 4;
            constexpr int aoff = K::AO.off[p];
            float a[n4 * 4];
            load_A<n4>(As + aoff, a);
            if constexpr (d1 <= d3) {
                float u[d1][V];
#pragma unroll
                for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
                    for (int v = 0; v < V; ++v) u[m1][v] = wv[p][v] * xv[o1 + m1][v];
#pragma unroll
                for (int m3 = 0; m3 < d3; ++m3)
#pragma unroll
                    for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
                        for (int v = 0; v < V; ++v)
                            acc[o3 + m3][v] = fmaf(a[m3 * d1 + m1], u[m1][v], acc[o3 + m3][v]);
            } else {
#pragma unroll
                for (int m3 = 0; m3 < d3; ++m3) {
                    float t[V];
#pragma unroll
                    for (int v = 0; v < V; ++v) t[v] = a[m3 * d1] * xv[o1][v];
#pragma unroll
                    for (int m1 = 1; m1 < d1; ++m1)
#pragma unroll
                        for (int v = 0; v < V; ++v) t[v] = fmaf(a[m3 * d1 + m1], xv[o1 + m1][v], t[v]);
#pragma unroll
                    for (int v = 0; v < V; ++v) acc[o3 + m3][v] = fmaf(wv[p][v], t[v], acc[o3 + m3][v]);
                }
            }
        }
    });
}

// ----------------------------------------------------------- backward math

// Row accessors for the per-edge math: a row block lives either in registers
// (the warp's resident node) or in the shared-memory stage of the edge; the
// math asks for one row (component) at a time so that only the rows of the
// current path are live in registers.
template <int V, int D>
struct RegRows {
    const float (&r)[D][V];
    __device__ __forceinline__ void get(int d, float* out) const {
#pragma unroll
        for (int v = 0; v < V; ++v) out[v] = r[d][v];
    }
};
template <int V>
struct SmemRows {
    const float* base;  // row 0 of this lane's channels
    int stride;         // floats between rows
    bool on;            // false: rows read as zero (inactive lane)
    __device__ __forceinline__ void get(int d, float* out) const {
        if (on) {
            lds_vec<V>(out, base + d * stride);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) out[v] = 0.f;
        }
    }
};

// One edge of the backward: with x (sender rows), g (receiver output-gradient
// rows) and w (weight rows) given by accessors,
//   t_p = A_p^T g_l3,  dw_p = x_l1 . t_p (stored through store_dw),
//   dx_l1 += w_p t_p,  gyl[l2 m2] += w_p sum_{m1,m3} C_p[m1,m2,m3] x[m1] g[m3]
// (gyl is this lane's partial over its channels).
// DIRECT: dx accumulates straight into dx_full (the deterministic pass keeps
// its sender's dx in registers).  Otherwise the dx of one input block (paths
// are ordered by l1) is summed in a small block and handed to
// dx_sink(o1, d1, block) after the block's last path (atomic pass).
template <class K, bool DIRECT, class XR, class GR, class WR, class StoreDw, class DxSink>
__device__ __forceinline__ void bwd_edge(const float* As, const XR& X, const GR& Gr, const WR& Wr,
                                         float (&dx_full)[DIRECT ? K::D_IN : 1][K::VEC], DxSink&& dx_sink,
                                         float (&gyl)[K::G > 0 ? K::G : 1], StoreDw&& store_dw) {
    constexpr int V = K::VEC;
    float dxg[DIRECT ? 1 : 2 * kMaxL + 1][V];
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o3 = K::PL.o3[p];
        [[maybe_unused]] constexpr bool first_of_block = (p == 0) || (K::PL.l1[p == 0 ? 0 : p - 1] != l1);
        [[maybe_unused]] constexpr bool last_of_block = (p == K::NP - 1) || (K::PL.l1[p + 1 < K::NP ? p + 1 : p] != l1);
        if constexpr (!DIRECT && first_of_block) {
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) dxg[m][v] = 0.f;
        }
        float gv[d3][V], xv[d1][V], wp[V];
#pragma unroll
        for (int m = 0; m < d3; ++m) Gr.get(o3 + m, gv[m]);
#pragma unroll
        for (int m = 0; m < d1; ++m) X.get(o1 + m, xv[m]);
        Wr.get(p, wp);
        float t[d1][V];
        [[maybe_unused]] float hG[(l2 > 0 && EQC_BWD_H) ? 2 * l2 + 1 : 1][V];   // sum_m1 x[m1] h[m1][m2]
        if constexpr (l2 == 0) {
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) t[m][v] = gv[m][v];
        } else if constexpr (EQC_BWD_H) {
            // h[m1][m2] = sum_m3 C_p[m1,m2,m3] g[m3] gives both t[m1] = sum_m2 Y[m2] h
            // (= (A_p^T g)[m1]) and the harmonic gradient sum_m1 x[m1] h
            constexpr int d2 = 2 * l2 + 1, o2 = l2 * l2;
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) t[m][v] = 0.f;
#pragma unroll
            for (int m = 0; m < d2; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) hG[m][v] = 0.f;
            static_for<d2>([&](auto m2c) {
                constexpr int m2 = EQC_CV(m2c);
                const float y2 = As[o2 + m2];                 // this edge's Y, broadcast
                static_for<d1>([&](auto m1c) {
                    constexpr int m1 = EQC_CV(m1c);
                    if constexpr (cg_row_nonzero<l1, l2, l3>(m1, m2)) {
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            float h = 0.f;
                            static_for<d3>([&](auto m3c) {
                                constexpr int m3 = EQC_CV(m3c);
                                constexpr double c = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                                if constexpr (c != 0.0) h = fmaf((float)c, gv[m3][v], h);
                            });
                            t[m1][v] = fmaf(y2, h, t[m1][v]);
                            hG[m2][v] = fmaf(xv[m1][v], h, hG[m2][v]);
                        }
                    }
                });
            });
        } else {
            constexpr int n4 = (d1 * d3 + 3) / 4;
            constexpr int aoff = K::AO.off[p];
            float a[n4 * 4];
            load_A<n4>(As + aoff, a);
#pragma unroll
            for (int m1 = 0; m1 < d1; ++m1) {
#pragma unroll
                for (int v = 0; v < V; ++v) t[m1][v] = a[m1] * gv[0][v];
#pragma unroll
                for (int m3 = 1; m3 < d3; ++m3)
#pragma unroll
                    for (int v = 0; v < V; ++v) t[m1][v] = fmaf(a[m3 * d1 + m1], gv[m3][v], t[m1][v]);
            }
        }
        float dw[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float s = xv[0][v] * t[0][v];
#pragma unroll
            for (int m1 = 1; m1 < d1; ++m1) s = fmaf(xv[m1][v], t[m1][v], s);
            dw[v] = s;
        }
        store_dw(p, dw);
        if constexpr (DIRECT) {
#pragma unroll
            for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
                for (int v = 0; v < V; ++v) dx_full[o1 + m1][v] = fmaf(wp[v], t[m1][v], dx_full[o1 + m1][v]);
        } else {
#pragma unroll
            for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
                for (int v = 0; v < V; ++v) dxg[m1][v] = fmaf(wp[v], t[m1][v], dxg[m1][v]);
            if constexpr (last_of_block) dx_sink(o1, d1, dxg);
        }
        if constexpr (l2 > 0 && EQC_BWD_H) {
            constexpr int d2 = 2 * l2 + 1, o2 = l2 * l2;
#pragma unroll
            for (int m2 = 0; m2 < d2; ++m2) {
                float gsum = 0.f;
#pragma unroll
                for (int v = 0; v < V; ++v) gsum = fmaf(wp[v], hG[m2][v], gsum);
                gyl[o2 + m2 - 1] += gsum;
            }
        } else if constexpr (l2 > 0) {
            constexpr int d2 = 2 * l2 + 1, o2 = l2 * l2;
            static_for<d2>([&](auto m2c) {
                constexpr int m2 = EQC_CV(m2c);
                float gsum = 0.f;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float g = 0.f;
                    static_for<d1>([&](auto m1c) {
                        constexpr int m1 = EQC_CV(m1c);
                        if constexpr (cg_row_nonzero<l1, l2, l3>(m1, m2)) {
                            float s = 0.f;
                            static_for<d3>([&](auto m3c) {
                                constexpr int m3 = EQC_CV(m3c);
                                constexpr double c = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                                if constexpr (c != 0.0) s = fmaf((float)c, gv[m3][v], s);
                            });
                            g = fmaf(xv[m1][v], s, g);
                        }
                    });
                    gsum = fmaf(wp[v], g, gsum);
                }
                gyl[o2 + m2 - 1] += gsum;
            });
        }
    });
}

// --------------------------------------------------------------- parameters

struct FwdParams {
    const float* x;
    const float* r;
    const float* w;
    float* y;
    const int* ptr;    // recv_ptr
    const int* perm;   // recv_perm
    const int* other;  // senders
    int N, C, E;
    int band_lo, band_hi;  // only edges whose sender is in [band_lo, band_hi)
    int accumulate;        // 0: y = sum over the band; 1: y += sum over the band
    unsigned* status;
};

struct BwdParams {
    const float* x;
    const float* r;
    const float* w;
    const float* gy;
    float* dx;
    float* dw;
    float* dr;
    float* gy_part;    // [E][T][G] when the dr reduction spans channel tiles
    const int* ptr;    // DET: send_ptr   ATOMIC: recv_ptr
    const int* perm;   // DET: send_perm  ATOMIC: recv_perm
    const int* other;  // DET: receivers  ATOMIC: senders
    int N, C, T, E;
    int band_lo, band_hi;  // only edges whose `other` node is in [band_lo, band_hi)
    int accumulate;        // DET: 0: dx = band sum; 1: dx += band sum
    unsigned* status;
};

// ------------------------------------------------------ async row staging
//
// Each warp owns a ring of S stages in shared memory.  A stage holds one
// edge's rows for the warp's channel tile: the weight row w[e, 0..P) and the
// gathered row (x[s] in the forward and the atomic backward, gy[i] in the
// deterministic backward), each component a run of TILE_C channels.  One
// mbarrier per stage counts the bytes of the bulk copies (cp.async.bulk, no
// multicast) that fill it; the warp waits on the stage's phase before reading
// it, and refills it S edges later.  Every wait is bounded: after
// kWaitLimitNs the kernel sets status bit 4 and stops processing.

// Every wait on a stage gives up after this much time (globaltimer ns); a
// row copy that has not landed by then will not land.  Each poll may suspend
// the thread for at most kWaitSuspendNs (the try_wait time hint), so the
// bound holds whatever the hardware's own suspend limit is.
#ifndef EQC_WAIT_LIMIT_NS
#define EQC_WAIT_LIMIT_NS 200000000ull   // 0.2 s
#endif
constexpr uint64_t kWaitLimitNs = EQC_WAIT_LIMIT_NS;
constexpr uint32_t kWaitSuspendNs = 1000;
// Extra bytes every stage fill expects beyond what its copies carry.  Always 0
// in the library; a test build sets it so that no fill can complete and the
// bounded waits below must give up.
#ifndef EQC_TEST_FILL_DEFICIT
#define EQC_TEST_FILL_DEFICIT 0
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Warp-collective bounded wait on one phase of `bar`: every lane polls and
// the warp leaves the loop together (the phase stays complete once it has
// completed, so all lanes see it within one poll of each other; a timeout
// seen by any lane ends the wait for all).  Returns false, on every lane, if
// the phase did not complete within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_addr(bar);
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity), "r"(kWaitSuspendNs)
            : "memory");
        if (__all_sync(0xffffffffu, done)) return true;
        const uint64_t now = globaltimer_ns();
        if (it == 0) t0 = now;
        if (__any_sync(0xffffffffu, now - t0 > kWaitLimitNs)) return false;
    }
}

// After a wait gave up: wait (bounded again) for the fills still in flight,
// those of edges [from, to) of the warp's staging sequence (edge u sits in
// stage u % S and completes phase (u / S) & 1), so that no copy lands in
// shared memory after the warp has left.  Stages without a fill in flight are
// not waited on.
template <int S>
__device__ __forceinline__ void drain_fills(uint64_t* bars, uint32_t from, uint32_t to) {
    for (uint32_t u = from; u < to; ++u) mbar_wait(&bars[2 * (u % S)], (u / S) & 1u);
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One tensor-map box [rows][TILE_C] at (c0, 0, idx) of a [count][rows][C] tensor.
__device__ __forceinline__ void tma_rows(void* dst, const CUtensorMap* map, int c0, int idx, uint64_t* bar,
                                         uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(0), "r"(idx),
        "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

// Stage geometry: NP weight rows then NG gathered rows, TILE_C floats each.
template <class K, int NG>
struct Stage {
    static constexpr int ROWS = K::NP + NG;
    static constexpr int FLOATS = ROWS * K::TILE_C;   // per stage (a multiple of 64 floats)
    static constexpr uint32_t BYTES = FLOATS * 4;
};

// Fill stage `st` with w[e, :, tile] and g[o, :, tile] (o >= 0): two tensor-map
// copies issued by lane 0.  The caller has __syncwarp()ed after the stage's
// previous readers; the proxy fence orders those reads before the async writes.
template <class K, int NG>
__device__ __forceinline__ void stage_fill(float* st, uint64_t* bar, const CUtensorMap* tw, const CUtensorMap* tg,
                                           int e, int o, int c0, uint64_t pol_w, uint64_t pol_g, int lane) {
    if (lane == 0) {
        fence_proxy_async();
        mbar_expect_tx(bar, Stage<K, NG>::BYTES + EQC_TEST_FILL_DEFICIT);
        tma_rows(st, tw, c0, e, bar, pol_w);
        tma_rows(st + K::NP * K::TILE_C, tg, c0, o, bar, pol_g);
    }
}


// Per-warp shared-memory layout (floats), every region 128-byte aligned:
// [stages: S x FLOATS] [mbarriers: 16 B each] [A: CH x NA_PAD] [gY: CH x GS]
template <class K, int NG, bool WITH_GY, int CH>
struct WarpSmem {
    static constexpr int S = K::STAGES;
    static constexpr int up32(int f) { return (f + 31) & ~31; }
    static constexpr int ST_F = S * Stage<K, NG>::FLOATS;
    static constexpr int BAR_F = up32(4 * S);
    // the backward without coupling matrices keeps only each edge's harmonics
    static constexpr int A_F = up32(CH * ((WITH_GY && EQC_BWD_H) ? K::YS : K::A_ROW));
    static constexpr int GY_F = WITH_GY ? up32(CH * K::GS) : 0;
    static constexpr int TOTAL_F = ST_F + BAR_F + A_F + GY_F;
    static constexpr int BYTES = TOTAL_F * 4;
};

// Warps resident on one SM when CTAs of w warps take `warp_bytes` of shared
// memory per warp (228 KB per SM, 1 KB of it reserved per CTA, at most 227 KB
// per CTA).
constexpr int resident_warps(int w, int warp_bytes) {
    return w * warp_bytes > 227 * 1024 ? 0 : (228 * 1024 / (w * warp_bytes + 1024)) * w;
}

// Warps per CTA (1..4): the largest CTA that keeps within 10% of the most
// warps resident any CTA size allows (larger CTAs mean fewer CTA launches
// and tensor-map prefetches per SM).
constexpr int best_warps(int warp_bytes) {
    int most = 0;
    for (int w = 1; w <= 4; ++w)
        if (resident_warps(w, warp_bytes) > most) most = resident_warps(w, warp_bytes);
    for (int w = 4; w > 1; --w)
        if (10 * resident_warps(w, warp_bytes) >= 9 * most) return w;
    return 1;
}

// Shared-memory layout and CTA shape of the forward and the backward kernels.
template <class K>
struct FwdShape {
    static constexpr int CH = K::chunk(false);
    using L = WarpSmem<K, K::D_IN, false, CH>;
    static constexpr int WARPS = best_warps(L::BYTES);
};
template <class K, bool DET>
struct BwdShape {
    static constexpr int CH = (EQC_BWD_H && EQC_CHUNK_BWD_H > 0) ? EQC_CHUNK_BWD_H : K::chunk(!DET);
    static constexpr int DL = DET ? K::D_OUT : K::D_IN;     // rows gathered per edge
    using L = WarpSmem<K, DL, true, CH>;
    // the atomic kernel keeps the receiver's gy rows in registers and is held
    // by them (up to 255 per thread at l = 3), not by shared memory: it takes
    // 4-warp CTAs, which the register file fits twice
    static constexpr int WARPS = (!DET && resident_warps(4, L::BYTES) > 0) ? 4 : best_warps(L::BYTES);
};

// Collects the next window of up to 32 edges of a node's list whose gathered
// node `other[e]` lies in [lo, hi), scanning 32 list positions at a time from
// position k (advanced past the positions consumed) and keeping list order.
// Out-of-range nodes set status bit 1 and are dropped.  Lanes < n receive
// (e, o, r_e); returns n (0 only when the list is exhausted).
__device__ __forceinline__ int gather_window(const int* perm, const int* other, const float* r, int N, int lo,
                                             int hi, int& k, int ke, unsigned* status, int lane, int& my_e,
                                             int& my_o, float& rx, float& ry, float& rz) {
    int n = 0;
    my_e = 0;
    my_o = 0;
    while (k < ke) {
        const int n_all = min(32, ke - k);
        int e_l = 0, o_l = 0;
        bool in_band = false;
        if (lane < n_all) {
            e_l = perm[k + lane];
            o_l = other[e_l];
            if ((unsigned)o_l >= (unsigned)N)
                atomicOr(status, 1u);
            else
                in_band = o_l >= lo && o_l < hi;
        }
        const unsigned mask = __ballot_sync(0xffffffffu, in_band);
        const int cnt = __popc(mask);
        if (n + cnt > 32) break;                      // the block goes to the next window
        const int slot = lane - n;
        const bool mine = slot >= 0 && slot < cnt;
        const int src = mine ? (int)__fns(mask, 0u, slot + 1) : 0;
        const int e2 = __shfl_sync(0xffffffffu, e_l, src), o2 = __shfl_sync(0xffffffffu, o_l, src);
        if (mine) {
            my_e = e2;
            my_o = o2;
        }
        n += cnt;
        k += n_all;
        if (n == 32) break;
    }
    rx = ry = rz = 0.f;
    if (lane < n) {
        const float* re = r + (size_t)my_e * 3;
        rx = re[0];
        ry = re[1];
        rz = re[2];
    }
    return n;
}

// ---------------------------------------------------------------- forward

template <class K>
__global__ void __launch_bounds__(FwdShape<K>::WARPS * 32)
    eqconv_fwd_kernel(const FwdParams prm, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_x) {
    constexpr int V = K::VEC;
    constexpr int S = K::STAGES;
    constexpr int CH = FwdShape<K>::CH;
    constexpr int WARPS = FwdShape<K>::WARPS;
    using L = typename FwdShape<K>::L;
    constexpr int SF = Stage<K, K::D_IN>::FLOATS;
    extern __shared__ __align__(128) float4 smem4[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * WARPS + warp;
    if (node >= prm.N) return;
    float* stages = reinterpret_cast<float*>(smem4) + warp * L::TOTAL_F;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + L::ST_F);
    float* As = stages + L::ST_F + L::BAR_F;
    const int tile = blockIdx.y;
    const int C = prm.C;
    const int c0 = tile * K::TILE_C;
    const int ct_len = min(K::TILE_C, C - c0);
    const int cl = lane * V;                 // lane's channel offset inside the tile
    const bool active = cl < ct_len;
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bars[2 * s], 1);
        mbar_fence_init();
    }
    __syncwarp();

    float acc[K::D_OUT][V];
#pragma unroll
    for (int d = 0; d < K::D_OUT; ++d)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[d][v] = 0.f;

    uint32_t g = 0;        // edges staged so far by this warp (stage = g % S, phase = (g / S) & 1)
    bool ok_all = true;
    uint32_t fill_from = 0, fill_to = 0;   // after a failed wait: staged edges whose fills are in flight
    int k = prm.ptr[node];
    const int ke = prm.ptr[node + 1];
    while (k < ke && ok_all) {
        int my_e, my_s;
        float rx, ry, rz;
        const int n = gather_window(prm.perm, prm.other, prm.r, prm.N, prm.band_lo, prm.band_hi, k, ke, prm.status,
                                    lane, my_e, my_s, rx, ry, rz);
        if (n == 0) continue;
        // the copy pipeline runs S edges ahead across the whole window
        const int pre = min(S, n);
        for (int t = 0; t < pre; ++t) {
            const int e = __shfl_sync(0xffffffffu, my_e, t), s = __shfl_sync(0xffffffffu, my_s, t);
            const uint32_t gi = g + t;
            stage_fill<K, K::D_IN>(stages + (gi % S) * SF, &bars[2 * (gi % S)], &tmap_w, &tmap_x, e, s, c0,
                                   pol_stream, pol_keep, lane);
        }
        for (int b0 = 0; b0 < n && ok_all; b0 += CH) {
            const int nb = min(CH, n - b0);
            if (lane >= b0 && lane < b0 + nb) {
                float ux, uy, uz, il;
                const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                float Y[K::D_SH];
                sh_eval<K::LSH>(ok, ux, uy, uz, Y);
                compute_A<K>(Y, As + (lane - b0) * K::NA_PAD);
            }
            __syncwarp();
            for (int t = b0; t < b0 + nb; ++t) {
                const uint32_t gi = g + t;
                float* st = stages + (gi % S) * SF;
                if (!mbar_wait(&bars[2 * (gi % S)], (gi / S) & 1u)) {
                    if (lane == 0) atomicOr(prm.status, 4u);
                    ok_all = false;
                    fill_from = gi;                       // fills of edges [gi, g + min(n, t + S)) are in flight
                    fill_to = g + (uint32_t)min(n, t + S);
                    break;
                }
                // Lanes past C in a ragged tile read the tensor map's zero fill, so
                // the reads need no predicate for correctness; at wide tiles the
                // predicate keeps ptxas from hoisting every row load (registers).
                constexpr bool kPred = EQC_FWD_PRED == 2 || (EQC_FWD_PRED == 1 && V >= 4);
                const bool rd = !kPred || active;
                float xv[K::D_IN][V], wv[K::NP][V];
#pragma unroll
                for (int p = 0; p < K::NP; ++p) {
                    if (rd)
                        lds_vec<V>(wv[p], st + p * K::TILE_C + cl);
                    else
#pragma unroll
                        for (int v = 0; v < V; ++v) wv[p][v] = 0.f;
                }
#pragma unroll
                for (int d = 0; d < K::D_IN; ++d) {
                    if (rd)
                        lds_vec<V>(xv[d], st + (K::NP + d) * K::TILE_C + cl);
                    else
#pragma unroll
                        for (int v = 0; v < V; ++v) xv[d][v] = 0.f;
                }
                fwd_edge<K>(As + (t - b0) * K::NA_PAD, xv, wv, acc);
                __syncwarp();
                if (t + S < n) {
                    const int e = __shfl_sync(0xffffffffu, my_e, t + S), s = __shfl_sync(0xffffffffu, my_s, t + S);
                    stage_fill<K, K::D_IN>(st, &bars[2 * (gi % S)], &tmap_w, &tmap_x, e, s, c0, pol_stream,
                                           pol_keep, lane);
                }
            }
            __syncwarp();
        }
        g += n;
    }
    if (!ok_all) {
        drain_fills<S>(bars, fill_from, fill_to);
        return;
    }
    // a later band adds its sum; a band without edges for this node leaves y as it is
    if (active && (!prm.accumulate || g > 0)) {
        float* yi = prm.y + (size_t)node * K::D_OUT * C + c0 + cl;
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) {
            if (prm.accumulate) {
                float old[V];
                ld_keep<V>(old, yi + (size_t)d * C, pol_stream);
#pragma unroll
                for (int v = 0; v < V; ++v) acc[d][v] += old[v];
            }
            st_stream<V>(yi + (size_t)d * C, acc[d]);
        }
    }
}

// --------------------------------------------------------------- backward

// Sums NV values (a power of two <= 32) over the warp's 32 lanes at once:
// each halving step trades half of the values with the partner lane, so the
// cost is NV - 1 + 5 - log2(NV) shuffles instead of 5 NV.  Lane L returns the
// sum of value L >> (5 - log2 NV).  The order of the additions is fixed
// (bitwise reproducible).
template <int NV>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[NV], int lane) {
    static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "NV: a power of two <= 32");
    constexpr int LOG = NV >= 32 ? 5 : NV >= 16 ? 4 : NV >= 8 ? 3 : NV >= 4 ? 2 : NV >= 2 ? 1 : 0;
#pragma unroll
    for (int st = 0; st < LOG; ++st) {
        const int n = NV >> (st + 1), o = 16 >> st;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float send = upper ? v[i] : v[i + n];
            const float keep = upper ? v[i + n] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float r = v[0];
#pragma unroll
    for (int st = LOG; st < 5; ++st) r += __shfl_xor_sync(0xffffffffu, r, 16 >> st);
    return r;
}

// Butterfly sum across the warp (fixed order: bitwise reproducible).
template <int G>
__device__ __forceinline__ void warp_sum(float (&v)[G]) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < G; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
}

// The smallest power of two >= n (n <= 32), for warp_transpose_sum.
constexpr int pow2_at_least(int n) { return n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : n <= 8 ? 8 : n <= 16 ? 16 : 32; }
// log2 of the lanes that share one result of warp_transpose_sum<NV>.
constexpr int transpose_sum_shift(int nv) { return nv >= 32 ? 0 : nv >= 16 ? 1 : nv >= 8 ? 2 : nv >= 4 ? 3 : nv >= 2 ? 4 : 5; }

// DET: node = sender j, resident x_j, dx_j summed in registers in send_perm order.
// !DET: node = receiver i, resident gy_i, dx scattered with atomic adds.
// FUSED: the tile covers every channel (T == 1): dr is finished in-kernel.
template <class K, bool DET, bool FUSED>
__device__ __forceinline__ void eqconv_bwd_body(const BwdParams& prm, const CUtensorMap* tmap_w,
                                                const CUtensorMap* tmap_g) {
    constexpr int V = K::VEC;
    constexpr int S = K::STAGES;
    constexpr int GG = K::G > 0 ? K::G : 1;
    constexpr int DL = BwdShape<K, DET>::DL;         // rows gathered per edge
    constexpr int CH = BwdShape<K, DET>::CH;
    constexpr int WARPS = BwdShape<K, DET>::WARPS;
    using L = typename BwdShape<K, DET>::L;
    constexpr int SF = Stage<K, DL>::FLOATS;
    extern __shared__ __align__(128) float4 smem4[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * WARPS + warp;
    if (node >= prm.N) return;
    float* stages = reinterpret_cast<float*>(smem4) + warp * L::TOTAL_F;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + L::ST_F);
    float* As = stages + L::ST_F + L::BAR_F;
    float* gYs = As + L::A_F;
    const int tile = blockIdx.y;
    const int C = prm.C;
    const int c0 = tile * K::TILE_C;
    const int ct_len = min(K::TILE_C, C - c0);
    const int cl = lane * V;
    const bool active = cl < ct_len;
    const size_t c_off = (size_t)c0 + cl;
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&bars[2 * s], 1);
        mbar_fence_init();
    }
    __syncwarp();

    // resident rows: x_j (DET) or gy_i (!DET)
    float xres[DET ? K::D_IN : 1][V];
    float gres[DET ? 1 : K::D_OUT][V];
    float dxacc[DET ? K::D_IN : 1][V];
    if constexpr (DET) {
        const float* xj = prm.x + (size_t)node * K::D_IN * C + c_off;
#pragma unroll
        for (int d = 0; d < K::D_IN; ++d) {
            if (active)
                ld_keep<V>(xres[d], xj + (size_t)d * C, pol_keep);
            else
#pragma unroll
                for (int v = 0; v < V; ++v) xres[d][v] = 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) dxacc[d][v] = 0.f;
        }
    } else {
        const float* gi = prm.gy + (size_t)node * K::D_OUT * C + c_off;
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) {
            if (active)
                ld_keep<V>(gres[d], gi + (size_t)d * C, pol_keep);
            else
#pragma unroll
                for (int v = 0; v < V; ++v) gres[d][v] = 0.f;
        }
    }

    uint32_t g = 0;
    bool ok_all = true;
    uint32_t fill_from = 0, fill_to = 0;   // after a failed wait: staged edges whose fills are in flight
    int k = prm.ptr[node];
    const int ke = prm.ptr[node + 1];
    while (k < ke && ok_all) {
        int my_e, my_o;
        float rx, ry, rz;
        const int n = gather_window(prm.perm, prm.other, prm.r, prm.N, prm.band_lo, prm.band_hi, k, ke, prm.status,
                                    lane, my_e, my_o, rx, ry, rz);
        if (n == 0) continue;
        // the copy pipeline runs S edges ahead across the whole window
        const int pre = min(S, n);
        for (int t = 0; t < pre; ++t) {
            const int e = __shfl_sync(0xffffffffu, my_e, t), o = __shfl_sync(0xffffffffu, my_o, t);
            const uint32_t gi = g + t;
            stage_fill<K, DL>(stages + (gi % S) * SF, &bars[2 * (gi % S)], tmap_w, tmap_g, e, o, c0, pol_stream,
                              pol_keep, lane);
        }
        for (int b0 = 0; b0 < n && ok_all; b0 += CH) {
            const int nb = min(CH, n - b0);
            if (lane >= b0 && lane < b0 + nb) {
                float ux, uy, uz, il;
                const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                float Y[K::D_SH];
                sh_eval<K::LSH>(ok, ux, uy, uz, Y);
                if constexpr (EQC_BWD_H) {
                    float* yrow = As + (lane - b0) * K::YS;
#pragma unroll
                    for (int q = 0; q < K::D_SH; ++q) yrow[q] = Y[q];
                } else {
                    compute_A<K>(Y, As + (lane - b0) * K::NA_PAD);
                }
            }
            __syncwarp();
            for (int t = b0; t < b0 + nb; ++t) {
                const uint32_t gi = g + t;
                float* st = stages + (gi % S) * SF;
                if (!mbar_wait(&bars[2 * (gi % S)], (gi / S) & 1u)) {
                    if (lane == 0) atomicOr(prm.status, 4u);
                    ok_all = false;
                    fill_from = gi;                       // fills of edges [gi, g + min(n, t + S)) are in flight
                    fill_to = g + (uint32_t)min(n, t + S);
                    break;
                }
                const int e = __shfl_sync(0xffffffffu, my_e, t), o = __shfl_sync(0xffffffffu, my_o, t);
                // inactive lanes (past C in a ragged tile) read zeros; the predicate
                // also keeps the compiler from hoisting every row load
                const SmemRows<V> Wr{st + cl, K::TILE_C, active};
                const SmemRows<V> Lr{st + K::NP * K::TILE_C + cl, K::TILE_C, active};
                float gyl[GG];
#pragma unroll
                for (int q = 0; q < GG; ++q) gyl[q] = 0.f;
                float* dwe = prm.dw + (size_t)e * K::NP * C + c_off;
                auto store_dw = [&](int p, const float* dwv) {
                    if (active) st_stream<V>(dwe + (size_t)p * C, dwv);
                };
                if constexpr (DET) {
                    auto no_sink = [](int, int, const float (&)[1][V]) {};
                    bwd_edge<K, true>(As + (t - b0) * (EQC_BWD_H ? K::YS : K::NA_PAD), RegRows<V, K::D_IN>{xres}, Lr,
                                      Wr, dxacc, no_sink,
                                      gyl, store_dw);
                } else {
                    float* dxs = prm.dx + (size_t)o * K::D_IN * C + c_off;
                    auto sink = [&](int o1, int d1, const float (&blk)[2 * kMaxL + 1][V]) {
                        if (active)
#pragma unroll
                            for (int m = 0; m < d1; ++m) red_add<V>(dxs + (size_t)(o1 + m) * C, blk[m]);
                    };
                    bwd_edge<K, false>(As + (t - b0) * (EQC_BWD_H ? K::YS : K::NA_PAD), Lr,
                                       RegRows<V, K::D_OUT>{gres}, Wr, dxacc, sink,
                                       gyl, store_dw);
                }
                if constexpr (K::G > 0 && V == 1) {
                    // value q of the warp's sum lands on lanes q << SH .. (q + 1) << SH
                    constexpr int NV = pow2_at_least(K::G), SH = transpose_sum_shift(NV);
                    float tv[NV];
#pragma unroll
                    for (int q = 0; q < NV; ++q) tv[q] = q < K::G ? gyl[q] : 0.f;
                    const float sum = warp_transpose_sum<NV>(tv, lane);
                    const int q = lane >> SH;
                    if ((lane & ((1 << SH) - 1)) == 0 && q < K::G) {
                        if constexpr (FUSED)
                            gYs[(t - b0) * K::GS + q] = sum;
                        else
                            prm.gy_part[((size_t)e * prm.T + tile) * K::G + q] = sum;
                    }
                } else if constexpr (K::G > 0) {
                    // wider channel tiles are held by registers: the plain butterfly needs fewer
                    warp_sum<K::G>(gyl);
                    if (lane == 0) {
                        if constexpr (FUSED) {
#pragma unroll
                            for (int q = 0; q < K::G; ++q) gYs[(t - b0) * K::GS + q] = gyl[q];
                        } else {
                            float* gp = prm.gy_part + ((size_t)e * prm.T + tile) * K::G;
#pragma unroll
                            for (int q = 0; q < K::G; ++q) gp[q] = gyl[q];
                        }
                    }
                }
                __syncwarp();
                if (t + S < n) {
                    const int e2 = __shfl_sync(0xffffffffu, my_e, t + S), o2 = __shfl_sync(0xffffffffu, my_o, t + S);
                    stage_fill<K, DL>(st, &bars[2 * (gi % S)], tmap_w, tmap_g, e2, o2, c0, pol_stream, pol_keep,
                                      lane);
                }
            }
            __syncwarp();
            if constexpr (FUSED) {
                if (ok_all && lane >= b0 && lane < b0 + nb) {
                    float ux, uy, uz, il;
                    const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                    float d0 = 0.f, d1 = 0.f, d2 = 0.f;
                    if constexpr (K::G > 0)
                        sh_grad_contract<K::LSH>(ok, ux, uy, uz, il, gYs + (lane - b0) * K::GS, d0, d1, d2);
                    float* dre = prm.dr + (size_t)my_e * 3;
                    dre[0] = d0;
                    dre[1] = d1;
                    dre[2] = d2;
                }
                __syncwarp();
            }
        }
        g += n;
    }
    if (!ok_all) {
        drain_fills<S>(bars, fill_from, fill_to);
        return;
    }
    if constexpr (DET) {
        // a later band adds its sum; a band without edges for this node leaves dx as it is
        if (active && (!prm.accumulate || g > 0)) {
            float* dxj = prm.dx + (size_t)node * K::D_IN * C + c_off;
#pragma unroll
            for (int d = 0; d < K::D_IN; ++d) {
                if (prm.accumulate) {
                    float old[V];
                    ld_keep<V>(old, dxj + (size_t)d * C, pol_stream);
#pragma unroll
                    for (int v = 0; v < V; ++v) dxacc[d][v] += old[v];
                }
                st_stream<V>(dxj + (size_t)d * C, dxacc[d]);
            }
        }
    }
}

template <class K, bool DET, bool FUSED>
__global__ void __launch_bounds__(BwdShape<K, DET>::WARPS * 32)
    eqconv_bwd_kernel(const BwdParams prm, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_g) {
    eqconv_bwd_body<K, DET, FUSED>(prm, &tmap_w, &tmap_g);
}

// The deterministic kernel that leaves dr to the epilogue (several channel
// tiles) at 128-channel tiles, capped at 168 registers (shared memory then
// allows 3 CTAs of 3 warps per SM): left to its own heuristic it takes 232
// and holds 2 CTAs, with no spill either way.
template <class K>
__global__ void __launch_bounds__(BwdShape<K, true>::WARPS * 32, 4)
    eqconv_bwd_tiles_kernel(const BwdParams prm, const __grid_constant__ CUtensorMap tmap_w,
                            const __grid_constant__ CUtensorMap tmap_g) {
    eqconv_bwd_body<K, true, false>(prm, &tmap_w, &tmap_g);
}

// dr for edges whose gY is split over T channel tiles: fixed-order sum, then
// the harmonic-gradient contraction.  One thread per edge.
template <int LSH>
__global__ void eqconv_dr_epilogue(const float* gy_part, int T, const float* r, float* dr, int E) {
    constexpr int G = (LSH + 1) * (LSH + 1) - 1;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    float g[G > 0 ? G : 1];
#pragma unroll
    for (int k = 0; k < (G > 0 ? G : 1); ++k) g[k] = 0.f;
    for (int t = 0; t < T; ++t) {
        const float* gp = gy_part + ((size_t)e * T + t) * G;
#pragma unroll
        for (int k = 0; k < G; ++k) g[k] += gp[k];
    }
    const float* re = r + (size_t)e * 3;
    float ux, uy, uz, il;
    const bool ok = unit_dir(re[0], re[1], re[2], ux, uy, uz, il);
    float d0 = 0.f, d1 = 0.f, d2 = 0.f;
    if constexpr (G > 0) sh_grad_contract<LSH>(ok, ux, uy, uz, il, g, d0, d1, d2);
    dr[(size_t)e * 3] = d0;
    dr[(size_t)e * 3 + 1] = d1;
    dr[(size_t)e * 3 + 2] = d2;
}

template <int LSH>
__global__ void eqconv_sh_kernel(const float* r, float* Y, int E) {
    constexpr int D = (LSH + 1) * (LSH + 1);
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const float* re = r + (size_t)e * 3;
    float ux, uy, uz, il;
    const bool ok = unit_dir(re[0], re[1], re[2], ux, uy, uz, il);
    float y[D];
    sh_eval<LSH>(ok, ux, uy, uz, y);
#pragma unroll
    for (int k = 0; k < D; ++k) Y[(size_t)e * D + k] = y[k];
}

}  // namespace eqc

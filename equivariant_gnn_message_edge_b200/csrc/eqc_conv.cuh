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
//   * edges are processed in chunks of CHUNK: lane t of the warp reads edge t
//     of the chunk, evaluates Y(r_e) and the per-edge coupling matrices
//       A_p[m3][m1] = sum_m2 C_p[m1,m2,m3] Y_{l2 m2}(r_e)        (l2 > 0)
//     with the CG as compile-time immediates (zeros skipped), and stores
//     them in shared memory; paths with l2 = 0 have A = identity;
//   * then the warp walks the chunk's edges; every lane reads A (broadcast)
//     and applies it to its channels, with the next edge's w / x rows loaded
//     into registers while the current edge is computed;
//   * forward:  acc[l3 m3] += w_p * sum_m1 A_p[m3][m1] x[s, l1 m1]
//   * backward: t = A_p^T gy_i,  dw_p = x_s . t,  dx_s += w_p t,
//               gY[l2 m2] += w_p sum_{m1,m3} C_p[m1,m2,m3] x_s[m1] gy_i[m3]
//     (gY summed over the lane's channels, then across the warp by a fixed
//     butterfly; dr = (dY/dr)^T gY).
// Streams (w read, dw written) carry L2 evict-first hints; gathered rows
// (x or gy, reused ~45 times) carry evict-last hints.
#pragma once

#include <cstdint>
#include <type_traits>
#include <utility>

#include "eqc_sh.cuh"
#include "eqc_tables.h"

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

template <int LIN_, int LSH_, int LOUT_, int VEC_>
struct Cfg {
    static constexpr int LIN = LIN_, LSH = LSH_, LOUT = LOUT_, VEC = VEC_;
    static constexpr PathList PL = make_paths(LIN, LSH, LOUT);
    static constexpr int NP = PL.n;
    static constexpr int D_IN = (LIN + 1) * (LIN + 1);
    static constexpr int D_SH = (LSH + 1) * (LSH + 1);
    static constexpr int D_OUT = (LOUT + 1) * (LOUT + 1);
    static constexpr int G = D_SH - 1;              // dr needs gY for l2 > 0 only
    static constexpr AOffsets AO = make_aoffsets(PL);
    static constexpr int NA = AO.total;
    static constexpr int NA_PAD = pad_odd4(NA);     // row stride; NA_PAD/4 odd: conflict-free STS.128
    static constexpr int CHUNK = NA_PAD <= 128 ? 32 : (NA_PAD <= 256 ? 16 : 8);
    static constexpr int GS = G | 1;                // gY row stride in shared memory (odd)
    static constexpr int WARPS = 4;
    static constexpr int TILE_C = 32 * VEC;
    // register estimate of the double-buffered edge rows
    static constexpr int FWD_ROWS = (D_IN + NP) * VEC;
    static constexpr bool FWD_PREFETCH = 2 * FWD_ROWS + D_OUT * VEC <= 160;
    static constexpr bool BWD_PREFETCH = 2 * (D_OUT + NP) * VEC + 2 * D_IN * VEC <= 160;
    static constexpr int FWD_SMEM = WARPS * CHUNK * NA_PAD * 4;
    static constexpr int BWD_SMEM = WARPS * CHUNK * (NA_PAD + GS) * 4;
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
    if constexpr (VEC == 4) {
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
    if constexpr (VEC == 4) {
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
    if constexpr (VEC == 4)
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}
template <int VEC>
__device__ __forceinline__ void st_stream(float* p, const float* v) {
    if constexpr (VEC == 4)
        __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    else
        __stcs(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
}
template <int VEC>
__device__ __forceinline__ void red_add(float* p, const float* v) {
    if constexpr (VEC == 4)
        atomicAdd(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    else
        atomicAdd(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
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
        constexpr int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o3 = l3 * l3;
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

// Given x (sender rows), g (receiver output-gradient rows) and w for one edge:
// dw[p] (stored through `dwp`), dx += w_p A_p^T g, gyl += per-lane partial of gY.
template <class K, class StoreDw>
__device__ __forceinline__ void bwd_edge(const float* As, const float (&xv)[K::D_IN][K::VEC],
                                         const float (&gv)[K::D_OUT][K::VEC], const float (&wv)[K::NP][K::VEC],
                                         float (&dxv)[K::D_IN][K::VEC], float (&gyl)[K::G > 0 ? K::G : 1],
                                         StoreDw&& store_dw) {
    constexpr int V = K::VEC;
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o3 = l3 * l3;
        float t[d1][V];
        if constexpr (l2 == 0) {
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) t[m][v] = gv[o3 + m][v];
        } else {
            constexpr int n4 = (d1 * d3 + 3) / 4;
            constexpr int aoff = K::AO.off[p];
            float a[n4 * 4];
            load_A<n4>(As + aoff, a);
#pragma unroll
            for (int m1 = 0; m1 < d1; ++m1) {
#pragma unroll
                for (int v = 0; v < V; ++v) t[m1][v] = a[m1] * gv[o3][v];
#pragma unroll
                for (int m3 = 1; m3 < d3; ++m3)
#pragma unroll
                    for (int v = 0; v < V; ++v) t[m1][v] = fmaf(a[m3 * d1 + m1], gv[o3 + m3][v], t[m1][v]);
            }
        }
        float dw[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float s = xv[o1][v] * t[0][v];
#pragma unroll
            for (int m1 = 1; m1 < d1; ++m1) s = fmaf(xv[o1 + m1][v], t[m1][v], s);
            dw[v] = s;
        }
        store_dw(p, dw);
#pragma unroll
        for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
            for (int v = 0; v < V; ++v) dxv[o1 + m1][v] = fmaf(wv[p][v], t[m1][v], dxv[o1 + m1][v]);
        if constexpr (l2 > 0) {
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
                                if constexpr (c != 0.0) s = fmaf((float)c, gv[o3 + m3][v], s);
                            });
                            g = fmaf(xv[o1 + m1][v], s, g);
                        }
                    });
                    gsum = fmaf(wv[p][v], g, gsum);
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
    int N, C;
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
    int N, C, T;
    unsigned* status;
};

// ---------------------------------------------------------------- forward

template <class K>
__global__ void __launch_bounds__(K::WARPS * 32) eqconv_fwd_kernel(const FwdParams prm) {
    constexpr int V = K::VEC;
    extern __shared__ float4 smem4[];
    float* smem = reinterpret_cast<float*>(smem4);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * K::WARPS + warp;
    if (node >= prm.N) return;
    float* As = smem + warp * (K::CHUNK * K::NA_PAD);
    const int c0 = blockIdx.y * K::TILE_C + lane * V;
    const bool active = c0 < prm.C;
    const size_t C = (size_t)prm.C;
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();

    float acc[K::D_OUT][V];
#pragma unroll
    for (int d = 0; d < K::D_OUT; ++d)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[d][v] = 0.f;

    auto load_edge = [&](int e, int s, float (&xv)[K::D_IN][V], float (&wv)[K::NP][V]) {
        if (active && s >= 0) {
            const float* xs = prm.x + (size_t)s * K::D_IN * C + c0;
#pragma unroll
            for (int d = 0; d < K::D_IN; ++d) ld_keep<V>(xv[d], xs + d * C, pol_keep);
        } else {
#pragma unroll
            for (int d = 0; d < K::D_IN; ++d)
#pragma unroll
                for (int v = 0; v < V; ++v) xv[d][v] = 0.f;
        }
        if (active) {
            const float* we = prm.w + (size_t)e * K::NP * C + c0;
#pragma unroll
            for (int p = 0; p < K::NP; ++p) ld_stream<V>(wv[p], we + p * C, pol_stream);
        } else {
#pragma unroll
            for (int p = 0; p < K::NP; ++p)
#pragma unroll
                for (int v = 0; v < V; ++v) wv[p][v] = 0.f;
        }
    };

    const int kb = prm.ptr[node], ke = prm.ptr[node + 1];
    for (int k0 = kb; k0 < ke; k0 += K::CHUNK) {
        const int n = min(K::CHUNK, ke - k0);
        int my_e = 0, my_s = -1;
        if (lane < n) {
            my_e = prm.perm[k0 + lane];
            const int s = prm.other[my_e];
            if ((unsigned)s < (unsigned)prm.N)
                my_s = s;
            else
                atomicOr(prm.status, 1u);
            const float* re = prm.r + (size_t)my_e * 3;
            float ux, uy, uz, il;
            const bool ok = unit_dir(re[0], re[1], re[2], ux, uy, uz, il);
            float Y[K::D_SH];
            sh_eval<K::LSH>(ok, ux, uy, uz, Y);
            compute_A<K>(Y, As + lane * K::NA_PAD);
        }
        __syncwarp();
        if constexpr (K::FWD_PREFETCH) {
            float xc[K::D_IN][V], wc[K::NP][V], xn[K::D_IN][V], wn[K::NP][V];
            load_edge(__shfl_sync(0xffffffffu, my_e, 0), __shfl_sync(0xffffffffu, my_s, 0), xc, wc);
            for (int t = 0; t < n; ++t) {
                if (t + 1 < n)
                    load_edge(__shfl_sync(0xffffffffu, my_e, t + 1), __shfl_sync(0xffffffffu, my_s, t + 1), xn, wn);
                fwd_edge<K>(As + t * K::NA_PAD, xc, wc, acc);
#pragma unroll
                for (int d = 0; d < K::D_IN; ++d)
#pragma unroll
                    for (int v = 0; v < V; ++v) xc[d][v] = xn[d][v];
#pragma unroll
                for (int p = 0; p < K::NP; ++p)
#pragma unroll
                    for (int v = 0; v < V; ++v) wc[p][v] = wn[p][v];
            }
        } else {
            for (int t = 0; t < n; ++t) {
                float xc[K::D_IN][V], wc[K::NP][V];
                load_edge(__shfl_sync(0xffffffffu, my_e, t), __shfl_sync(0xffffffffu, my_s, t), xc, wc);
                fwd_edge<K>(As + t * K::NA_PAD, xc, wc, acc);
            }
        }
        __syncwarp();
    }
    if (active) {
        float* yi = prm.y + (size_t)node * K::D_OUT * C + c0;
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) st_plain<V>(yi + d * C, acc[d]);
    }
}

// --------------------------------------------------------------- backward

// Butterfly sum across the warp (fixed order: bitwise reproducible).
template <int G>
__device__ __forceinline__ void warp_sum(float (&v)[G]) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < G; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
}

// DET: node = sender j, resident x_j, dx_j summed in registers in send_perm order.
// !DET: node = receiver i, resident gy_i, dx scattered with atomic adds.
// FUSED: the tile covers every channel (T == 1): dr is finished in-kernel.
template <class K, bool DET, bool FUSED>
__global__ void __launch_bounds__(K::WARPS * 32) eqconv_bwd_kernel(const BwdParams prm) {
    constexpr int V = K::VEC;
    constexpr int GG = K::G > 0 ? K::G : 1;
    extern __shared__ float4 smem4[];
    float* smem = reinterpret_cast<float*>(smem4);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * K::WARPS + warp;
    if (node >= prm.N) return;
    float* As = smem + warp * (K::CHUNK * (K::NA_PAD + K::GS));
    float* gYs = As + K::CHUNK * K::NA_PAD;
    const int tile = blockIdx.y;
    const int c0 = tile * K::TILE_C + lane * V;
    const bool active = c0 < prm.C;
    const size_t C = (size_t)prm.C;
    const uint64_t pol_stream = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();

    // resident rows: x_j (DET) or gy_i (!DET)
    float xres[DET ? K::D_IN : 1][V];
    float gres[DET ? 1 : K::D_OUT][V];
    float dxacc[DET ? K::D_IN : 1][V];
    if constexpr (DET) {
        const float* xj = prm.x + (size_t)node * K::D_IN * C + c0;
#pragma unroll
        for (int d = 0; d < K::D_IN; ++d) {
            if (active)
                ld_keep<V>(xres[d], xj + d * C, pol_keep);
            else
#pragma unroll
                for (int v = 0; v < V; ++v) xres[d][v] = 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) dxacc[d][v] = 0.f;
        }
    } else {
        const float* gi = prm.gy + (size_t)node * K::D_OUT * C + c0;
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) {
            if (active)
                ld_keep<V>(gres[d], gi + d * C, pol_keep);
            else
#pragma unroll
                for (int v = 0; v < V; ++v) gres[d][v] = 0.f;
        }
    }

    // rows loaded per edge: gy_i and w_e (DET) or x_s and w_e (!DET)
    constexpr int DL = DET ? K::D_OUT : K::D_IN;
    auto load_edge = [&](int e, int o, float (&lv)[DL][V], float (&wv)[K::NP][V]) {
        if (active && o >= 0) {
            const float* src = DET ? prm.gy + (size_t)o * K::D_OUT * C + c0 : prm.x + (size_t)o * K::D_IN * C + c0;
#pragma unroll
            for (int d = 0; d < DL; ++d) ld_keep<V>(lv[d], src + d * C, pol_keep);
        } else {
#pragma unroll
            for (int d = 0; d < DL; ++d)
#pragma unroll
                for (int v = 0; v < V; ++v) lv[d][v] = 0.f;
        }
        if (active) {
            const float* we = prm.w + (size_t)e * K::NP * C + c0;
#pragma unroll
            for (int p = 0; p < K::NP; ++p) ld_stream<V>(wv[p], we + p * C, pol_stream);
        } else {
#pragma unroll
            for (int p = 0; p < K::NP; ++p)
#pragma unroll
                for (int v = 0; v < V; ++v) wv[p][v] = 0.f;
        }
    };

    auto do_edge = [&](int t, int e, int o, const float (&lv)[DL][V], const float (&wv)[K::NP][V]) {
        float gyl[GG];
#pragma unroll
        for (int k = 0; k < GG; ++k) gyl[k] = 0.f;
        float* dwe = prm.dw + (size_t)e * K::NP * C + c0;
        auto store_dw = [&](int p, const float* dwv) {
            if (active) st_stream<V>(dwe + p * C, dwv);
        };
        if constexpr (DET) {
            bwd_edge<K>(As + t * K::NA_PAD, xres, lv, wv, dxacc, gyl, store_dw);
        } else {
            float dxe[K::D_IN][V];
#pragma unroll
            for (int d = 0; d < K::D_IN; ++d)
#pragma unroll
                for (int v = 0; v < V; ++v) dxe[d][v] = 0.f;
            bwd_edge<K>(As + t * K::NA_PAD, lv, gres, wv, dxe, gyl, store_dw);
            if (active && o >= 0) {
                float* dxs = prm.dx + (size_t)o * K::D_IN * C + c0;
#pragma unroll
                for (int d = 0; d < K::D_IN; ++d) red_add<V>(dxs + d * C, dxe[d]);
            }
        }
        if constexpr (K::G > 0) {
            warp_sum<K::G>(gyl);
            if (lane == 0) {
                if constexpr (FUSED) {
#pragma unroll
                    for (int k = 0; k < K::G; ++k) gYs[t * K::GS + k] = gyl[k];
                } else {
                    float* gp = prm.gy_part + ((size_t)e * prm.T + tile) * K::G;
#pragma unroll
                    for (int k = 0; k < K::G; ++k) gp[k] = gyl[k];
                }
            }
        }
    };

    const int kb = prm.ptr[node], ke = prm.ptr[node + 1];
    for (int k0 = kb; k0 < ke; k0 += K::CHUNK) {
        const int n = min(K::CHUNK, ke - k0);
        int my_e = 0, my_o = -1;
        float rx = 0.f, ry = 0.f, rz = 0.f;
        if (lane < n) {
            my_e = prm.perm[k0 + lane];
            const int o = prm.other[my_e];
            if ((unsigned)o < (unsigned)prm.N)
                my_o = o;
            else
                atomicOr(prm.status, 1u);
            const float* re = prm.r + (size_t)my_e * 3;
            rx = re[0];
            ry = re[1];
            rz = re[2];
            float ux, uy, uz, il;
            const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
            float Y[K::D_SH];
            sh_eval<K::LSH>(ok, ux, uy, uz, Y);
            compute_A<K>(Y, As + lane * K::NA_PAD);
        }
        __syncwarp();
        if constexpr (K::BWD_PREFETCH) {
            float lc[DL][V], wc[K::NP][V], ln[DL][V], wn[K::NP][V];
            int e_c = __shfl_sync(0xffffffffu, my_e, 0), o_c = __shfl_sync(0xffffffffu, my_o, 0);
            load_edge(e_c, o_c, lc, wc);
            for (int t = 0; t < n; ++t) {
                int e_n = 0, o_n = -1;
                if (t + 1 < n) {
                    e_n = __shfl_sync(0xffffffffu, my_e, t + 1);
                    o_n = __shfl_sync(0xffffffffu, my_o, t + 1);
                    load_edge(e_n, o_n, ln, wn);
                }
                do_edge(t, e_c, o_c, lc, wc);
#pragma unroll
                for (int d = 0; d < DL; ++d)
#pragma unroll
                    for (int v = 0; v < V; ++v) lc[d][v] = ln[d][v];
#pragma unroll
                for (int p = 0; p < K::NP; ++p)
#pragma unroll
                    for (int v = 0; v < V; ++v) wc[p][v] = wn[p][v];
                e_c = e_n;
                o_c = o_n;
            }
        } else {
            for (int t = 0; t < n; ++t) {
                float lc[DL][V], wc[K::NP][V];
                const int e = __shfl_sync(0xffffffffu, my_e, t), o = __shfl_sync(0xffffffffu, my_o, t);
                load_edge(e, o, lc, wc);
                do_edge(t, e, o, lc, wc);
            }
        }
        __syncwarp();
        if constexpr (FUSED) {
            if (lane < n) {
                float ux, uy, uz, il;
                const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                float d0 = 0.f, d1 = 0.f, d2 = 0.f;
                if constexpr (K::G > 0) sh_grad_contract<K::LSH>(ok, ux, uy, uz, il, gYs + lane * K::GS, d0, d1, d2);
                float* dre = prm.dr + (size_t)my_e * 3;
                dre[0] = d0;
                dre[1] = d1;
                dre[2] = d2;
            }
            __syncwarp();
        }
    }
    if constexpr (DET) {
        if (active) {
            float* dxj = prm.dx + (size_t)node * K::D_IN * C + c0;
#pragma unroll
            for (int d = 0; d < K::D_IN; ++d) st_plain<V>(dxj + d * C, dxacc[d]);
        }
    }
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

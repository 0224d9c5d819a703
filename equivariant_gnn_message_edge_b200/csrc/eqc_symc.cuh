// Symmetric contraction of correlation order 2 (the MACE product basis),
// forward and backward (device code).
//
// e3j (arXiv 2609.35099), abstract and Table 3: MACE(a)'s product basis of
// correlation order 2, the tensor-product operation the page measures at over
// 80% of the GPU's memory bandwidth; FlashCart (arXiv 2610.06409) §5 /
// App. B: the correlation ladder, channel-diagonal products of an atom's own
// features along the admissible paths, weighted per path, channel and
// element.  For A [N][(LA+1)^2][C] and species z [N]:
//   B[i, L M, c] = W1[z_i, L, c] A[i, L M, c]
//                + sum_q W2[z_i, q, c] sum_{m1,m2} C_q[m1,m2,M] A[i,l1 m1,c] A[i,l2 m2,c]
// q over the paths of make_sym_paths (l1 <= l2).  Backward given gB:
//   dA = W1 gB + sum_q W2 (C_q A_l2 gB  on block l1  +  C_q A_l1 gB  on block l2)
//   dW1[s, L, c] = sum_{i: z_i = s} A_L . gB_L,   dW2[s, q, c] = sum_{i: z_i = s} C_q A A gB
//
// One warp = one node x one channel tile at a time, nodes walked with a fixed
// grid stride.  The species' weight rows are tiny and stay in L1/L2, so A and
// B (gB, dA) are streamed once: an HBM-bound op.  The backward keeps each
// warp's weight-gradient partials per species in shared memory (each lane
// owns its channel, nodes are added in the warp's order) and a second launch
// sums the warps' partials in order: deterministic.
#pragma once

#include "eqc_conv.cuh"

namespace eqc {

template <int LA_, int LOUT_, int VEC_>
struct SymCfg {
    static constexpr int LA = LA_, LOUT = LOUT_, VEC = VEC_;
    static constexpr PathList PL = make_sym_paths(LA, LOUT);
    static constexpr int NP = PL.n;
    static constexpr int D_A = (LA + 1) * (LA + 1);
    static constexpr int D_OUT = (LOUT + 1) * (LOUT + 1);
    static constexpr int L1N = (LA < LOUT ? LA : LOUT) + 1;   // order-1 weights per species
    static constexpr int NW = L1N + NP;                        // weight rows per species
    static constexpr int TILE_C = 32 * VEC;
};

struct SymParams {
    const float* A;        // [N][D_A][C]
    const int* species;    // [N]
    const float* W1;       // [S][L1N][C]
    const float* W2;       // [S][NP][C]
    const float* gB;       // [N][D_OUT][C]
    float* B;              // [N][D_OUT][C]
    float* dA;             // [N][D_A][C]
    float* dw_part;        // [warps][S][NW][C]
    int N, C, S, warps;
    unsigned* status;
};

constexpr int kSymWarps = 4;

template <class K>
__global__ void __launch_bounds__(kSymWarps * 32) eqconv_symc_fwd_kernel(const SymParams prm) {
    constexpr int V = K::VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = prm.C, c = blockIdx.y * K::TILE_C + lane * V;
    const bool on = c < C;
    for (int i = blockIdx.x * kSymWarps + warp; i < prm.N; i += gridDim.x * kSymWarps) {
        const int z = prm.species[i];
        const bool zok = (unsigned)z < (unsigned)prm.S;
        if (!zok && lane == 0) atomicOr(prm.status, 1u);
        float a[K::D_A][V], b[K::D_OUT][V];
        const float* Ai = prm.A + (size_t)i * K::D_A * C + c;
#pragma unroll
        for (int d = 0; d < K::D_A; ++d) {
            if (on && zok)
                ld_stream<V>(a[d], Ai + (size_t)d * C, policy_evict_first());
            else
#pragma unroll
                for (int v = 0; v < V; ++v) a[d][v] = 0.f;
        }
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d)
#pragma unroll
            for (int v = 0; v < V; ++v) b[d][v] = 0.f;
        const float* w1 = prm.W1 + ((size_t)(zok ? z : 0) * K::L1N) * C + c;
        const float* w2 = prm.W2 + ((size_t)(zok ? z : 0) * K::NP) * C + c;
        static_for<K::L1N>([&](auto Lc) {
            constexpr int L = EQC_CV(Lc);
            float w[V];
#pragma unroll
            for (int v = 0; v < V; ++v) w[v] = on ? __ldg(w1 + (size_t)L * C + v) : 0.f;
#pragma unroll
            for (int m = 0; m < 2 * L + 1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) b[L * L + m][v] = w[v] * a[L * L + m][v];
        });
        static_for<K::NP>([&](auto pc) {
            constexpr int q = EQC_CV(pc);
            constexpr int l1 = K::PL.l1[q], l2 = K::PL.l2[q], L = K::PL.l3[q];
            float w[V];
#pragma unroll
            for (int v = 0; v < V; ++v) w[v] = on ? __ldg(w2 + (size_t)q * C + v) : 0.f;
            static_for<2 * L + 1>([&](auto Mc) {
                constexpr int M = EQC_CV(Mc);
                float t[V];
#pragma unroll
                for (int v = 0; v < V; ++v) t[v] = 0.f;
                static_for<2 * l1 + 1>([&](auto m1c) {
                    constexpr int m1 = EQC_CV(m1c);
                    static_for<2 * l2 + 1>([&](auto m2c) {
                        constexpr int m2 = EQC_CV(m2c);
                        constexpr double cg = RealCG<l1, l2, L>::t.v[m1][m2][M];
                        if constexpr (cg != 0.0) {
#pragma unroll
                            for (int v = 0; v < V; ++v)
                                t[v] = fmaf((float)cg * a[l1 * l1 + m1][v], a[l2 * l2 + m2][v], t[v]);
                        }
                    });
                });
#pragma unroll
                for (int v = 0; v < V; ++v) b[L * L + M][v] = fmaf(w[v], t[v], b[L * L + M][v]);
            });
        });
        if (on) {
            float* Bi = prm.B + (size_t)i * K::D_OUT * C + c;
#pragma unroll
            for (int d = 0; d < K::D_OUT; ++d) st_stream<V>(Bi + (size_t)d * C, b[d]);
        }
    }
}

// dynamic shared memory: kSymWarps * S * NW * TILE_C floats (weight-gradient
// partials, one row of TILE_C channels per (species, weight row) per warp)
template <class K>
__global__ void __launch_bounds__(kSymWarps * 32) eqconv_symc_bwd_kernel(const SymParams prm) {
    constexpr int V = K::VEC;
    extern __shared__ float sym_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = prm.C, c = blockIdx.y * K::TILE_C + lane * V;
    const bool on = c < C;
    float* part = sym_smem + (size_t)warp * prm.S * K::NW * K::TILE_C;   // [S][NW][TILE_C]
    for (int k = lane; k < prm.S * K::NW * K::TILE_C; k += 32) part[k] = 0.f;
    __syncwarp();
    for (int i = blockIdx.x * kSymWarps + warp; i < prm.N; i += gridDim.x * kSymWarps) {
        const int z = prm.species[i];
        const bool zok = (unsigned)z < (unsigned)prm.S;
        if (!zok && lane == 0) atomicOr(prm.status, 1u);
        float a[K::D_A][V], g[K::D_OUT][V], da[K::D_A][V];
        const float* Ai = prm.A + (size_t)i * K::D_A * C + c;
        const float* Gi = prm.gB + (size_t)i * K::D_OUT * C + c;
#pragma unroll
        for (int d = 0; d < K::D_A; ++d) {
#pragma unroll
            for (int v = 0; v < V; ++v) da[d][v] = 0.f;
            if (on && zok)
                ld_stream<V>(a[d], Ai + (size_t)d * C, policy_evict_first());
            else
#pragma unroll
                for (int v = 0; v < V; ++v) a[d][v] = 0.f;
        }
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) {
            if (on && zok)
                ld_stream<V>(g[d], Gi + (size_t)d * C, policy_evict_first());
            else
#pragma unroll
                for (int v = 0; v < V; ++v) g[d][v] = 0.f;
        }
        const int zz = zok ? z : 0;
        const float* w1 = prm.W1 + ((size_t)zz * K::L1N) * C + c;
        const float* w2 = prm.W2 + ((size_t)zz * K::NP) * C + c;
        float* pz = part + (size_t)zz * K::NW * K::TILE_C + lane * V;
        static_for<K::L1N>([&](auto Lc) {
            constexpr int L = EQC_CV(Lc);
            float w[V], s[V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                w[v] = on ? __ldg(w1 + (size_t)L * C + v) : 0.f;
                s[v] = 0.f;
            }
#pragma unroll
            for (int m = 0; m < 2 * L + 1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    da[L * L + m][v] = fmaf(w[v], g[L * L + m][v], da[L * L + m][v]);
                    s[v] = fmaf(a[L * L + m][v], g[L * L + m][v], s[v]);
                }
#pragma unroll
            for (int v = 0; v < V; ++v) pz[L * K::TILE_C + v] += s[v];
        });
        static_for<K::NP>([&](auto pc) {
            constexpr int q = EQC_CV(pc);
            constexpr int l1 = K::PL.l1[q], l2 = K::PL.l2[q], L = K::PL.l3[q];
            float w[V], s[V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                w[v] = on ? __ldg(w2 + (size_t)q * C + v) : 0.f;
                s[v] = 0.f;
            }
            static_for<2 * L + 1>([&](auto Mc) {
                constexpr int M = EQC_CV(Mc);
                static_for<2 * l1 + 1>([&](auto m1c) {
                    constexpr int m1 = EQC_CV(m1c);
                    static_for<2 * l2 + 1>([&](auto m2c) {
                        constexpr int m2 = EQC_CV(m2c);
                        constexpr double cg = RealCG<l1, l2, L>::t.v[m1][m2][M];
                        if constexpr (cg != 0.0) {
#pragma unroll
                            for (int v = 0; v < V; ++v) {
                                const float cgv = (float)cg * g[L * L + M][v];
                                const float wc = w[v] * cgv;
                                da[l1 * l1 + m1][v] = fmaf(wc, a[l2 * l2 + m2][v], da[l1 * l1 + m1][v]);
                                da[l2 * l2 + m2][v] = fmaf(wc, a[l1 * l1 + m1][v], da[l2 * l2 + m2][v]);
                                s[v] = fmaf(cgv * a[l1 * l1 + m1][v], a[l2 * l2 + m2][v], s[v]);
                            }
                        }
                    });
                });
            });
#pragma unroll
            for (int v = 0; v < V; ++v) pz[(K::L1N + q) * K::TILE_C + v] += s[v];
        });
        if (on) {
            float* dAi = prm.dA + (size_t)i * K::D_A * C + c;
#pragma unroll
            for (int d = 0; d < K::D_A; ++d) st_stream<V>(dAi + (size_t)d * C, da[d]);
        }
    }
    __syncwarp();
    // this warp's partials -> dw_part[warp][s][row][tile channels]
    const int gw = blockIdx.x * kSymWarps + warp;
    for (int k = lane; k < prm.S * K::NW * K::TILE_C; k += 32) {
        const int ch = k % K::TILE_C, row = k / K::TILE_C;   // row = s * NW + weight row
        const int cc = blockIdx.y * K::TILE_C + ch;
        if (cc < C) prm.dw_part[((size_t)gw * prm.S * K::NW + row) * C + cc] = part[k];
    }
}

// dW[s][row][c] = sum over warps, in order, of dw_part[warp][s][row][c];
// rows < L1N go to dW1 [S][L1N][C], the others to dW2 [S][NP][C].
template <class K>
__global__ void eqconv_symc_dw_reduce(const float* __restrict__ part, int warps, int S, int C, float* __restrict__ dW1,
                                      float* __restrict__ dW2) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)S * K::NW * C;
    if (idx >= total) return;
    float s = 0.f;
    for (int w = 0; w < warps; ++w) s += part[(size_t)w * total + idx];
    const int c = (int)(idx % C);
    const int row = (int)((idx / C) % K::NW);
    const int sp = (int)(idx / ((int64_t)C * K::NW));
    if (row < K::L1N)
        dW1[((size_t)sp * K::L1N + row) * C + c] = s;
    else
        dW2[((size_t)sp * K::NP + (row - K::L1N)) * C + c] = s;
}

}  // namespace eqc

// Double backward of the convolution: the VJP of eqconv_backward (device
// code).
//
// FlashCart (arXiv 2610.06409) §2: training on forces differentiates the
// force evaluation; §3 and App. C: for a weighted bilinear product the
// VJP-of-VJP follows from bilinearity as linear-map evaluations; App. D: it
// sums receiver contributions to the derivative of the incoming gradient and
// keeps all of a receiver's edges in one program.
//
// With cotangents a (of dx), b (of dw) and q (of dr) and rho_e = (dY/dr)(r_e) q_e,
// the gradient of S = <a,dx> + <b,dw> + <q,dr> is
//   g_gy[i] = sum_{e->i} sum_p [ w_p (A_p(Y) a_s + A_p(rho) x_s) + b_p A_p(Y) x_s ]
//   g_x[j]  = sum_{j->e} sum_p [ b_p A_p(Y)^T gy_i + w_p A_p(rho)^T gy_i ]
//   g_w[e]  = a_s . A_p(Y)^T gy_i + x_s . A_p(rho)^T gy_i
//   g_r[e]  = (dY/dr)^T gYv_e + H(r_e; gY1_e) q_e,
//     gYv[l2 m2] = sum_c sum_p (w_p G_p(a, gy) + b_p G_p(x, gy))[m2],
//     gY1[l2 m2] = sum_c sum_p w_p G_p(x, gy)[m2],
//     G_p(u, g)[m2] = sum_{m1,m3} C_p[m1,m2,m3] u[m1] g[m3],
// with A_p(Y)[m3][m1] = sum_m2 C_p[m1,m2,m3] Y[l2 m2] as in the forward.
//
// Three launches, all deterministic (no atomics):
//   * receiver pass (receiver CSR): g_gy, one warp per receiver and channel
//     tile, sums in registers; it contracts C directly with
//     Y (w a + b x) + rho (w x), one product per nonzero CG row;
//   * sender pass (sender CSR): g_x in registers, g_w stored per edge, the
//     per-tile partials of gYv and gY1 (one warp transpose-sum, fixed order)
//     to a workspace [E][T][2G]; it contracts through h = C.gy;
//   so neither pass builds coupling matrices: each needs only the edge's Y
//   and rho;
//   * r epilogue (one thread per edge): sums the tiles in order and applies
//     the gradient and the Hessian-vector product of the harmonics.
// Each warp stages its edges' rows through a ring of shared-memory stages
// filled by tensor-map copies (as the first-order kernels do), K::STAGES
// edges ahead: the receiver pass copies w_e, b_e, x_s and a_s per edge, the
// sender pass w_e, b_e and gy_i.
#pragma once

#include "eqc_conv.cuh"

namespace eqc {

struct DblParams {
    const float* x;
    const float* a;    // cotangent of dx  [N][D_in][C]
    const float* r;
    const float* q;    // cotangent of dr  [E][3]
    const float* w;
    const float* b;    // cotangent of dw  [E][P][C]
    const float* gy;
    float* g_x;
    float* g_w;
    float* g_gy;
    float* g_r;
    float* part;       // [E][T][2G]
    const int* ptr;    // receiver pass: recv_ptr   sender pass: send_ptr
    const int* perm;   // receiver pass: recv_perm  sender pass: send_perm
    const int* other;  // receiver pass: senders    sender pass: receivers
    int N, C, T, E;
    unsigned* status;
};

template <class K>
struct DblShape {
    static constexpr int CH = 8;   // edges whose harmonics (Y, rho) one batch evaluates
};

template <int V>
__device__ __forceinline__ void ldg_vec(float* d, const float* p) {
    if constexpr (V == 1) {
        d[0] = __ldg(p);
    } else if constexpr (V == 2) {
        const float2 t = __ldg(reinterpret_cast<const float2*>(p));
        d[0] = t.x;
        d[1] = t.y;
    } else {
        const float4 t = __ldg(reinterpret_cast<const float4*>(p));
        d[0] = t.x;
        d[1] = t.y;
        d[2] = t.z;
        d[3] = t.w;
    }
}

// rows [n][C] -> this lane's V channels of each row (zeros when inactive)
template <int V, int R>
__device__ __forceinline__ void load_rows(float (&d)[R][V], const float* base, int C, bool on) {
#pragma unroll
    for (int k = 0; k < R; ++k) {
        if (on) {
            ldg_vec<V>(d[k], base + (size_t)k * C);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) d[k][v] = 0.f;
        }
    }
}

// This lane's V channels of stage row `row` (zeros when the lane is past C;
// the predicate also keeps the compiler from hoisting every row load of the
// edge into registers).
template <class K>
__device__ __forceinline__ void stage_row(float (&d)[K::VEC], const float* st, int row, int cl, bool rd) {
    if (rd) {
        lds_vec<K::VEC>(d, st + row * K::TILE_C + cl);
    } else {
#pragma unroll
        for (int v = 0; v < K::VEC; ++v) d[v] = 0.f;
    }
}

// acc[o3] += w_p (A_p(Y) a + A_p(rho) x) + b_p A_p(Y) x for every path, in
// the form that needs no coupling matrices: with s1 = w a + b x and s2 = w x
// (per channel), acc[m3] += sum_{m1, m2} C_p[m1, m2, m3] (Y[m2] s1[m1] +
// rho[m2] s2[m1]), one product per nonzero (m1, m2) row of C_p.  Yrow holds
// the edge's Y, then rho.
// The edge's rows: read from its stage path by path (PRE = false: fewer live
// registers, for wide channel tiles) or taken from arrays the caller loaded
// up front (PRE = true).
template <class K>
struct DblRecvRows {
    float w[K::NP][K::VEC], b[K::NP][K::VEC], x[K::D_IN][K::VEC], a[K::D_IN][K::VEC];
};
template <class K, bool PRE>
__device__ __forceinline__ void dbl_recv_edge(const float* st, int cl, bool rd, const DblRecvRows<K>& pre,
                                              const float* Yrow, float (&acc)[K::D_OUT][K::VEC]) {
    constexpr int V = K::VEC;
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o2 = l2 * l2, o3 = K::PL.o3[p];
        float w[V], b[V];
        float xv[d1][V], av[d1][V];
        if constexpr (PRE) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                w[v] = pre.w[p][v];
                b[v] = pre.b[p][v];
            }
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    xv[m][v] = pre.x[o1 + m][v];
                    av[m][v] = pre.a[o1 + m][v];
                }
        } else {
            constexpr int XR = 2 * K::NP + o1, AR = 2 * K::NP + K::D_IN + o1;   // stage rows of x_l1, a_l1
            stage_row<K>(w, st, p, cl, rd);
            stage_row<K>(b, st, K::NP + p, cl, rd);
#pragma unroll
            for (int m = 0; m < d1; ++m) {
                stage_row<K>(xv[m], st, XR + m, cl, rd);
                stage_row<K>(av[m], st, AR + m, cl, rd);
            }
        }
        if constexpr (l2 == 0) {       // A(Y) = I, A(rho) = 0
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v)
                    acc[o3 + m][v] = fmaf(w[v], av[m][v], fmaf(b[v], xv[m][v], acc[o3 + m][v]));
        } else {
            float s1[d1][V], s2[d1][V];
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    s1[m][v] = fmaf(w[v], av[m][v], b[v] * xv[m][v]);
                    s2[m][v] = w[v] * xv[m][v];
                }
            static_for<d2>([&](auto m2c) {
                constexpr int m2 = EQC_CV(m2c);
                const float y2 = Yrow[o2 + m2], r2 = Yrow[K::D_SH + o2 + m2];
                static_for<d1>([&](auto m1c) {
                    constexpr int m1 = EQC_CV(m1c);
                    if constexpr (cg_row_nonzero<l1, l2, l3>(m1, m2)) {
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            const float z = fmaf(y2, s1[m1][v], r2 * s2[m1][v]);
                            static_for<d3>([&](auto m3c) {
                                constexpr int m3 = EQC_CV(m3c);
                                constexpr double c = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                                if constexpr (c != 0.0) acc[o3 + m3][v] = fmaf((float)c, z, acc[o3 + m3][v]);
                            });
                        }
                    }
                });
            });
        }
    });
}

// Sender-side terms of one edge: g_x, g_w (stored per path), and this lane's
// partials of gYv and gY1 (summed over its channels).  With
// h[m1][m2] = sum_m3 C_p[m1,m2,m3] gy[m3] (per channel), one h serves all four
// contractions: A_p(Y)^T gy = sum_m2 Y[m2] h, A_p(rho)^T gy = sum_m2 rho[m2] h,
// G_p(a, gy) = sum_m1 a[m1] h and G_p(x, gy) = sum_m1 x[m1] h; so the pass
// needs only each edge's Y and rho, not its coupling matrices.
// The edge's rows (w, b, gy): from its stage path by path, or (PRE) from
// arrays the caller loaded up front.
template <class K>
struct DblSendRows {
    float w[K::NP][K::VEC], b[K::NP][K::VEC], g[K::D_OUT][K::VEC];
};
template <class K, bool PRE>
__device__ __forceinline__ void dbl_send_edge(const float* st, int cl, bool rd, const DblSendRows<K>& pre,
                                              const float* Yrow, const float (&xv)[K::D_IN][K::VEC],
                                              const float (&av)[K::D_IN][K::VEC],
                                              float (&gacc)[K::D_IN][K::VEC], float* gw_row, int C, bool on,
                                              float* gYv, float* gY1) {
    constexpr int V = K::VEC;
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
        constexpr int o1 = l1 * l1, o2 = l2 * l2, o3 = K::PL.o3[p];
        float wv[V], bv[V], gv[d3][V];
        if constexpr (PRE) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                wv[v] = pre.w[p][v];
                bv[v] = pre.b[p][v];
            }
#pragma unroll
            for (int m = 0; m < d3; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) gv[m][v] = pre.g[o3 + m][v];
        } else {
            stage_row<K>(wv, st, p, cl, rd);
            stage_row<K>(bv, st, K::NP + p, cl, rd);
#pragma unroll
            for (int m = 0; m < d3; ++m) stage_row<K>(gv[m], st, 2 * K::NP + o3 + m, cl, rd);
        }
        float uY[d1][V], uR[d1][V];
        if constexpr (l2 == 0) {       // A(Y) = I, A(rho) = 0
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    uY[m][v] = gv[m][v];
                    uR[m][v] = 0.f;
                }
        } else {
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) uY[m][v] = uR[m][v] = 0.f;
            static_for<d2>([&](auto m2c) {
                constexpr int m2 = EQC_CV(m2c);
                const float y2 = Yrow[o2 + m2], r2 = Yrow[K::D_SH + o2 + m2];
                float Ga[V], Gx[V];
#pragma unroll
                for (int v = 0; v < V; ++v) Ga[v] = Gx[v] = 0.f;
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
                            uY[m1][v] = fmaf(y2, h, uY[m1][v]);
                            uR[m1][v] = fmaf(r2, h, uR[m1][v]);
                            Ga[v] = fmaf(av[o1 + m1][v], h, Ga[v]);
                            Gx[v] = fmaf(xv[o1 + m1][v], h, Gx[v]);
                        }
                    }
                });
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    gYv[o2 + m2 - 1] = fmaf(wv[v], Ga[v], fmaf(bv[v], Gx[v], gYv[o2 + m2 - 1]));
                    gY1[o2 + m2 - 1] = fmaf(wv[v], Gx[v], gY1[o2 + m2 - 1]);
                }
            });
        }
        float gw[V];
#pragma unroll
        for (int v = 0; v < V; ++v) gw[v] = 0.f;
#pragma unroll
        for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
            for (int v = 0; v < V; ++v) {
                gacc[o1 + m1][v] = fmaf(bv[v], uY[m1][v], fmaf(wv[v], uR[m1][v], gacc[o1 + m1][v]));
                gw[v] = fmaf(av[o1 + m1][v], uY[m1][v], fmaf(xv[o1 + m1][v], uR[m1][v], gw[v]));
            }
        if (on) st_stream<V>(gw_row + (size_t)p * C, gw);
    });
}

// Per-warp shared memory of the two passes (floats, regions 128-byte
// aligned): [stages: S x ROWS x TILE_C] [mbarriers] [per-batch rows].
// Receiver pass: rows w (NP), b (NP), x (D_IN), a (D_IN) per stage; sender
// pass: rows w, b, gy (D_OUT); both keep the batch's harmonics Y, rho.
template <class K, bool RECV>
struct DblRing {
    static constexpr int S = K::STAGES;
    static constexpr int CH = DblShape<K>::CH;
    static constexpr int up32(int f) { return (f + 31) & ~31; }
    static constexpr int ROWS = RECV ? 2 * K::NP + 2 * K::D_IN : 2 * K::NP + K::D_OUT;
    static constexpr int SF = ROWS * K::TILE_C;                       // floats per stage
    static constexpr uint32_t STAGE_BYTES = SF * 4;
    static constexpr int ST_F = S * SF;
    static constexpr int BAR_F = up32(4 * S);
    static constexpr int ROW_F = up32(CH * 2 * K::D_SH);   // per edge of a batch: Y, then rho
    static constexpr int TOTAL_F = ST_F + BAR_F + ROW_F;
    static constexpr int WARPS = best_warps(TOTAL_F * 4);
    static constexpr int SMEM = WARPS * TOTAL_F * 4;
};

// Fill stage `st` for edge e and its other end o: the edge's w and b rows,
// then the node rows of the two node maps (a null second map: one node map).
template <class K, bool RECV>
__device__ __forceinline__ void dbl_fill(float* st, uint64_t* bar, const CUtensorMap* tw, const CUtensorMap* tb,
                                         const CUtensorMap* tn0, const CUtensorMap* tn1, int e, int o, int c0,
                                         uint64_t pol_e, uint64_t pol_n, int lane) {
    if (lane == 0) {
        constexpr int DN = RECV ? K::D_IN : K::D_OUT;
        fence_proxy_async();
        mbar_expect_tx(bar, DblRing<K, RECV>::STAGE_BYTES + EQC_TEST_FILL_DEFICIT);
        tma_rows(st, tw, c0, e, bar, pol_e);
        tma_rows(st + K::NP * K::TILE_C, tb, c0, e, bar, pol_e);
        tma_rows(st + 2 * K::NP * K::TILE_C, tn0, c0, o, bar, pol_n);
        if constexpr (RECV) tma_rows(st + (2 * K::NP + DN) * K::TILE_C, tn1, c0, o, bar, pol_n);
    }
}

// Receiver pass: g_gy.  One warp per receiver and channel tile.
template <class K>
__global__ void __launch_bounds__(DblRing<K, true>::WARPS * 32)
    eqconv_dbl_recv_kernel(const DblParams prm, const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_a) {
    using L = DblRing<K, true>;
    constexpr int V = K::VEC, S = L::S, CH = L::CH, W = L::WARPS, SF = L::SF;
    extern __shared__ __align__(128) float4 smem4[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * W + warp;
    if (node >= prm.N) return;
    float* stages = reinterpret_cast<float*>(smem4) + warp * L::TOTAL_F;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + L::ST_F);
    float* Ys = stages + L::ST_F + L::BAR_F;   // rows of 2 D_SH: Y then rho
    const int C = prm.C;
    const int c0 = blockIdx.y * K::TILE_C, cl = lane * V;
    const bool on = c0 + cl < C;
    const uint64_t pol_e = policy_evict_first(), pol_n = policy_evict_last();
    if (lane == 0) {
        for (int q = 0; q < S; ++q) mbar_init(&bars[2 * q], 1);
        mbar_fence_init();
    }
    __syncwarp();
    float acc[K::D_OUT][V];
#pragma unroll
    for (int d = 0; d < K::D_OUT; ++d)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[d][v] = 0.f;
    uint32_t g = 0;   // edges staged so far (stage g % S, phase (g / S) & 1)
    bool ok_all = true;
    uint32_t fill_from = 0, fill_to = 0;
    int k = prm.ptr[node];
    const int ke = prm.ptr[node + 1];
    while (k < ke && ok_all) {
        int my_e, my_s;
        float rx, ry, rz;
        const int n = gather_window(prm.perm, prm.other, prm.r, prm.N, 0, prm.N, k, ke, prm.status, lane, my_e,
                                    my_s, rx, ry, rz);
        if (n == 0) continue;
        const int pre = min(S, n);
        for (int t = 0; t < pre; ++t) {
            const int e = __shfl_sync(0xffffffffu, my_e, t), o = __shfl_sync(0xffffffffu, my_s, t);
            const uint32_t gi = g + t;
            dbl_fill<K, true>(stages + (gi % S) * SF, &bars[2 * (gi % S)], &tmap_w, &tmap_b, &tmap_x, &tmap_a, e,
                              o, c0, pol_e, pol_n, lane);
        }
        for (int b0 = 0; b0 < n && ok_all; b0 += CH) {
            const int nb = min(CH, n - b0);
            if (lane >= b0 && lane < b0 + nb) {
                const float* qe = prm.q + 3 * (size_t)my_e;
                float ux, uy, uz, il;
                const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                float Y[K::D_SH], rho[K::D_SH];
                sh_eval<K::LSH>(ok, ux, uy, uz, Y);
                sh_jvp<K::LSH>(rx, ry, rz, qe[0], qe[1], qe[2], rho);
                float* yrow = Ys + (lane - b0) * 2 * K::D_SH;
#pragma unroll
                for (int q = 0; q < K::D_SH; ++q) {
                    yrow[q] = Y[q];
                    yrow[K::D_SH + q] = rho[q];
                }
            }
            __syncwarp();
            for (int t = b0; t < b0 + nb; ++t) {
                const uint32_t gi = g + t;
                float* st = stages + (gi % S) * SF;
                if (!mbar_wait(&bars[2 * (gi % S)], (gi / S) & 1u)) {
                    if (lane == 0) atomicOr(prm.status, 4u);
                    ok_all = false;
                    fill_from = gi;
                    fill_to = g + (uint32_t)min(n, t + S);
                    break;
                }
                // 32-channel tiles take every row up front, wider ones read them on demand
                constexpr bool PRE = V == 1;
                DblRecvRows<K> rows;
                if constexpr (PRE) {
#pragma unroll
                    for (int p = 0; p < K::NP; ++p) {
                        lds_vec<V>(rows.w[p], st + p * K::TILE_C + cl);
                        lds_vec<V>(rows.b[p], st + (K::NP + p) * K::TILE_C + cl);
                    }
#pragma unroll
                    for (int d = 0; d < K::D_IN; ++d) {
                        lds_vec<V>(rows.x[d], st + (2 * K::NP + d) * K::TILE_C + cl);
                        lds_vec<V>(rows.a[d], st + (2 * K::NP + K::D_IN + d) * K::TILE_C + cl);
                    }
                }
                dbl_recv_edge<K, PRE>(st, cl, on, rows, Ys + (t - b0) * 2 * K::D_SH, acc);
                __syncwarp();
                if (t + S < n) {
                    const int e = __shfl_sync(0xffffffffu, my_e, t + S), o = __shfl_sync(0xffffffffu, my_s, t + S);
                    dbl_fill<K, true>(st, &bars[2 * (gi % S)], &tmap_w, &tmap_b, &tmap_x, &tmap_a, e, o, c0, pol_e,
                                      pol_n, lane);
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
    if (on) {
        float* gi = prm.g_gy + (size_t)node * K::D_OUT * C + c0 + cl;
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) st_stream<V>(gi + (size_t)d * C, acc[d]);
    }
}

// Sender pass: g_x, g_w and the per-tile partials of gYv, gY1.  One warp per
// sender and channel tile; x_j and a_j stay in registers.
template <class K>
__global__ void __launch_bounds__(DblRing<K, false>::WARPS * 32)
    eqconv_dbl_send_kernel(const DblParams prm, const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_g) {
    using L = DblRing<K, false>;
    constexpr int V = K::VEC, S = L::S, CH = L::CH, W = L::WARPS, SF = L::SF;
    constexpr int G = K::G > 0 ? K::G : 1;
    extern __shared__ __align__(128) float4 smem4[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * W + warp;
    if (node >= prm.N) return;
    float* stages = reinterpret_cast<float*>(smem4) + warp * L::TOTAL_F;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + L::ST_F);
    float* Ys = stages + L::ST_F + L::BAR_F;   // rows of 2 D_SH: Y then rho
    const int C = prm.C;
    const int tile = blockIdx.y;
    const int c0 = tile * K::TILE_C, cl = lane * V;
    const bool on = c0 + cl < C;
    const uint64_t pol_e = policy_evict_first(), pol_n = policy_evict_last();
    if (lane == 0) {
        for (int q = 0; q < S; ++q) mbar_init(&bars[2 * q], 1);
        mbar_fence_init();
    }
    __syncwarp();
    float xv[K::D_IN][V], av[K::D_IN][V], gacc[K::D_IN][V];
    load_rows<V>(xv, prm.x + (size_t)node * K::D_IN * C + c0 + cl, C, on);
    load_rows<V>(av, prm.a + (size_t)node * K::D_IN * C + c0 + cl, C, on);
#pragma unroll
    for (int d = 0; d < K::D_IN; ++d)
#pragma unroll
        for (int v = 0; v < V; ++v) gacc[d][v] = 0.f;
    uint32_t g = 0;
    bool ok_all = true;
    uint32_t fill_from = 0, fill_to = 0;
    int k = prm.ptr[node];
    const int ke = prm.ptr[node + 1];
    while (k < ke && ok_all) {
        int my_e, my_i;
        float rx, ry, rz;
        const int n = gather_window(prm.perm, prm.other, prm.r, prm.N, 0, prm.N, k, ke, prm.status, lane, my_e,
                                    my_i, rx, ry, rz);
        if (n == 0) continue;
        const int pre = min(S, n);
        for (int t = 0; t < pre; ++t) {
            const int e = __shfl_sync(0xffffffffu, my_e, t), o = __shfl_sync(0xffffffffu, my_i, t);
            const uint32_t gi = g + t;
            dbl_fill<K, false>(stages + (gi % S) * SF, &bars[2 * (gi % S)], &tmap_w, &tmap_b, &tmap_g, nullptr, e,
                               o, c0, pol_e, pol_n, lane);
        }
        for (int b0 = 0; b0 < n && ok_all; b0 += CH) {
            const int nb = min(CH, n - b0);
            if (lane >= b0 && lane < b0 + nb) {
                const float* qe = prm.q + 3 * (size_t)my_e;
                float ux, uy, uz, il;
                const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                float Y[K::D_SH], rho[K::D_SH];
                sh_eval<K::LSH>(ok, ux, uy, uz, Y);
                sh_jvp<K::LSH>(rx, ry, rz, qe[0], qe[1], qe[2], rho);
                float* yrow = Ys + (lane - b0) * 2 * K::D_SH;
#pragma unroll
                for (int q = 0; q < K::D_SH; ++q) {
                    yrow[q] = Y[q];
                    yrow[K::D_SH + q] = rho[q];
                }
            }
            __syncwarp();
            for (int t = b0; t < b0 + nb; ++t) {
                const uint32_t gi = g + t;
                float* st = stages + (gi % S) * SF;
                if (!mbar_wait(&bars[2 * (gi % S)], (gi / S) & 1u)) {
                    if (lane == 0) atomicOr(prm.status, 4u);
                    ok_all = false;
                    fill_from = gi;
                    fill_to = g + (uint32_t)min(n, t + S);
                    break;
                }
                const int e = __shfl_sync(0xffffffffu, my_e, t);
                float gYv[G], gY1[G];
#pragma unroll
                for (int q = 0; q < G; ++q) gYv[q] = gY1[q] = 0.f;
                constexpr bool PRE = V == 1;
                DblSendRows<K> rows;
                if constexpr (PRE) {
#pragma unroll
                    for (int p = 0; p < K::NP; ++p) {
                        lds_vec<V>(rows.w[p], st + p * K::TILE_C + cl);
                        lds_vec<V>(rows.b[p], st + (K::NP + p) * K::TILE_C + cl);
                    }
#pragma unroll
                    for (int d = 0; d < K::D_OUT; ++d) lds_vec<V>(rows.g[d], st + (2 * K::NP + d) * K::TILE_C + cl);
                }
                dbl_send_edge<K, PRE>(st, cl, on, rows, Ys + (t - b0) * 2 * K::D_SH, xv, av, gacc,
                                      prm.g_w + (size_t)e * K::NP * C + c0 + cl, C, on, gYv, gY1);
                __syncwarp();
                if (t + S < n) {
                    const int e2 = __shfl_sync(0xffffffffu, my_e, t + S), o2 = __shfl_sync(0xffffffffu, my_i, t + S);
                    dbl_fill<K, false>(st, &bars[2 * (gi % S)], &tmap_w, &tmap_b, &tmap_g, nullptr, e2, o2, c0,
                                       pol_e, pol_n, lane);
                }
                if constexpr (K::G > 0) {
                    // the 2G partials summed over the warp at once; value q lands on lanes q << SH ..
                    constexpr int NV = pow2_at_least(2 * G), SH = transpose_sum_shift(NV);
                    float tv[NV];
#pragma unroll
                    for (int q = 0; q < NV; ++q) tv[q] = q < G ? gYv[q] : (q < 2 * G ? gY1[q - G] : 0.f);
                    const float sum = warp_transpose_sum<NV>(tv, lane);
                    const int q = lane >> SH;
                    if ((lane & ((1 << SH) - 1)) == 0 && q < 2 * G)
                        prm.part[((size_t)e * prm.T + tile) * 2 * G + q] = sum;
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
    if (on) {
        float* gj = prm.g_x + (size_t)node * K::D_IN * C + c0 + cl;
#pragma unroll
        for (int d = 0; d < K::D_IN; ++d) st_stream<V>(gj + (size_t)d * C, gacc[d]);
    }
}

// g_r[e] = (dY/dr)^T gYv + H(r; gY1) q, the tiles summed in order.
template <int LSH>
__global__ void eqconv_dbl_r_epilogue(const float* part, int T, const float* r, const float* q, float* g_r, int E) {
    constexpr int G = (LSH + 1) * (LSH + 1) - 1;
    constexpr int GG = G > 0 ? G : 1;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    float gv[GG], g1[GG];
#pragma unroll
    for (int k = 0; k < GG; ++k) gv[k] = g1[k] = 0.f;
    if constexpr (G > 0) {
        for (int t = 0; t < T; ++t) {
            const float* pp = part + ((size_t)e * T + t) * 2 * G;
#pragma unroll
            for (int k = 0; k < G; ++k) {
                gv[k] += pp[k];
                g1[k] += pp[G + k];
            }
        }
    }
    const float* re = r + (size_t)e * 3;
    const float* qe = q + (size_t)e * 3;
    float grad_v[3] = {0.f, 0.f, 0.f}, grad_1[3], hq[3];
    if constexpr (G > 0) {
        float ux, uy, uz, il;
        const bool ok = unit_dir(re[0], re[1], re[2], ux, uy, uz, il);
        sh_grad_contract<LSH>(ok, ux, uy, uz, il, gv, grad_v[0], grad_v[1], grad_v[2]);
    }
    sh_grad_and_hvp<LSH>(re[0], re[1], re[2], qe[0], qe[1], qe[2], g1, grad_1, hq);
#pragma unroll
    for (int k = 0; k < 3; ++k) g_r[(size_t)e * 3 + k] = grad_v[k] + hq[k];
}

}  // namespace eqc

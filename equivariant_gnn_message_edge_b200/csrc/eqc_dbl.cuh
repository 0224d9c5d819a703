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
//     tile, sums in registers;
//   * sender pass (sender CSR): g_x in registers, g_w stored per edge, the
//     per-tile partials of gYv and gY1 (warp butterfly, fixed order) to a
//     workspace [E][T][2G]; it contracts through h = C.gy and needs only
//     each edge's Y and rho, not its coupling matrices;
//   * r epilogue (one thread per edge): sums the tiles in order and applies
//     the gradient and the Hessian-vector product of the harmonics.
// Rows are read with plain vector loads (no staging ring): the double
// backward is a training-time op with twice the streamed bytes of the
// backward (w and b).
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

#ifndef EQC_DBL_PREFETCH
#define EQC_DBL_PREFETCH 1   // load the next edge's rows while the current edge is computed
#endif

template <class K>
struct DblShape {
    // prefetching doubles the row registers: it paid at lmax 2 (17.3 -> 16.7 ms)
    // and cost at lmax 3 (41.6 -> 46.8 ms), where the per-edge code is larger
    static constexpr bool PF = EQC_DBL_PREFETCH && K::NA_PAD <= 128;
    static constexpr int CH = K::NA_PAD > 128 ? 4 : 8;        // edges per coupling batch
    // receiver pass: A(Y) and A(rho); sender pass: Y and rho
    static constexpr int WARP_FLOATS = 2 * CH * (K::NA_PAD > K::D_SH ? K::NA_PAD : K::D_SH);
    static constexpr int WARPS = 4;
    static constexpr int SMEM = WARPS * WARP_FLOATS * 4;
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

// Lane t of the warp: harmonics, their derivative along q, and the coupling
// matrices A(Y), A(rho) of edge e into shared memory.
template <class K>
__device__ __forceinline__ void dbl_couplings(const float* r, const float* q, int e, float* AY, float* AR) {
    const float rx = r[3 * (size_t)e], ry = r[3 * (size_t)e + 1], rz = r[3 * (size_t)e + 2];
    float ux, uy, uz, il;
    const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
    float Y[K::D_SH], rho[K::D_SH];
    sh_eval<K::LSH>(ok, ux, uy, uz, Y);
    sh_jvp<K::LSH>(rx, ry, rz, q[3 * (size_t)e], q[3 * (size_t)e + 1], q[3 * (size_t)e + 2], rho);
    compute_A<K>(Y, AY);
    compute_A<K>(rho, AR);
}

// Lane t of the warp: the harmonics Y and rho = (dY/dr) q of edge e into
// shared memory (rows of K::YS floats: Y first, then rho), for the sender
// pass, which needs no coupling matrices.
template <class K>
__device__ __forceinline__ void dbl_harmonics(const float* r, const float* q, int e, float* Yrow) {
    const float rx = r[3 * (size_t)e], ry = r[3 * (size_t)e + 1], rz = r[3 * (size_t)e + 2];
    float ux, uy, uz, il;
    const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
    float Y[K::D_SH], rho[K::D_SH];
    sh_eval<K::LSH>(ok, ux, uy, uz, Y);
    sh_jvp<K::LSH>(rx, ry, rz, q[3 * (size_t)e], q[3 * (size_t)e + 1], q[3 * (size_t)e + 2], rho);
#pragma unroll
    for (int k = 0; k < K::D_SH; ++k) {
        Yrow[k] = Y[k];
        Yrow[K::D_SH + k] = rho[k];
    }
}

// acc[o3] += w_p (A_p(Y) a + A_p(rho) x) + b_p A_p(Y) x for every path.
template <class K>
__device__ __forceinline__ void dbl_recv_edge(const float* AY, const float* AR, const float (&xv)[K::D_IN][K::VEC],
                                              const float (&av)[K::D_IN][K::VEC], const float (&wv)[K::NP][K::VEC],
                                              const float (&bv)[K::NP][K::VEC], float (&acc)[K::D_OUT][K::VEC]) {
    constexpr int V = K::VEC;
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o3 = K::PL.o3[p];
        if constexpr (l2 == 0) {       // A(Y) = I, A(rho) = 0
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v)
                    acc[o3 + m][v] = fmaf(wv[p][v], av[o1 + m][v], fmaf(bv[p][v], xv[o1 + m][v], acc[o3 + m][v]));
        } else {
            constexpr int n4 = (d1 * d3 + 3) / 4;
            constexpr int aoff = K::AO.off[p];
            float ay[n4 * 4], ar[n4 * 4];
            load_A<n4>(AY + aoff, ay);
            load_A<n4>(AR + aoff, ar);
#pragma unroll
            for (int m3 = 0; m3 < d3; ++m3) {
                float ta[V], tx[V], tr[V];
#pragma unroll
                for (int v = 0; v < V; ++v) ta[v] = tx[v] = tr[v] = 0.f;
#pragma unroll
                for (int m1 = 0; m1 < d1; ++m1)
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        ta[v] = fmaf(ay[m3 * d1 + m1], av[o1 + m1][v], ta[v]);
                        tx[v] = fmaf(ay[m3 * d1 + m1], xv[o1 + m1][v], tx[v]);
                        tr[v] = fmaf(ar[m3 * d1 + m1], xv[o1 + m1][v], tr[v]);
                    }
#pragma unroll
                for (int v = 0; v < V; ++v)
                    acc[o3 + m3][v] = fmaf(wv[p][v], ta[v] + tr[v], fmaf(bv[p][v], tx[v], acc[o3 + m3][v]));
            }
        }
    });
}

// Sender-side terms of one edge: g_x, g_w (stored per path), and this lane's
// partials of gYv and gY1 (summed over its channels).  With
// h[m1][m2] = sum_m3 C_p[m1,m2,m3] gy[m3] (per channel), one h serves all four
// contractions: A_p(Y)^T gy = sum_m2 Y[m2] h, A_p(rho)^T gy = sum_m2 rho[m2] h,
// G_p(a, gy) = sum_m1 a[m1] h and G_p(x, gy) = sum_m1 x[m1] h; so the pass
// needs only each edge's Y and rho, not its coupling matrices.
template <class K>
__device__ __forceinline__ void dbl_send_edge(const float* Yrow, const float (&xv)[K::D_IN][K::VEC],
                                              const float (&av)[K::D_IN][K::VEC],
                                              const float (&gv)[K::D_OUT][K::VEC],
                                              const float (&wv)[K::NP][K::VEC], const float (&bv)[K::NP][K::VEC],
                                              float (&gacc)[K::D_IN][K::VEC], float* gw_row, int C, bool on,
                                              float* gYv, float* gY1) {
    constexpr int V = K::VEC;
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p], l2 = K::PL.l2[p], l3 = K::PL.l3[p];
        constexpr int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
        constexpr int o1 = l1 * l1, o2 = l2 * l2, o3 = K::PL.o3[p];
        float uY[d1][V], uR[d1][V];
        if constexpr (l2 == 0) {       // A(Y) = I, A(rho) = 0
#pragma unroll
            for (int m = 0; m < d1; ++m)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    uY[m][v] = gv[o3 + m][v];
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
                                if constexpr (c != 0.0) h = fmaf((float)c, gv[o3 + m3][v], h);
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
                    gYv[o2 + m2 - 1] = fmaf(wv[p][v], Ga[v], fmaf(bv[p][v], Gx[v], gYv[o2 + m2 - 1]));
                    gY1[o2 + m2 - 1] = fmaf(wv[p][v], Gx[v], gY1[o2 + m2 - 1]);
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
                gacc[o1 + m1][v] = fmaf(bv[p][v], uY[m1][v], fmaf(wv[p][v], uR[m1][v], gacc[o1 + m1][v]));
                gw[v] = fmaf(av[o1 + m1][v], uY[m1][v], fmaf(xv[o1 + m1][v], uR[m1][v], gw[v]));
            }
        if (on) st_stream<V>(gw_row + (size_t)p * C, gw);
    });
}

// Rows of one edge for the receiver pass (weights, weight cotangent, sender
// features and their cotangent) and for the sender pass (weights, weight
// cotangent, receiver output gradient), this lane's channels.
template <class K>
struct RecvRows {
    float w[K::NP][K::VEC], b[K::NP][K::VEC], x[K::D_IN][K::VEC], a[K::D_IN][K::VEC];
};
template <class K>
struct SendRows {
    float w[K::NP][K::VEC], b[K::NP][K::VEC], g[K::D_OUT][K::VEC];
};

// Receiver pass: g_gy.
template <class K>
__global__ void __launch_bounds__(DblShape<K>::WARPS * 32) eqconv_dbl_recv_kernel(const DblParams prm) {
    constexpr int V = K::VEC, CH = DblShape<K>::CH, W = DblShape<K>::WARPS;
    extern __shared__ __align__(128) float4 smem4[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * W + warp;
    if (node >= prm.N) return;
    float* AY = reinterpret_cast<float*>(smem4) + warp * DblShape<K>::WARP_FLOATS;
    float* AR = AY + CH * K::NA_PAD;
    const int C = prm.C;
    const int c0 = blockIdx.y * K::TILE_C, cl = lane * V;
    const bool on = c0 + cl < C;
    float acc[K::D_OUT][V];
#pragma unroll
    for (int d = 0; d < K::D_OUT; ++d)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[d][v] = 0.f;
    const int kb = prm.ptr[node], ke = prm.ptr[node + 1];
    for (int k0 = kb; k0 < ke; k0 += CH) {
        const int nb = min(CH, ke - k0);
        int my_e = 0, my_s = -1;
        if (lane < nb) {
            my_e = prm.perm[k0 + lane];
            if ((unsigned)my_e < (unsigned)prm.E) my_s = prm.other[my_e];
            if ((unsigned)my_s >= (unsigned)prm.N) {
                atomicOr(prm.status, 1u);
                my_s = -1;
            } else {
                dbl_couplings<K>(prm.r, prm.q, my_e, AY + lane * K::NA_PAD, AR + lane * K::NA_PAD);
            }
        }
        __syncwarp();
        RecvRows<K> cur, nxt;
        const auto load = [&](RecvRows<K>& rw, int t) {
            const int e = __shfl_sync(0xffffffffu, my_e, t);
            const int s = __shfl_sync(0xffffffffu, my_s, t);
            const bool ld = on && s >= 0;
            load_rows<V>(rw.w, prm.w + (size_t)e * K::NP * C + c0 + cl, C, ld);
            load_rows<V>(rw.b, prm.b + (size_t)e * K::NP * C + c0 + cl, C, ld);
            load_rows<V>(rw.x, prm.x + (size_t)max(s, 0) * K::D_IN * C + c0 + cl, C, ld);
            load_rows<V>(rw.a, prm.a + (size_t)max(s, 0) * K::D_IN * C + c0 + cl, C, ld);
        };
        if (DblShape<K>::PF) load(cur, 0);
        for (int t = 0; t < nb; ++t) {
            if (DblShape<K>::PF) {
                if (t + 1 < nb) load(nxt, t + 1);
            } else {
                load(cur, t);
            }
            if (__shfl_sync(0xffffffffu, my_s, t) >= 0)
                dbl_recv_edge<K>(AY + t * K::NA_PAD, AR + t * K::NA_PAD, cur.x, cur.a, cur.w, cur.b, acc);
            if (DblShape<K>::PF) cur = nxt;
        }
        __syncwarp();
    }
    if (on) {
        float* gi = prm.g_gy + (size_t)node * K::D_OUT * C + c0 + cl;
#pragma unroll
        for (int d = 0; d < K::D_OUT; ++d) st_stream<V>(gi + (size_t)d * C, acc[d]);
    }
}

// Sender pass: g_x, g_w and the per-tile partials of gYv, gY1.
template <class K>
__global__ void __launch_bounds__(DblShape<K>::WARPS * 32) eqconv_dbl_send_kernel(const DblParams prm) {
    constexpr int V = K::VEC, CH = DblShape<K>::CH, W = DblShape<K>::WARPS;
    constexpr int G = K::G > 0 ? K::G : 1;
    extern __shared__ __align__(128) float4 smem4[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int node = blockIdx.x * W + warp;
    if (node >= prm.N) return;
    float* AY = reinterpret_cast<float*>(smem4) + warp * DblShape<K>::WARP_FLOATS;   // Y, rho rows
    const int C = prm.C;
    const int tile = blockIdx.y;
    const int c0 = tile * K::TILE_C, cl = lane * V;
    const bool on = c0 + cl < C;
    float xv[K::D_IN][V], av[K::D_IN][V], gacc[K::D_IN][V];
    load_rows<V>(xv, prm.x + (size_t)node * K::D_IN * C + c0 + cl, C, on);
    load_rows<V>(av, prm.a + (size_t)node * K::D_IN * C + c0 + cl, C, on);
#pragma unroll
    for (int d = 0; d < K::D_IN; ++d)
#pragma unroll
        for (int v = 0; v < V; ++v) gacc[d][v] = 0.f;
    const int kb = prm.ptr[node], ke = prm.ptr[node + 1];
    for (int k0 = kb; k0 < ke; k0 += CH) {
        const int nb = min(CH, ke - k0);
        int my_e = 0, my_i = -1;
        if (lane < nb) {
            my_e = prm.perm[k0 + lane];
            if ((unsigned)my_e < (unsigned)prm.E) my_i = prm.other[my_e];
            if ((unsigned)my_i >= (unsigned)prm.N) {
                atomicOr(prm.status, 1u);
                my_i = -1;
            } else {
                dbl_harmonics<K>(prm.r, prm.q, my_e, AY + lane * 2 * K::D_SH);
            }
        }
        __syncwarp();
        SendRows<K> cur, nxt;
        const auto load = [&](SendRows<K>& rw, int t) {
            const int e = __shfl_sync(0xffffffffu, my_e, t);
            const int i = __shfl_sync(0xffffffffu, my_i, t);
            const bool ld = on && i >= 0;
            load_rows<V>(rw.w, prm.w + (size_t)e * K::NP * C + c0 + cl, C, ld);
            load_rows<V>(rw.b, prm.b + (size_t)e * K::NP * C + c0 + cl, C, ld);
            load_rows<V>(rw.g, prm.gy + (size_t)max(i, 0) * K::D_OUT * C + c0 + cl, C, ld);
        };
        if (DblShape<K>::PF) load(cur, 0);
        for (int t = 0; t < nb; ++t) {
            if (DblShape<K>::PF) {
                if (t + 1 < nb) load(nxt, t + 1);
            } else {
                load(cur, t);
            }
            const int e = __shfl_sync(0xffffffffu, my_e, t);
            const int i = __shfl_sync(0xffffffffu, my_i, t);
            if (i < 0) {
                if (DblShape<K>::PF) cur = nxt;
                continue;
            }
            float gYv[G], gY1[G];
#pragma unroll
            for (int k = 0; k < G; ++k) gYv[k] = gY1[k] = 0.f;
            dbl_send_edge<K>(AY + t * 2 * K::D_SH, xv, av, cur.g, cur.w, cur.b, gacc,
                             prm.g_w + (size_t)e * K::NP * C + c0 + cl, C, on, gYv, gY1);
            if (DblShape<K>::PF) cur = nxt;
            if constexpr (K::G > 0) {
                warp_sum<G>(gYv);
                warp_sum<G>(gY1);
                if (lane == 0) {
                    float* pp = prm.part + ((size_t)e * prm.T + tile) * 2 * G;
#pragma unroll
                    for (int k = 0; k < G; ++k) {
                        pp[k] = gYv[k];
                        pp[G + k] = gY1[k];
                    }
                }
            }
        }
        __syncwarp();
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

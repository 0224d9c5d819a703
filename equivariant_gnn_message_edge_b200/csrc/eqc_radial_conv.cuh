// The convolution with its radial weights produced on the chip (sm_100a):
// w[e, p, c] never exists in global memory.
//
//   y[i, l3 m3, c] = sum_{e -> i} sum_p w[e, p, c] sum_{m1, m2} C_p[m1, m2, m3] x[s(e), l1 m1, c] Y_{l2 m2}(r_e)
//   w[e, p, c]     = u(|r_e|) * (h2(|r_e|) . W3)[p*C + c]                     (eqc_radial.cuh)
//
// (e3j, arXiv 2609.35099, abstract and Table 3: the MACE convolution with 8
// Bessel radial functions; FlashCart, arXiv 2610.06409, §4 / App. D for the
// receiver-sorted scheme and App. B / App. E for the radial envelope.)
//
// One CTA takes a range of receivers (their in-edges are consecutive
// positions of the receiver CSR), one slice of 32 channels and a group of up
// to 4 paths.  Its 192 threads are 6 warps with fixed roles (two CTAs share
// an SM; grouping 4 paths per CTA keeps the distinct per-path code an SM runs
// small and lets a light path's CTA finish early instead of waiting on the
// heaviest path of a larger group):
//   * warp 4 (one thread): stages the group's W3^T rows (one tile of 4
//     paths x 32 channels, fp16 hi/lo, resident for the whole CTA) and the
//     h2 tiles of 64 positions (TMA, 2 stages), and issues the MMAs
//       D[(path, channel), edge] = W3^T . h2^T      (M = 128, N = 64, K = 64)
//     into one of two tensor-memory buffers (64 columns each);
//   * warp 5: copies the sender rows x[s, :, slice] of each batch of 8
//     positions into a ring of shared-memory slots (TMA, one box of
//     D_in x 32 floats per position) and publishes each position's
//     harmonics, edge factor and receiver beside them;
//   * warps 0..3 (the path warps): warp w owns path p = 4 g + w.  Its lanes
//     are the slice's 32 channels, and tensor-memory lanes 32 w .. +31 hold
//     exactly that path's 32 channels, so each lane reads its own
//     w[e, p, c] with tcgen05.ld.  Per batch it forms the path's coupling
//     A_p = C_p . Y(r_e) (lane t for position t, into shared memory), and per
//     edge accumulates
//       acc[m3] += w * sum_m1 A_p[m3][m1] x[m1]
//     for the current receiver, writing the path's output block of a
//     receiver when its edges end.
// Outputs are per-path blocks (every path its own 2 l3 + 1 rows); a plan
// that sums paths by output irrep adds the blocks afterwards in path order
// (radial_sum_paths_kernel), so the result is deterministic.
#pragma once

#include "eqc_radial.cuh"

namespace eqc {
namespace radial {

constexpr int kSlice = 32;         // channels per CTA: one per lane of a path warp
constexpr int kGroupPaths = 4;     // paths per CTA: one MMA tile of 4 paths x 32 channels
constexpr int kGroupTiles = 1;
constexpr int kPathWarps = 4;
constexpr int kMmaWarp = 4, kXWarp = 5;
constexpr int kConvThreads = 6 * 32;
constexpr int kXBatches = 2;       // sender-row batches in flight (double buffer)
constexpr int kTmemCols = 128;     // 2 buffers x 1 tile x 64 columns (several CTAs share an SM)

struct RadFwdParams {
    const float* x;      // [N][D_in][C]
    const int* ptr;      // recv_ptr [N+1]
    const float4* rec;   // [E] (r_e, uscale) by receiver position
    const int2* ids;     // [E] (sender, receiver) by receiver position
    float* y_pp;         // [N][D_pp][C] per-path output blocks
    int N, C, E;
    int nodes_per_cta;
    unsigned* status;
};

template <class K>
constexpr int max_coupling_floats() {
    int m = 4;
    for (int p = 0; p < K::NP; ++p) {
        const int sz = ((2 * K::PL.l1[p] + 1) * (2 * K::PL.l3[p] + 1) + 3) & ~3;
        if (sz > m) m = sz;
    }
    return m;
}

// Shared-memory layout of the fused forward (bytes; tiles 1024-aligned).
template <class K>
struct RadFwdSmem {
    static constexpr int BT = 8;                                            // positions per batch
    static constexpr int A_TILE = kRowTile * kTileRowBytes;                 // 16 KB: 128 rows of W3^T
    static constexpr int H_TILE = kEdgeTile * kTileRowBytes;                // 8 KB: 64 rows of h2
    static constexpr int W3_OFF = 0;                                        // [tile][hi, lo]
    static constexpr int H_OFF = W3_OFF + kGroupTiles * 2 * A_TILE;         // [stage][hi, lo]
    static constexpr int X_SLOT = K::D_IN * kSlice * 4;
    static constexpr int X_OFF = H_OFF + 2 * 2 * H_TILE;                    // [batch buffer][BT slots]
    static constexpr int NA = max_coupling_floats<K>();
    static constexpr int CPL_OFF = X_OFF + kXBatches * BT * X_SLOT;
    static constexpr int CPL_WARP = BT * NA * 4;
    static constexpr int WS_OFF = CPL_OFF + kPathWarps * CPL_WARP;          // per path warp: w of the batch
    static constexpr int WS_WARP = BT * 32 * 4;
    // per batch buffer, written by the sender-row warp: each position's harmonics
    // (rows of YS floats), edge factor and receiver
    static constexpr int YS = (K::D_SH + 3) & ~3;
    static constexpr int YB_OFF = WS_OFF + kPathWarps * WS_WARP;
    static constexpr int YB_BATCH = BT * (YS + 4) * 4;                      // Y row + (us, own) per position
    static constexpr int BAR_OFF = YB_OFF + kXBatches * YB_BATCH;
    // barriers: w3, h_full[2], h_empty[2], t_full[2], t_empty[2], x_full[2], x_empty[2]
    static constexpr int NBAR = 9 + 2 * kXBatches;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int END = MISC_OFF + 16;
    static constexpr int BYTES = END + 1024;                               // + alignment slack
    static_assert(BYTES <= 227 * 1024, "fused radial forward: shared memory");
    static_assert(kEdgeTile % BT == 0, "batches tile the MMA tile");
};

// Per-edge coupling of one path: Arow[m3 * d1 + m1] = sum_m2 C_p[m1,m2,m3] Y[l2^2 + m2].
template <int L1, int L2, int L3>
__device__ __forceinline__ void path_coupling(const float* Y, float* Arow) {
    constexpr int d1 = 2 * L1 + 1, d2 = 2 * L2 + 1, d3 = 2 * L3 + 1, o2 = L2 * L2;
    constexpr int n4 = (d1 * d3 + 3) / 4;
    float a[n4 * 4];
#pragma unroll
    for (int q = d1 * d3; q < n4 * 4; ++q) a[q] = 0.f;
    static_for<d3>([&](auto m3c) {
        static_for<d1>([&](auto m1c) {
            constexpr int m1 = EQC_CV(m1c), m3 = EQC_CV(m3c);
            float s = 0.f;
            static_for<d2>([&](auto m2c) {
                constexpr int m2 = EQC_CV(m2c);
                constexpr double c = RealCG<L1, L2, L3>::t.v[m1][m2][m3];
                if constexpr (c != 0.0) s = fmaf((float)c, Y[o2 + m2], s);
            });
            a[m3 * d1 + m1] = s;
        });
    });
#pragma unroll
    for (int q = 0; q < n4; ++q)
        reinterpret_cast<float4*>(Arow)[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
}

__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    uint32_t v;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v) : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(v) : : "memory");
    return __uint_as_float(v);
}

// BT consecutive columns of this warp's lanes into `dst` [BT][32] (shared).
template <int BT>
__device__ __forceinline__ void tmem_stash(uint32_t taddr, float* dst, int lane) {
    if constexpr (BT == 16) {
        float v[16];
        tmem_ld16(taddr, v);
#pragma unroll
        for (int t = 0; t < 16; ++t) dst[t * 32 + lane] = v[t];
    } else if constexpr (BT == 8) {
        float v[8];
        tmem_ld8(taddr, v);
#pragma unroll
        for (int t = 0; t < 8; ++t) dst[t * 32 + lane] = v[t];
    } else if constexpr (BT == 4) {
        float v[4];
        tmem_ld4(taddr, v);
#pragma unroll
        for (int t = 0; t < 4; ++t) dst[t * 32 + lane] = v[t];
    } else {
#pragma unroll
        for (int t = 0; t < BT; ++t) dst[t * 32 + lane] = tmem_ld1(taddr + (uint32_t)t);
    }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// The path warp's whole run for path P_ (compile-time), over the CTA's
// positions [k0, k1) and receivers [n0, n1), batch by batch: one wait for
// the batch's sender rows, one tensor-memory read of its w, per-edge
// records read in position order (prefetched one batch ahead).
template <class K, int P_>
__device__ __forceinline__ void path_warp_fwd(const RadFwdParams& prm, uint8_t* base, uint32_t tmem, int warp,
                                              int lane, int n0, int n1, int k0, int k1, int c0,
                                              volatile int* abort_flag) {
    using S = RadFwdSmem<K>;
    constexpr int BT = S::BT;
    constexpr int l1 = K::PL.l1[P_], l2 = K::PL.l2[P_], l3 = K::PL.l3[P_];
    constexpr int d1 = 2 * l1 + 1, d3 = 2 * l3 + 1, o1 = l1 * l1, o3 = K::PL.o3[P_];
    constexpr int NA = S::NA;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::BAR_OFF);
    uint64_t* t_full = bars + 5;
    uint64_t* t_empty = bars + 7;
    uint64_t* x_full = bars + 9;
    uint64_t* x_empty = bars + 9 + kXBatches;
    float* cpl = reinterpret_cast<float*>(base + S::CPL_OFF + warp * S::CPL_WARP);
    float* ws = reinterpret_cast<float*>(base + S::WS_OFF + warp * S::WS_WARP);
    const float* xring = reinterpret_cast<const float*>(base + S::X_OFF);
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tile_col = (uint32_t)(64 * (warp >> 2));
    const int C = prm.C;

    float acc[d3];
#pragma unroll
    for (int m = 0; m < d3; ++m) acc[m] = 0.f;
    int cur = n0;
    auto flush = [&]() {   // the current receiver's block, then reset
        float* yo = prm.y_pp + ((size_t)cur * K::D_OUT + o3) * C + c0 + lane;
#pragma unroll
        for (int m = 0; m < d3; ++m) {
            __stcs(yo + (size_t)m * C, acc[m]);
            acc[m] = 0.f;
        }
    };

    const int ntiles = (k1 - k0 + kEdgeTile - 1) / kEdgeTile;
    for (int j = 0; j < ntiles; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&t_full[s], (uint32_t)(j >> 1) & 1u) || __any_sync(0xffffffffu, *abort_flag)) {
            if (lane == 0) atomicOr(prm.status, 4u);
            *abort_flag = 1;
            return;
        }
        tc_fence_after();
        const uint32_t tcol = tmem + lane_base + (uint32_t)(s * kGroupTiles * kEdgeTile) + tile_col;
        const int kt = k0 + j * kEdgeTile;
        const int kt_end = min(k1, kt + kEdgeTile);
        for (int kb = kt; kb < kt_end; kb += BT) {
            const int nb = min(BT, kt_end - kb);
            const int b = (kb - k0) / BT;
            tmem_stash<BT>(tcol + (uint32_t)(kb - kt), ws, lane);
            // the batch's sender rows, harmonics, edge factors and receivers
            if (!mbar_wait(&x_full[b % kXBatches], (uint32_t)(b / kXBatches) & 1u) ||
                __any_sync(0xffffffffu, *abort_flag)) {
                if (lane == 0) atomicOr(prm.status, 4u);
                *abort_flag = 1;
                return;
            }
            const float* yb = reinterpret_cast<const float*>(base + S::YB_OFF + (b % kXBatches) * S::YB_BATCH);
            if constexpr (l2 > 0) {
                if (lane < nb) path_coupling<l1, l2, l3>(yb + lane * (S::YS + 4), cpl + lane * NA);
                __syncwarp();
            }
            const float* xb = xring + (b % kXBatches) * BT * (S::X_SLOT / 4) + o1 * kSlice + lane;
            for (int t = 0; t < nb; ++t) {
                const float* yt = yb + t * (S::YS + 4);
                const int own_t = __float_as_int(yt[S::YS + 1]);
                while (cur < own_t) {   // receivers done (and any without edges)
                    flush();
                    ++cur;
                }
                const float w = ws[t * 32 + lane] * yt[S::YS];
                const float* xs = xb + t * (S::X_SLOT / 4);
                float xv[d1];
#pragma unroll
                for (int m = 0; m < d1; ++m) xv[m] = xs[m * kSlice];
                if constexpr (l2 == 0) {
#pragma unroll
                    for (int m = 0; m < d1; ++m) acc[m] = fmaf(w, xv[m], acc[m]);
                } else {
                    const float* A = cpl + t * NA;
#pragma unroll
                    for (int m3 = 0; m3 < d3; ++m3) {
                        float u = 0.f;
#pragma unroll
                        for (int m1 = 0; m1 < d1; ++m1) u = fmaf(A[m3 * d1 + m1], xv[m1], u);
                        acc[m3] = fmaf(w, u, acc[m3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&x_empty[b % kXBatches]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_empty[s]);
    }
    while (cur < n1) {   // the last receiver and any empty ones after it
        flush();
        ++cur;
    }
}

template <class K>
__global__ void __launch_bounds__(kConvThreads, 2)
    radial_conv_fwd_kernel(const RadFwdParams prm, const __grid_constant__ CUtensorMap map_a_hi,
                           const __grid_constant__ CUtensorMap map_a_lo, const __grid_constant__ CUtensorMap map_h_hi,
                           const __grid_constant__ CUtensorMap map_h_lo, const __grid_constant__ CUtensorMap map_x) {
    using S = RadFwdSmem<K>;
    constexpr int BT = S::BT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::BAR_OFF);
    uint64_t* w3_full = bars;
    uint64_t* h_full = bars + 1;
    uint64_t* h_empty = bars + 3;
    uint64_t* t_full = bars + 5;
    uint64_t* t_empty = bars + 7;
    uint64_t* x_full = bars + 9;
    uint64_t* x_empty = bars + 9 + kXBatches;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + S::MISC_OFF + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int n0 = blockIdx.x * prm.nodes_per_cta;
    const int n1 = min(prm.N, n0 + prm.nodes_per_cta);
    const int c0 = blockIdx.y * kSlice;
    const int g0 = blockIdx.z * kGroupPaths;                       // first path of the group
    const int gp = min(kGroupPaths, K::NP - g0);                   // paths in the group
    const int gtiles = (gp + 3) / 4;
    const int k0 = prm.ptr[n0], k1 = prm.ptr[n1];
    const int ntiles = (k1 - k0 + kEdgeTile - 1) / kEdgeTile;

    if (tid == 0) {
        mbar_init(w3_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&h_full[s], 1);
            mbar_init(&h_empty[s], 1);
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], gp);
        }
        for (int q = 0; q < kXBatches; ++q) {
            mbar_init(&x_full[q], 2);   // the copies' bytes + the batch info
            mbar_init(&x_empty[q], gp);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kPathWarps) {
        const int p = g0 + warp;
        if (warp < gp) {
            static_for<K::NP>([&](auto pc) {
                if (EQC_CV(pc) == p)
                    path_warp_fwd<K, EQC_CV(pc)>(prm, base, tmem, warp, lane, n0, n1, k0, k1, c0, abort_flag);
            });
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0 && ntiles > 0) {
            // the group's W3^T rows: tile t, quarter q = path g0 + 4 t + q, channels [c0, c0 + 32)
            mbar_expect_tx(w3_full, gtiles * 2 * S::A_TILE);
            for (int t = 0; t < gtiles; ++t)
                for (int q = 0; q < 4; ++q) {
                    const int row = (g0 + 4 * t + q) * prm.C + c0;   // past P * C: zero fill
                    uint8_t* dst = base + S::W3_OFF + t * 2 * S::A_TILE + q * 32 * kTileRowBytes;
                    tma_2d(dst, &map_a_hi, 0, row, w3_full);
                    tma_2d(dst + S::A_TILE, &map_a_lo, 0, row, w3_full);
                }
            int h_issued = 0, h_waited = 0, committed = 0;
            auto load_h = [&](int j) {
                const int s = j & 1;
                uint8_t* dst = base + S::H_OFF + s * 2 * S::H_TILE;
                mbar_expect_tx(&h_full[s], 2 * S::H_TILE);
                tma_2d(dst, &map_h_hi, 0, k0 + j * kEdgeTile, &h_full[s]);
                tma_2d(dst + S::H_TILE, &map_h_lo, 0, k0 + j * kEdgeTile, &h_full[s]);
                h_issued = j + 1;
            };
            load_h(0);
            if (ntiles > 1) load_h(1);
            const bool w3_ok = mbar_wait_one(w3_full, 0);
            bool ok = w3_ok;
            constexpr uint32_t id = idesc_f16(kRowTile, kEdgeTile);
            for (int j = 0; j < ntiles && ok; ++j) {
                const int s = j & 1;
                ok = mbar_wait_one(&h_full[s], (uint32_t)(j >> 1) & 1u);
                if (!ok) break;
                h_waited = j + 1;
                ok = (j < 2 || mbar_wait_one(&t_empty[s], (uint32_t)((j >> 1) - 1) & 1u)) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                const uint8_t* hs = base + S::H_OFF + s * 2 * S::H_TILE;
                const uint64_t dbh = sw128_desc(smem_addr(hs)), dbl = sw128_desc(smem_addr(hs + S::H_TILE));
                for (int t = 0; t < gtiles; ++t) {
                    const uint8_t* at = base + S::W3_OFF + t * 2 * S::A_TILE;
                    const uint64_t dah = sw128_desc(smem_addr(at)), dal = sw128_desc(smem_addr(at + S::A_TILE));
                    const uint32_t d = tmem + (uint32_t)(s * kGroupTiles * kEdgeTile + t * kEdgeTile);
#pragma unroll
                    for (int kk = 0; kk < kH / 16; ++kk) {
                        const uint64_t adv = (uint64_t)(kk * 32) >> 4;
                        umma_f16(d, dah + adv, dbh + adv, id, kk > 0);
                        umma_f16(d, dah + adv, dbl + adv, id, 1);
                        umma_f16(d, dal + adv, dbh + adv, id, 1);
                    }
                }
                umma_commit(&t_full[s]);
                umma_commit(&h_empty[s]);
                committed = j + 1;
                if (j + 2 < ntiles) {
                    ok = mbar_wait_one(&h_empty[s], (uint32_t)(j >> 1) & 1u);
                    if (ok) load_h(j + 2);
                }
            }
            if (!ok) {
                atomicOr(prm.status, 4u);
                *abort_flag = 1;
                // let the copies and products in flight land before the CTA lets go of its memory
                if (!w3_ok) mbar_wait_one(w3_full, 0);
                for (int u = h_waited; u < h_issued; ++u) mbar_wait_one(&h_full[u & 1], (uint32_t)(u >> 1) & 1u);
                for (int u = committed > 2 ? committed - 2 : 0; u < committed; ++u)
                    mbar_wait_one(&t_full[u & 1], (uint32_t)(u >> 1) & 1u);
            }
        }
    } else if (warp == kXWarp) {
        // sender rows, batch by batch: one barrier per batch of BT positions;
        // lane t copies the row of position kb + t
        const int nbatch = (k1 - k0 + BT - 1) / BT;
        int issued = 0;
        for (int b = 0; b < nbatch; ++b) {
            const int kb = k0 + b * BT;
            const int nb = min(BT, k1 - kb);
            int sidx = 0, own = 0;
            float4 rc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane < nb) {
                const int2 id = prm.ids[kb + lane];
                rc = prm.rec[kb + lane];
                sidx = id.x;
                own = id.y;
                if ((unsigned)sidx >= (unsigned)prm.N) {   // out of range: flagged, read as node 0
                    atomicOr(prm.status, 1u);
                    sidx = 0;
                }
            }
            int go = 1;
            if (lane == 0) {
                if (b >= kXBatches &&
                    !mbar_wait_one(&x_empty[b % kXBatches], (uint32_t)(b / kXBatches - 1) & 1u)) {
                    atomicOr(prm.status, 4u);
                    *abort_flag = 1;
                }
                go = *abort_flag ? 0 : 1;
                if (go) mbar_expect_tx(&x_full[b % kXBatches], nb * S::X_SLOT);
            }
            if (!__shfl_sync(0xffffffffu, go, 0)) break;
            if (lane < nb)
                tma_rows(base + S::X_OFF + ((b % kXBatches) * BT + lane) * S::X_SLOT, &map_x, c0, sidx,
                         &x_full[b % kXBatches], policy_evict_last());
            issued = b + 1;
            // each position's harmonics, edge factor and receiver for the path warps
            if (lane < nb) {
                float* yrow = reinterpret_cast<float*>(base + S::YB_OFF + (b % kXBatches) * S::YB_BATCH) +
                              lane * (S::YS + 4);
                float ux, uy, uz, il;
                const bool okd = unit_dir(rc.x, rc.y, rc.z, ux, uy, uz, il);
                float Y[K::D_SH];
                sh_eval<K::LSH>(okd, ux, uy, uz, Y);
#pragma unroll
                for (int q = 0; q < K::D_SH; ++q) yrow[q] = Y[q];
                yrow[S::YS] = rc.w;
                yrow[S::YS + 1] = __int_as_float(own);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&x_full[b % kXBatches]);
        }
        // the last fills of each buffer land before the CTA lets go of its memory
        // (immediate when their consumers already saw them)
        if (lane == 0)
            for (int b = issued > kXBatches ? issued - kXBatches : 0; b < issued; ++b)
                mbar_wait_one(&x_full[b % kXBatches], (uint32_t)(b / kXBatches) & 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// y[i, l3^2 + m, c] = sum over paths p with that l3, in path order, of
// y_pp[i, o3pp(p) + m, c]  (KS: the summed plan's Cfg; KP: its per-path Cfg).
template <class KS, class KP>
__global__ void radial_sum_paths_kernel(const float* __restrict__ y_pp, float* __restrict__ y, int N, int C) {
    const int c4 = C / 4;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)N * KS::D_OUT * c4;
    if (idx >= total) return;
    const int cq = (int)(idx % c4);
    const int row = (int)((idx / c4) % KS::D_OUT);
    const int i = (int)(idx / ((int64_t)c4 * KS::D_OUT));
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    static_for<KP::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l3 = KP::PL.l3[p];
        if (row >= l3 * l3 && row < (l3 + 1) * (l3 + 1)) {
            const float4 v = __ldcs(reinterpret_cast<const float4*>(
                y_pp + ((size_t)i * KP::D_OUT + KP::PL.o3[p] + (row - l3 * l3)) * C) + cq);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
    });
    __stcs(reinterpret_cast<float4*>(y + ((size_t)i * KS::D_OUT + row) * C) + cq, s);
}

}  // namespace radial
}  // namespace eqc

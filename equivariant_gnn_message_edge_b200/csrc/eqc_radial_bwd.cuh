// Backward of the convolution with on-chip radial weights (sm_100a): dx, the
// MLP weight gradients and dr through both routes of r, with w and dw never
// in global memory.
//
// With w = u(d) z3, z3 = h2 . W3, and dw the weight gradient of the
// convolution's VJP (FlashCart, arXiv 2610.06409, §4 / App. D: a
// sender-ordered pass sums each sender's input gradient deterministically):
//   g_W3[k, pc] = sum_e h2[e, k] u dw[e, pc]                   (tensor cores)
//   g_h2[e, k]  = sum_pc W3[k, pc] u dw[e, pc]                 (tensor cores)
//   g_u[e]      = sum_pc dw[e, pc] z3[e, pc]                   (lane sums)
//   then the small MLP backward per edge
//   dr_e = (dY/dr)^T gY[e] + g_d(|r_e|) r_e / |r_e|
// (FlashCart §2: forces are the energy's gradient in the positions, so both
// routes of r count).
//
// radial_conv_bwd_kernel: one CTA per sender range x 32-channel slice x
// group of up to 4 paths (one MMA tile of 4 paths x 32 channels); two CTAs
// share an SM where their shared memory allows.  Warps:
//   * 0..3 (path warps): warp w owns path 4 g + w, its lanes the 32 channels
//     and tensor-memory subpartition w.  For every out-edge of the current
//     sender (positions of the sender CSR) it reads w from tensor memory,
//     the receiver's gy rows from the ring, the edge's harmonics, and with
//     h[m1][m2] = sum_m3 C_p gy[m3]:
//       t[m1] = sum_m2 Y[m2] h,  dw = x . t,  dx += w t,
//       gY[m2] += w sum_m1 x[m1] h      (summed over the 32 lanes)
//     u dw goes, scaled and split into fp16 halves, into the G tile
//     [(path, channel) rows][64 edges] in shared memory.  Each also copies
//     its subpartition's rows of Gd per tile and its path's g_W3 rows at the
//     end out of tensor memory (a warp without a path copies only Gd);
//   * 4 (one thread): stages W3^T and h2 tiles with TMA and issues the
//     MMAs: w = W3^T . h2^T, then per tile g_W3 += G . h2 and Gd = W3 . G
//     (K over the tile's edges / the group's rows), G the tile of u dw;
//   * 5: copies each batch's receiver rows gy[i, :, slice] (one lane per
//     position).
// Per-path dx blocks, per-edge gY partials, Gd partials and g_W3 partials go
// to the workspace; radial_bwd_epilogue_kernel and the reductions finish dr,
// dx and the weight gradients in a fixed order (deterministic).
//
// Scaling of u dw for fp16: G = u dw 2^sG 2^-sB(e) (sB(e) the power of two of
// the edge's h2), with sG chosen from a bound of |dw| (49 max|x| max|gy|:
// |dw| <= |x_l1| |A_p| |gy_l3| and |A_p|_F <= sqrt((2 l2 + 1)(2 l3 + 1))) and
// of |h2| so that |G| < 2^14; the per-edge powers of two cancel against those
// of h2 in g_W3.  g_u = sum_pc dw z3 is summed over the lanes with the
// harmonic gradient, from z3 in tensor memory, so it needs no division by u.
#pragma once

#include "eqc_radial_conv.cuh"

namespace eqc {
namespace radial {

constexpr int kBwdGroupPaths = 4;
constexpr int kBwdGroupTiles = 1;
constexpr int kBwdPathWarps = 4;
constexpr int kBwdMmaWarp = 4, kBwdGyWarp = 5;
constexpr int kBwdThreads = 6 * 32;
constexpr int kBwdTmemCols = 256;   // two CTAs share an SM's tensor memory
constexpr int kGySlots = 16;
constexpr uint32_t kColW = 0;       // w: [2 buffers][1 tile][64]
constexpr uint32_t kColGW = 128;    // g_W3 accumulators: [1 tile][64 (k)]
constexpr uint32_t kColGD = 192;    // Gd: 64 columns (M = 64 layout)

struct RadBwdParams {
    const float* x;        // [N][D_in][C]
    const float* gy;       // [N][D_out][C] (the plan's output layout)
    const int* ptr;        // send_ptr [N+1]
    const float4* rec;     // [E] (r_e, uscale) by sender position
    const int2* ids;       // [E] (receiver, sender) by sender position
    const float* scal;     // [0] 2^-sA; [1..3] bits of max|x|, max|gy|, max|u h2|
    float* dx_pp;          // [N][DX_PP][C] per-path dx blocks
    float* gy_part;        // [E][slices][SD2] per-path harmonic-gradient partials
    float* gd_part;        // [slices * groups][E][64] Gd partials (scaled)
    float* gw3_part;       // [ranges][P * C][64] g_W3 partials (scaled)
    int N, C, E, nodes_per_cta;
    unsigned* status;
};

// per-path dx rows (2 l1 + 1 each, in path order) and per-edge partial
// offsets (1 + (2 l2 + 1 if l2 > 0) per path)
template <class K>
struct BwdRows {
    static constexpr int dx_off(int p) {
        int o = 0;
        for (int q = 0; q < p; ++q) o += 2 * K::PL.l1[q] + 1;
        return o;
    }
    // per path: [sum of dw z3 (for g_u), then the 2 l2 + 1 harmonic-gradient values if l2 > 0]
    static constexpr int gy_off(int p) {
        int o = 0;
        for (int q = 0; q < p; ++q) o += 1 + (K::PL.l2[q] > 0 ? 2 * K::PL.l2[q] + 1 : 0);
        return o;
    }
    static constexpr int DX_PP = dx_off(K::NP);
    static constexpr int SD2 = gy_off(K::NP);
};

__device__ __forceinline__ int inv_pow2_exponent(float v) {   // v = 2^-s -> s
    int e;
    frexpf(v, &e);   // v = 0.5 * 2^e
    return 1 - e;
}

// Exponent g = sG + sA of the G tile: G = dw * 2^g * uscale_e = u dw 2^sG
// 2^-sB(e), with sG from the bounds |dw| <= 49 max|x| max|gy|, u <= 1 and
// 2^-sB(e) <= 2^-13 max|h2|, so that |G| < 2^14.  Computed on the device
// from the maxima (scal[1..3]) and 2^-sA (scal[0]).
__device__ __forceinline__ int g_scale_exponent(const float* scal) {
    const float mx = __uint_as_float(reinterpret_cast<const unsigned*>(scal)[1]);
    const float mg = __uint_as_float(reinterpret_cast<const unsigned*>(scal)[2]);
    const float mh = __uint_as_float(reinterpret_cast<const unsigned*>(scal)[3]);
    const float bound = 49.f * mx * mg * mh;
    int e = 0;
    if (bound > 0.f) frexpf(bound, &e);   // bound < 2^e
    return (27 - e) + inv_pow2_exponent(scal[0]);
}

template <class K>
struct RadBwdSmem {
    static constexpr int A_TILE = kRowTile * kTileRowBytes;               // 16 KB
    static constexpr int H_TILE = kEdgeTile * kTileRowBytes;              // 8 KB
    static constexpr int G_TILE = kRowTile * kEdgeTile * 2;               // 16 KB: 128 rows x 64 edges fp16
    static constexpr int GY_SLOT = K::D_OUT * kSlice * 4;
    static constexpr int YS = (K::D_SH + 3) & ~3;                         // harmonics row (floats)
    // per path warp, for a batch of up to 8 positions: w
    static constexpr int WS_WARP8 = 8 * 32 * 4;
    // per ring position: the gy rows, then the harmonics row, edge factor and sender
    static constexpr int POS_BYTES = GY_SLOT + (YS + 4) * 4;
    // everything but the gy ring, with hs stages of h2
    static constexpr int fixed_for(int hs) {
        return kBwdGroupTiles * 2 * A_TILE + hs * 2 * H_TILE + kBwdGroupTiles * 2 * G_TILE +
               kBwdPathWarps * WS_WARP8 + (14 + 2 * 4) * 8 + 16 + 1024;
    }
    static constexpr bool two_for(int hs) { return (113 * 1024 - fixed_for(hs)) / POS_BYTES >= 8; }
    // Two CTAs share an SM (113 KB each) when a gy ring of two 4-position
    // batches fits beside the rest, else one (227 KB).  Two h2 stages: with
    // one, the next tile's h2 waits for this tile's products (measured slower
    // at lmax3 even with two CTAs per SM).
    static constexpr int HS = 2;
    static constexpr bool TWO = two_for(HS);
    static constexpr int W3_OFF = 0;                                      // [tile][hi, lo]
    static constexpr int H_OFF = W3_OFF + kBwdGroupTiles * 2 * A_TILE;    // [stage][hi, lo]
    static constexpr int G_OFF = H_OFF + HS * 2 * H_TILE;                 // [tile][hi, lo]
    static constexpr int GY_OFF = G_OFF + kBwdGroupTiles * 2 * G_TILE;
    // gy ring: batches of BT receiver rows, as many (2 .. 4) as fit beside the
    // rest; BT = 8 where two batches of 8 fit, else 4, else 2
    static constexpr int FIXED = fixed_for(HS);
    static constexpr int FIT = ((TWO ? 113 : 227) * 1024 - FIXED) / POS_BYTES;
    static constexpr int BT = FIT >= 16 ? 8 : (FIT >= 8 ? 4 : 2);
    static constexpr int GYB = FIT / BT >= 4 ? 4 : FIT / BT;
    // per gy batch buffer, written by the gy warp: each position's harmonics
    // (rows of YS floats), edge factor and sender
    static constexpr int YB_BATCH = BT * (YS + 4) * 4;
    static constexpr int WS_WARP = BT * 32 * 4;
    static constexpr int Y_OFF = GY_OFF + GYB * BT * GY_SLOT;
    static constexpr int WS_OFF = Y_OFF + GYB * YB_BATCH;
    static constexpr int BAR_OFF = WS_OFF + kBwdPathWarps * WS_WARP;
    // w3, h_full[2], h_empty[2], t_full[2], t_empty[2], g_full, g_empty, gd_full, gd_empty, gw_full,
    // gy_full[GYB], gy_empty[GYB]
    static constexpr int NBAR = 14 + 2 * GYB;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int END = MISC_OFF + 16;
    static constexpr int BYTES = END + 1024;
    static_assert(GYB >= 2, "fused radial backward: room for two gy batches");
    static_assert(BYTES <= (TWO ? 113 : 227) * 1024, "fused radial backward: shared memory");
    static_assert(kEdgeTile % BT == 0, "batches tile the MMA tile");
};

// One fp16 chunk of 8 edges for G row `row` at edge chunk `q8` of a 128 x 64
// swizzled tile (rows of 128 B, 8-row groups of 1024 B).
__device__ __forceinline__ uint32_t g_chunk_offset(int row, int q8) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((q8 ^ (row & 7)) << 4));
}

// Gd of the tile starting at position kt (tensor-memory lanes 16 q .. +15 of
// subpartition q hold rows k = 16 q + lane of the M = 64 layout) to the
// workspace, positions below k1.
__device__ __noinline__ void copy_gd(const RadBwdParams& prm, uint32_t tmem, int q, int lane, int kt, int k1,
                                        int sg) {
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float* dst = prm.gd_part + ((size_t)sg * prm.E + kt) * kH + 16 * q + lane;
    const int n = k1 - kt;   // positions of the tile below k1
#pragma unroll 1
    for (int c16 = 0; c16 < kEdgeTile; c16 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + kColGD + (uint32_t)c16, v);
        if (lane < 16) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (c16 + i < n) dst[(size_t)(c16 + i) * kH] = v[i];
        }
    }
}

// The CTA's g_W3 rows of path p (row 32 q + lane = channel c0 + lane) out of
// tensor memory, or zeros for a range without edges.
__device__ __noinline__ void copy_gw3(const RadBwdParams& prm, uint32_t tmem, int q, int lane, int p, int NP,
                                         int c0, bool zero) {
    float* dst = prm.gw3_part + ((size_t)blockIdx.x * NP * prm.C + (size_t)p * prm.C + c0 + lane) * kH;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
#pragma unroll 1
    for (int c16 = 0; c16 < kH; c16 += 16) {
        float v[16];
        if (zero) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.f;
        } else {
            tmem_ld16(tmem + lane_base + kColGW + (uint32_t)c16, v);
        }
#pragma unroll
        for (int i = 0; i < 16; i += 4) *reinterpret_cast<float4*>(dst + c16 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
}

template <class K, int P_>
__device__ __forceinline__ void path_warp_bwd(const RadBwdParams& prm, uint8_t* base, uint32_t tmem, int warp,
                                              int lane, int n0, int n1, int k0, int k1, int c0, int slice,
                                              int slices, int sg, int gexp, volatile int* abort_flag) {
    using S = RadBwdSmem<K>;
    using R = BwdRows<K>;
    constexpr int BT = S::BT;
    constexpr int l1 = K::PL.l1[P_], l2 = K::PL.l2[P_], l3 = K::PL.l3[P_];
    constexpr int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
    constexpr int o1 = l1 * l1, o3 = K::PL.o3[P_], o2 = l2 * l2;
    constexpr int oxp = R::dx_off(P_), ogp = R::gy_off(P_);
    constexpr int NVAL = l2 > 0 ? 1 + d2 : 1;                    // partials of one edge
    constexpr int NV = pow2_at_least(NVAL);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::BAR_OFF);
    uint64_t* t_full = bars + 5;
    uint64_t* t_empty = bars + 7;
    uint64_t* g_full = bars + 9;
    uint64_t* g_empty = bars + 10;
    uint64_t* gd_full = bars + 11;
    uint64_t* gd_empty = bars + 12;
    uint64_t* gw_full = bars + 13;
    uint64_t* gy_full = bars + 14;
    uint64_t* gy_empty = bars + 14 + S::GYB;
    float* wst = reinterpret_cast<float*>(base + S::WS_OFF + warp * S::WS_WARP);  // [BT][32]
    const float* gring = reinterpret_cast<const float*>(base + S::GY_OFF);
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int tile = warp >> 2;                    // MMA tile of this path
    const int grow = 32 * (warp & 3) + lane;       // G row (path, channel) inside the tile
    uint8_t* g_hi = base + S::G_OFF + tile * 2 * S::G_TILE;
    uint8_t* g_lo = g_hi + S::G_TILE;
    const float gscale0 = ldexpf(1.f, gexp);       // G / dw = 2^gexp * uscale_e
    const int C = prm.C;
    const size_t cl = (size_t)c0 + lane;
    auto abort_now = [&]() {
        if (lane == 0) atomicOr(prm.status, 4u);
        *abort_flag = 1;
    };

    // x rows of the current sender, and of the next one (prefetched)
    float xv[d1], xn[d1], dxa[d1];
    int cur = n0;
    auto load_x = [&](int node, float (&dst)[d1]) {
        if (node < n1) {
            const float* xs = prm.x + ((size_t)node * K::D_IN + o1) * C + cl;
#pragma unroll
            for (int m = 0; m < d1; ++m) dst[m] = __ldg(xs + (size_t)m * C);
        }
    };
    auto flush = [&]() {
        float* dxo = prm.dx_pp + ((size_t)cur * R::DX_PP + oxp) * C + cl;
#pragma unroll
        for (int m = 0; m < d1; ++m) {
            __stcs(dxo + (size_t)m * C, dxa[m]);
            dxa[m] = 0.f;
        }
    };
    auto next_sender = [&]() {   // cur -> cur + 1, x from the prefetch
        flush();
        ++cur;
#pragma unroll
        for (int m = 0; m < d1; ++m) xv[m] = xn[m];
        load_x(cur + 1, xn);
    };
#pragma unroll
    for (int m = 0; m < d1; ++m) {
        xv[m] = 0.f;
        xn[m] = 0.f;
        dxa[m] = 0.f;
    }
    load_x(cur, xv);
    load_x(cur + 1, xn);

    uint32_t ghi[4] = {0u, 0u, 0u, 0u}, glo[4] = {0u, 0u, 0u, 0u};   // 8 edges of fp16 G values
    // partials of the last edge, summed over the warp one edge later
    float vp[NV];
    int kp = -1;
    auto reduce_store = [&]() {
        const float sum = warp_transpose_sum<NV>(vp, lane);
        constexpr int sh = transpose_sum_shift(NV);
        const int vi = lane >> sh;
        if ((lane & ((1 << sh) - 1)) == 0 && vi < NVAL)
            prm.gy_part[((size_t)kp * slices + slice) * R::SD2 + ogp + vi] = sum;
    };
    const int ntiles = (k1 - k0 + kEdgeTile - 1) / kEdgeTile;
    for (int j = 0; j < ntiles; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&t_full[s], (uint32_t)(j >> 1) & 1u) || __any_sync(0xffffffffu, *abort_flag)) {
            abort_now();
            return;
        }
        tc_fence_after();
        // the G tile of the previous tile has been read by the MMAs; that
        // tile's Gd (same products) goes to the workspace
        if (j > 0) {
            if (!mbar_wait(g_empty, (uint32_t)(j - 1) & 1u)) {
                abort_now();
                return;
            }
            tc_fence_after();
            copy_gd(prm, tmem, warp & 3, lane, k0 + (j - 1) * kEdgeTile, k1, sg);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(gd_empty);
        }
        const uint32_t tcol = tmem + lane_base + kColW + (uint32_t)((s * kBwdGroupTiles + tile) * kEdgeTile);
        const int kt = k0 + j * kEdgeTile;
        const int kt_end = min(k1, kt + kEdgeTile);
        for (int kb = kt; kb < kt + kEdgeTile; kb += BT) {
            const int nb = max(0, min(BT, kt_end - kb));
            const int b = (kb - k0) / BT;
            const float* gb = gring;
            const float* ys = gring;   // the batch's harmonics rows (written by the gy warp)
            if (nb > 0) {
                tmem_stash<BT>(tcol + (uint32_t)(kb - kt), wst, lane);   // z3 * 2^(sA + sB), BT positions
                // the batch's receiver rows, harmonics, edge factors and senders
                if (!mbar_wait(&gy_full[b % S::GYB], (uint32_t)(b / S::GYB) & 1u) ||
                    __any_sync(0xffffffffu, *abort_flag)) {
                    abort_now();
                    return;
                }
                gb = gring + (b % S::GYB) * BT * (S::GY_SLOT / 4) + o3 * kSlice + lane;
                ys = reinterpret_cast<const float*>(base + S::Y_OFF + (b % S::GYB) * S::YB_BATCH);
            }
            for (int t = 0; t < BT; ++t) {
                float gval = 0.f;
                if (t < nb) {
                    const float* yrow = ys + t * (S::YS + 4);
                    const int own_t = __float_as_int(yrow[S::YS + 1]);
                    while (cur < own_t) next_sender();   // the current sender's edges are done (empty ones too)
                    const float us = yrow[S::YS];
                    const float Dv = wst[t * 32 + lane];
                    const float w = Dv * us;
                    const float* gs = gb + t * (S::GY_SLOT / 4);
                    float gv[d3];
#pragma unroll
                    for (int m = 0; m < d3; ++m) gv[m] = gs[m * kSlice];
                    float tv[d1];
                    [[maybe_unused]] float hG[d2];
                    if constexpr (l2 == 0) {
#pragma unroll
                        for (int m = 0; m < d1; ++m) tv[m] = gv[m];
                    } else {
#pragma unroll
                        for (int m = 0; m < d1; ++m) tv[m] = 0.f;
#pragma unroll
                        for (int m = 0; m < d2; ++m) hG[m] = 0.f;
                        static_for<d2>([&](auto m2c) {
                            constexpr int m2 = EQC_CV(m2c);
                            const float y2 = yrow[o2 + m2];
                            static_for<d1>([&](auto m1c) {
                                constexpr int m1 = EQC_CV(m1c);
                                if constexpr (cg_row_nonzero<l1, l2, l3>(m1, m2)) {
                                    float h = 0.f;
                                    static_for<d3>([&](auto m3c) {
                                        constexpr int m3 = EQC_CV(m3c);
                                        constexpr double c = RealCG<l1, l2, l3>::t.v[m1][m2][m3];
                                        if constexpr (c != 0.0) h = fmaf((float)c, gv[m3], h);
                                    });
                                    tv[m1] = fmaf(y2, h, tv[m1]);
                                    hG[m2] = fmaf(xv[m1], h, hG[m2]);
                                }
                            });
                        });
                    }
                    float dw = xv[0] * tv[0];
#pragma unroll
                    for (int m = 1; m < d1; ++m) dw = fmaf(xv[m], tv[m], dw);
#pragma unroll
                    for (int m = 0; m < d1; ++m) dxa[m] = fmaf(w, tv[m], dxa[m]);
                    gval = dw * gscale0 * us;
                    // this path's partials of the edge, summed over the 32 channels:
                    // sum dw z3 (scaled; for g_u) and the harmonic gradient
                    float v[NV];
                    v[0] = dw * Dv;
#pragma unroll
                    for (int q = 1; q < NV; ++q) v[q] = 0.f;
                    if constexpr (l2 > 0) {
#pragma unroll
                        for (int m = 0; m < d2; ++m) v[1 + m] = w * hG[m];
                    }
                    // the previous edge's partials are summed now, so their shuffle
                    // chain overlaps this edge's arithmetic
                    if (kp >= 0) reduce_store();
#pragma unroll
                    for (int q = 0; q < NV; ++q) vp[q] = v[q];
                    kp = kb + t;
                }
                // pack G (zero for edges past the range) and store every 8 edges
                __half gh, gl;
                split_f16(gval, gh, gl);
                const int pos = kb - kt + t;
                const int pr = pos & 7;
                const uint32_t bh = __half_as_ushort(gh), bl = __half_as_ushort(gl);
                // 128-bit shift registers: after 8 edges edge i sits at bits 16 i
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    ghi[q] = __funnelshift_r(ghi[q], ghi[q + 1], 16);
                    glo[q] = __funnelshift_r(glo[q], glo[q + 1], 16);
                }
                ghi[3] = (ghi[3] >> 16) | (bh << 16);
                glo[3] = (glo[3] >> 16) | (bl << 16);
                if (pr == 7) {
                    const uint32_t off = g_chunk_offset(grow, pos >> 3);
                    *reinterpret_cast<uint4*>(g_hi + off) = make_uint4(ghi[0], ghi[1], ghi[2], ghi[3]);
                    *reinterpret_cast<uint4*>(g_lo + off) = make_uint4(glo[0], glo[1], glo[2], glo[3]);
                }
            }
            __syncwarp();
            if (nb > 0 && lane == 0) mbar_arrive(&gy_empty[b % S::GYB]);
        }
        // G written (generic proxy) -> visible to the tensor cores (async proxy)
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(g_full);
            mbar_arrive(&t_empty[s]);
        }
    }
    if (kp >= 0) reduce_store();
    // the last tile's Gd, then the CTA's g_W3 rows of this path
    if (ntiles > 0) {
        if (!mbar_wait(gd_full, (uint32_t)(ntiles - 1) & 1u) || !mbar_wait(gw_full, 0u)) {
            abort_now();
            return;
        }
        tc_fence_after();
        copy_gd(prm, tmem, warp & 3, lane, k0 + (ntiles - 1) * kEdgeTile, k1, sg);
        copy_gw3(prm, tmem, warp & 3, lane, P_, K::NP, c0, false);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(gd_empty);
    } else {
        copy_gw3(prm, tmem, warp & 3, lane, P_, K::NP, c0, true);
    }
    // the last sender and any empty ones after it
    while (cur + 1 < n1) next_sender();
    flush();
}

template <class K>
__global__ void __launch_bounds__(kBwdThreads, 2)
    radial_conv_bwd_kernel(const RadBwdParams prm, const __grid_constant__ CUtensorMap map_a_hi,
                           const __grid_constant__ CUtensorMap map_a_lo, const __grid_constant__ CUtensorMap map_h_hi,
                           const __grid_constant__ CUtensorMap map_h_lo, const __grid_constant__ CUtensorMap map_gy) {
    using S = RadBwdSmem<K>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::BAR_OFF);
    uint64_t* w3_full = bars;
    uint64_t* h_full = bars + 1;
    uint64_t* h_empty = bars + 3;
    uint64_t* t_full = bars + 5;
    uint64_t* t_empty = bars + 7;
    uint64_t* g_full = bars + 9;
    uint64_t* g_empty = bars + 10;
    uint64_t* gd_full = bars + 11;
    uint64_t* gd_empty = bars + 12;
    uint64_t* gw_full = bars + 13;
    uint64_t* gy_full = bars + 14;
    uint64_t* gy_empty = bars + 14 + S::GYB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base + S::MISC_OFF + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int n0 = blockIdx.x * prm.nodes_per_cta;
    const int n1 = min(prm.N, n0 + prm.nodes_per_cta);
    const int slice = blockIdx.y, slices = gridDim.y;
    const int c0 = slice * kSlice;
    const int g0 = blockIdx.z * kBwdGroupPaths;
    const int gp = min(kBwdGroupPaths, K::NP - g0);
    const int gtiles = (gp + 3) / 4;
    const int k0 = prm.ptr[n0], k1 = prm.ptr[n1];
    const int ntiles = (k1 - k0 + kEdgeTile - 1) / kEdgeTile;
    const int sg = blockIdx.z * slices + slice;     // this CTA's (slice, group) partial index
    const int gexp = g_scale_exponent(prm.scal);

    if (tid == 0) {
        mbar_init(w3_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&h_full[s], 1);
            mbar_init(&h_empty[s], 1);
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], gp);
        }
        mbar_init(g_full, gp);
        mbar_init(g_empty, 1);
        mbar_init(gd_full, 1);
        mbar_init(gd_empty, 4);
        mbar_init(gw_full, 1);
        for (int q = 0; q < S::GYB; ++q) {
            mbar_init(&gy_full[q], 2);   // the copies' bytes + the batch info
            mbar_init(&gy_empty[q], gp);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    // G rows of absent paths (gp < 8) and of a missing second tile stay zero
    for (int i = tid; i < kBwdGroupTiles * 2 * S::G_TILE / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(base + S::G_OFF)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
    if (warp == 0) tmem_alloc(tmem_slot, kBwdTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kBwdPathWarps) {
        const int p = g0 + warp;
        if (warp < gp) {
            static_for<K::NP>([&](auto pc) {
                if (EQC_CV(pc) == p)
                    path_warp_bwd<K, EQC_CV(pc)>(prm, base, tmem, warp, lane, n0, n1, k0, k1, c0, slice, slices,
                                                 sg, gexp, abort_flag);
            });
        } else {
            // a subpartition without a path still copies its rows of every tile's Gd
            for (int j = 0; j < ntiles; ++j) {
                if (!mbar_wait(gd_full, (uint32_t)j & 1u) || __any_sync(0xffffffffu, *abort_flag)) {
                    if (lane == 0) atomicOr(prm.status, 4u);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                copy_gd(prm, tmem, warp & 3, lane, k0 + j * kEdgeTile, k1, sg);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(gd_empty);
            }
        }
    } else if (warp == kBwdMmaWarp) {
        if (lane == 0 && ntiles > 0) {
            mbar_expect_tx(w3_full, gtiles * 2 * S::A_TILE);
            for (int t = 0; t < gtiles; ++t)
                for (int q = 0; q < 4; ++q) {
                    const int row = (g0 + 4 * t + q) * prm.C + c0;
                    uint8_t* dst = base + S::W3_OFF + t * 2 * S::A_TILE + q * 32 * kTileRowBytes;
                    tma_2d(dst, &map_a_hi, 0, row, w3_full);
                    tma_2d(dst + S::A_TILE, &map_a_lo, 0, row, w3_full);
                }
            int h_issued = 0, h_waited = 0, committed = 0, g_done = 0;
            // h2 tile j sits in stage j % HS, phase (j / HS) & 1
            auto load_h = [&](int j) {
                const int hs = j % S::HS;
                uint8_t* dst = base + S::H_OFF + hs * 2 * S::H_TILE;
                mbar_expect_tx(&h_full[hs], 2 * S::H_TILE);
                tma_2d(dst, &map_h_hi, 0, k0 + j * kEdgeTile, &h_full[hs]);
                tma_2d(dst + S::H_TILE, &map_h_lo, 0, k0 + j * kEdgeTile, &h_full[hs]);
                h_issued = j + 1;
            };
            load_h(0);
            if (S::HS > 1 && ntiles > 1) load_h(1);
            const bool w3_ok = mbar_wait_one(w3_full, 0);
            bool ok = w3_ok;
            constexpr uint32_t id_w = idesc_f16(kRowTile, kEdgeTile);                 // W3^T . H^T
            constexpr uint32_t id_gw = idesc_f16(kRowTile, kH, false, true);          // G . H (B MN-major)
            constexpr uint32_t id_gd = idesc_f16(kH, kEdgeTile, true, true);          // W3 . G (both MN-major)
            for (int j = 0; j < ntiles && ok; ++j) {
                const int s = j & 1, hst = j % S::HS;
                ok = mbar_wait_one(&h_full[hst], (uint32_t)(j / S::HS) & 1u);
                if (!ok) break;
                h_waited = j + 1;
                ok = (j < 2 || mbar_wait_one(&t_empty[s], (uint32_t)((j >> 1) - 1) & 1u)) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                const uint8_t* hs = base + S::H_OFF + hst * 2 * S::H_TILE;
                const uint64_t dbh = sw128_desc(smem_addr(hs)), dbl = sw128_desc(smem_addr(hs + S::H_TILE));
                // w of this tile
                for (int t = 0; t < gtiles; ++t) {
                    const uint8_t* at = base + S::W3_OFF + t * 2 * S::A_TILE;
                    const uint64_t dah = sw128_desc(smem_addr(at)), dal = sw128_desc(smem_addr(at + S::A_TILE));
                    const uint32_t d = tmem + kColW + (uint32_t)((s * kBwdGroupTiles + t) * kEdgeTile);
#pragma unroll
                    for (int kk = 0; kk < kH / 16; ++kk) {
                        const uint64_t adv = (uint64_t)(kk * 32) >> 4;
                        umma_f16(d, dah + adv, dbh + adv, id_w, kk > 0);
                        umma_f16(d, dah + adv, dbl + adv, id_w, 1);
                        umma_f16(d, dal + adv, dbh + adv, id_w, 1);
                    }
                }
                umma_commit(&t_full[s]);
                committed = j + 1;
                // the path warps' G tile of this tile, then g_W3 += G . H and Gd = W3 . G
                ok = mbar_wait_one(g_full, (uint32_t)j & 1u) &&
                     (j == 0 || mbar_wait_one(gd_empty, (uint32_t)(j - 1) & 1u)) && !*abort_flag;
                if (!ok) break;
                tc_fence_after();
                for (int t = 0; t < gtiles; ++t) {
                    const uint8_t* gt = base + S::G_OFF + t * 2 * S::G_TILE;
                    const uint64_t dgh = sw128_desc(smem_addr(gt)), dgl = sw128_desc(smem_addr(gt + S::G_TILE));
                    const uint32_t d = tmem + kColGW + (uint32_t)(t * kH);
#pragma unroll
                    for (int kk = 0; kk < kEdgeTile / 16; ++kk) {
                        const uint64_t a_adv = (uint64_t)(kk * 32) >> 4;      // G: K-major, 16 edges = 32 B
                        const uint64_t b_adv = (uint64_t)(kk * 2048) >> 4;    // H: MN-major, 16 edge rows
                        umma_f16(d, dgh + a_adv, dbh + b_adv, id_gw, (j > 0 || kk > 0) ? 1u : 0u);
                        umma_f16(d, dgh + a_adv, dbl + b_adv, id_gw, 1);
                        umma_f16(d, dgl + a_adv, dbh + b_adv, id_gw, 1);
                    }
                }
                for (int t = 0; t < gtiles; ++t) {
                    const uint8_t* at = base + S::W3_OFF + t * 2 * S::A_TILE;
                    const uint8_t* gt = base + S::G_OFF + t * 2 * S::G_TILE;
                    const uint64_t dah = sw128_desc(smem_addr(at)), dal = sw128_desc(smem_addr(at + S::A_TILE));
                    const uint64_t dgh = sw128_desc(smem_addr(gt)), dgl = sw128_desc(smem_addr(gt + S::G_TILE));
#pragma unroll
                    for (int kk = 0; kk < kRowTile / 16; ++kk) {
                        const uint64_t adv = (uint64_t)(kk * 2048) >> 4;      // 16 (path, channel) rows
                        umma_f16(tmem + kColGD, dah + adv, dgh + adv, id_gd, (t > 0 || kk > 0) ? 1u : 0u);
                        umma_f16(tmem + kColGD, dah + adv, dgl + adv, id_gd, 1);
                        umma_f16(tmem + kColGD, dal + adv, dgh + adv, id_gd, 1);
                    }
                }
                umma_commit(g_empty);
                umma_commit(gd_full);
                umma_commit(&h_empty[hst]);
                g_done = j + 1;
                if (j + S::HS < ntiles) {
                    ok = mbar_wait_one(&h_empty[hst], (uint32_t)(j / S::HS) & 1u);
                    if (ok) load_h(j + S::HS);
                }
            }
            if (ok && !*abort_flag) {
                umma_commit(gw_full);
            } else {
                atomicOr(prm.status, 4u);
                *abort_flag = 1;
                // let the copies and products in flight land before the CTA lets go of its memory
                if (!w3_ok) mbar_wait_one(w3_full, 0);
                for (int u = h_waited; u < h_issued; ++u)
                    mbar_wait_one(&h_full[u % S::HS], (uint32_t)(u / S::HS) & 1u);
                for (int u = committed > 2 ? committed - 2 : 0; u < committed; ++u)
                    mbar_wait_one(&t_full[u & 1], (uint32_t)(u >> 1) & 1u);
                if (g_done > 0) mbar_wait_one(g_empty, (uint32_t)(g_done - 1) & 1u);
            }
        }
    } else if (warp == kBwdGyWarp) {
        // receiver rows of gy, batch by batch: one barrier per batch of BT
        // positions; lane t copies the row of position kb + t
        constexpr int BT = S::BT;
        const int nbatch = (k1 - k0 + BT - 1) / BT;
        int issued = 0;
        for (int b = 0; b < nbatch; ++b) {
            const int kb = k0 + b * BT;
            const int nb = min(BT, k1 - kb);
            int ridx = 0, own = 0;
            float4 rc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane < nb) {
                const int2 id = prm.ids[kb + lane];
                rc = prm.rec[kb + lane];
                ridx = id.x;
                own = id.y;
                if ((unsigned)ridx >= (unsigned)prm.N) {   // out of range: flagged, read as node 0
                    atomicOr(prm.status, 1u);
                    ridx = 0;
                }
            }
            int go = 1;
            if (lane == 0) {
                if (b >= S::GYB && !mbar_wait_one(&gy_empty[b % S::GYB], (uint32_t)(b / S::GYB - 1) & 1u)) {
                    atomicOr(prm.status, 4u);
                    *abort_flag = 1;
                }
                go = *abort_flag ? 0 : 1;
                if (go) mbar_expect_tx(&gy_full[b % S::GYB], nb * S::GY_SLOT);
            }
            if (!__shfl_sync(0xffffffffu, go, 0)) break;
            if (lane < nb)
                tma_rows(base + S::GY_OFF + ((b % S::GYB) * BT + lane) * S::GY_SLOT, &map_gy, c0, ridx,
                         &gy_full[b % S::GYB], policy_evict_last());
            issued = b + 1;
            // each position's harmonics, edge factor and sender for the path warps
            if (lane < nb) {
                float* yrow = reinterpret_cast<float*>(base + S::Y_OFF + (b % S::GYB) * S::YB_BATCH) +
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
            if (lane == 0) mbar_arrive(&gy_full[b % S::GYB]);
        }
        // the last fills of each buffer land before the CTA lets go of its memory
        if (lane == 0)
            for (int b = issued > S::GYB ? issued - S::GYB : 0; b < issued; ++b)
                mbar_wait_one(&gy_full[b % S::GYB], (uint32_t)(b / S::GYB) & 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kBwdTmemCols);
    }
}

}  // namespace radial
}  // namespace eqc

namespace eqc {
namespace radial {

// ---------------------------------------------------------------- helpers

// out[0] = max |a| over n floats (as the bits of a non-negative float);
// out must be zeroed first.  Grid-stride, float4 loads (n % 4 == 0).
__global__ void radial_absmax_kernel(const float* __restrict__ a, int64_t n4, unsigned* __restrict__ out) {
    float m = 0.f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(a) + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(out, __float_as_uint(m));
}

__device__ __forceinline__ float silu_grad(float z) {
    const float s = 1.f / (1.f + expf(-z));
    return s * (1.f + z * (1.f - s));
}

// dx[j, l1^2 + m, c] = sum over paths p with that l1, in path order, of
// dx_pp[j, dx_off(p) + m, c].
template <class K>
__global__ void radial_sum_dx_kernel(const float* __restrict__ dx_pp, float* __restrict__ dx, int N, int C) {
    using R = BwdRows<K>;
    const int c4 = C / 4;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)N * K::D_IN * c4) return;
    const int cq = (int)(idx % c4);
    const int row = (int)((idx / c4) % K::D_IN);
    const int j = (int)(idx / ((int64_t)c4 * K::D_IN));
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    static_for<K::NP>([&](auto pc) {
        constexpr int p = EQC_CV(pc);
        constexpr int l1 = K::PL.l1[p];
        if (row >= l1 * l1 && row < (l1 + 1) * (l1 + 1)) {
            const float4 v = __ldcs(reinterpret_cast<const float4*>(
                dx_pp + ((size_t)j * R::DX_PP + R::dx_off(p) + (row - l1 * l1)) * C) + cq);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
    });
    __stcs(reinterpret_cast<float4*>(dx + ((size_t)j * K::D_IN + row) * C) + cq, s);
}

// Per tile of 64 sender positions k (edge e = perm[k]); 256 threads, the CTA
// walking `chunks` tiles in order:
//   Gd = sum of the (slice, group) partials, unscaled;  g_z2 = u Gd silu'(z2);
//   g_u = h2 . Gd;  back through the two SiLU layers (recomputed) to g_b;
//   g_d = g_b . b'(d) + g_u u'(d);  gY = sum of the per-path partials;
//   dr[e] = (dY/dr)^T gY + g_d r / d.
// The MLP layers of a tile are small GEMMs ([64 positions] x [64] x [64]):
// each thread owns a 4 x 4 block of every product (rows 4 tk.., columns
// 4 tj..), operands from shared memory as float4 rows.  The CTA's partial
// sums of g_W2 = sum_k h1 (x) g_z2 and g_W1 = sum_k b (x) g_z1 stay in the
// threads' registers (positions in order: deterministic) and go to
// gw2_part / gw1_part [CTA].
constexpr int kEpiThreads = 256;
constexpr int kEpiTile = 64;             // positions per tile
constexpr int kEpiLd = kH + 4;           // padded row stride of the activation tiles
constexpr int kEpiSmemFloats =
    kMaxBasis * kH + 2 * kH * kH + 3 * kEpiTile * kEpiLd + 2 * kEpiTile * kMaxBasis + 3 * kEpiTile;
constexpr int kEpiSmemBytes = kEpiSmemFloats * 4;

template <class K>
__global__ void __launch_bounds__(kEpiThreads, 2)
    radial_bwd_epilogue_kernel(const float* __restrict__ r, const int* __restrict__ perm, int E,
                               const float* __restrict__ W1, const float* __restrict__ W2, int NB, float rc,
                               const float* __restrict__ scal, const float* __restrict__ zscale,
                               const float* __restrict__ gy_part, int slices, const float* __restrict__ gd_part,
                               int SG, int chunks, float* __restrict__ dr, float* __restrict__ gw1_part,
                               float* __restrict__ gw2_part) {
    using R = BwdRows<K>;
    extern __shared__ __align__(16) float epi_smem[];   // kEpiSmemBytes
    float* sW1 = epi_smem;                               // [kMaxBasis][kH], rows >= NB zero
    float* sW2 = sW1 + kMaxBasis * kH;                   // [kH][kH]
    float* sW2T = sW2 + kH * kH;                         // [kH][kH] transposed
    float* sH1 = sW2T + kH * kH;                         // [64][kEpiLd] h1
    float* sG2 = sH1 + kEpiTile * kEpiLd;                // [64][kEpiLd] g_z2
    float* sG1 = sG2 + kEpiTile * kEpiLd;                // [64][kEpiLd] g_z1
    float* sB = sG1 + kEpiTile * kEpiLd;                 // [64][kMaxBasis] Bessel values
    float* sGb = sB + kEpiTile * kMaxBasis;              // [64][kMaxBasis] their derivatives in d
    float* sFac = sGb + kEpiTile * kMaxBasis;            // [64] unscaling of Gd
    float* sGud = sFac + kEpiTile;                       // [64] g_u u'(d)
    float* sGdl = sGud + kEpiTile;                       // [64] g_b . b'(d)
    const int t = threadIdx.x, tk = t >> 4, tj = t & 15;
    for (int i = t; i < kMaxBasis * kH; i += kEpiThreads) sW1[i] = i < NB * kH ? W1[i] : 0.f;
    for (int i = t; i < kH * kH; i += kEpiThreads) {
        const float v = W2[i];
        sW2[i] = v;
        sW2T[(i % kH) * kH + i / kH] = v;
    }
    const int sA = inv_pow2_exponent(scal[0]);
    const int gexp = g_scale_exponent(scal);
    float gw2[4][4];   // g_W2 rows 4 tk + i, columns 4 tj + c
    float gw1[4];      // g_W1 rows (t >> 6) + 4 i, column t & 63
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        gw1[i] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) gw2[i][c] = 0.f;
    }

    for (int ch = 0; ch < chunks; ++ch) {
        const int kbase = (blockIdx.x * chunks + ch) * kEpiTile;
        if (kbase >= E) break;   // uniform over the CTA
        __syncthreads();   // weights loaded / the previous tile consumed
        // 1. per-position terms (threads 0..63)
        float d0 = 0.f, d1v = 0.f, d2v = 0.f, rx = 0.f, ry = 0.f, rz = 0.f, inv_d = 0.f, d = 0.f;
        int e = -1;
        if (t < kEpiTile) {
            const int k = kbase + t;
            float* bb = sB + t * kMaxBasis;
            float* gb = sGb + t * kMaxBasis;
            if (k < E) {
                e = perm[k];
                rx = r[(size_t)e * 3];
                ry = r[(size_t)e * 3 + 1];
                rz = r[(size_t)e * 3 + 2];
                d = sqrtf(fmaf(rx, rx, fmaf(ry, ry, rz * rz)));
                inv_d = 1.f / fmaxf(d, 1e-12f);
                const float pref = sqrtf(2.f / rc);
                const float kd = 3.14159265358979323846f * d / rc;
                for (int n = 0; n < NB; ++n) {
                    float sn, cn;
                    sincosf((float)(n + 1) * kd, &sn, &cn);
                    const float kn = (float)(n + 1) * 3.14159265358979323846f / rc;
                    bb[n] = pref * sn * inv_d;
                    gb[n] = pref * (kn * cn * inv_d - sn * inv_d * inv_d);
                }
                const float x = fminf(d / rc, 1.f);
                // u'(d) = (-168 x^5 + 336 x^6 - 168 x^7) / rc, zero from the cutoff on
                const float x2 = x * x, x5 = x2 * x2 * x;
                const float du = d < rc ? x5 * fmaf(x, fmaf(-168.f, x, 336.f), -168.f) / rc : 0.f;
                // with G = dw 2^gexp uscale_e = u dw 2^gexp zscale_e, the summed partials are
                // D = sum_pc (W3 2^sA) G = 2^(sA + gexp) zscale_e u W3 . dw
                const float zs = zscale[k];
                sFac[t] = ldexpf(1.f, -(sA + gexp)) / zs;
                // g_u = sum_pc dw z3: the paths' partials (each sum dw D, D = z3 / zscale)
                float gu = 0.f;
                for (int s = 0; s < slices; ++s) {
                    const float* gp = gy_part + ((size_t)k * slices + s) * R::SD2;
                    static_for<K::NP>([&](auto pc) { gu += gp[R::gy_off(EQC_CV(pc))]; });
                }
                sGud[t] = gu * zs * du;
                // harmonic gradient: the per-path partials, in (slice, path) order
                float ux, uy, uz, il;
                const bool ok = unit_dir(rx, ry, rz, ux, uy, uz, il);
                if constexpr (K::G > 0) {
                    float gY[K::G];
#pragma unroll
                    for (int q = 0; q < K::G; ++q) gY[q] = 0.f;
                    for (int s = 0; s < slices; ++s) {
                        const float* gp = gy_part + ((size_t)k * slices + s) * R::SD2;
                        static_for<K::NP>([&](auto pc) {
                            constexpr int p = EQC_CV(pc);
                            constexpr int l2 = K::PL.l2[p];
                            if constexpr (l2 > 0) {
#pragma unroll
                                for (int m = 0; m < 2 * l2 + 1; ++m) gY[l2 * l2 - 1 + m] += gp[R::gy_off(p) + 1 + m];
                            }
                        });
                    }
                    sh_grad_contract<K::LSH>(ok, ux, uy, uz, il, gY, d0, d1v, d2v);
                }
            } else {
                for (int n = 0; n < NB; ++n) bb[n] = gb[n] = 0.f;
                sFac[t] = 0.f;
                sGud[t] = 0.f;
            }
        }
        __syncthreads();
        // 2. z1 = b . W1, h1 = silu(z1)
        float dz1[4][4];
        {
            float z[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) z[i][c] = 0.f;
            for (int n = 0; n < NB; ++n) {
                const float4 w = *reinterpret_cast<const float4*>(sW1 + n * kH + 4 * tj);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float a = sB[(4 * tk + i) * kMaxBasis + n];
                    z[i][0] = fmaf(a, w.x, z[i][0]);
                    z[i][1] = fmaf(a, w.y, z[i][1]);
                    z[i][2] = fmaf(a, w.z, z[i][2]);
                    z[i][3] = fmaf(a, w.w, z[i][3]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float h[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    h[c] = silu(z[i][c]);
                    dz1[i][c] = silu_grad(z[i][c]);
                }
                *reinterpret_cast<float4*>(sH1 + (4 * tk + i) * kEpiLd + 4 * tj) = make_float4(h[0], h[1], h[2], h[3]);
            }
        }
        __syncthreads();
        // 3. z2 = h1 . W2, g_z2 = Gd fac silu'(z2)
        {
            float z[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) z[i][c] = 0.f;
#pragma unroll 4
            for (int q = 0; q < kH; q += 4) {
                float4 a[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(sH1 + (4 * tk + i) * kEpiLd + q);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const float4 w = *reinterpret_cast<const float4*>(sW2 + (q + qq) * kH + 4 * tj);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float av = qq == 0 ? a[i].x : qq == 1 ? a[i].y : qq == 2 ? a[i].z : a[i].w;
                        z[i][0] = fmaf(av, w.x, z[i][0]);
                        z[i][1] = fmaf(av, w.y, z[i][1]);
                        z[i][2] = fmaf(av, w.z, z[i][2]);
                        z[i][3] = fmaf(av, w.w, z[i][3]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int k = kbase + 4 * tk + i;
                float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
                if (k < E)
                    for (int q = 0; q < SG; ++q) {
                        const float4 v = __ldcs(reinterpret_cast<const float4*>(gd_part + ((size_t)q * E + k) * kH + 4 * tj));
                        g.x += v.x;
                        g.y += v.y;
                        g.z += v.z;
                        g.w += v.w;
                    }
                const float f = sFac[4 * tk + i];
                *reinterpret_cast<float4*>(sG2 + (4 * tk + i) * kEpiLd + 4 * tj) =
                    make_float4(g.x * f * silu_grad(z[i][0]), g.y * f * silu_grad(z[i][1]),
                                g.z * f * silu_grad(z[i][2]), g.w * f * silu_grad(z[i][3]));
            }
        }
        __syncthreads();
        // 4. g_z1 = (g_z2 . W2^T) silu'(z1);  g_W2 += h1^T g_z2
        {
            float z[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) z[i][c] = 0.f;
#pragma unroll 4
            for (int j = 0; j < kH; j += 4) {
                float4 a[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(sG2 + (4 * tk + i) * kEpiLd + j);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const float4 w = *reinterpret_cast<const float4*>(sW2T + (j + jj) * kH + 4 * tj);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float av = jj == 0 ? a[i].x : jj == 1 ? a[i].y : jj == 2 ? a[i].z : a[i].w;
                        z[i][0] = fmaf(av, w.x, z[i][0]);
                        z[i][1] = fmaf(av, w.y, z[i][1]);
                        z[i][2] = fmaf(av, w.z, z[i][2]);
                        z[i][3] = fmaf(av, w.w, z[i][3]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4*>(sG1 + (4 * tk + i) * kEpiLd + 4 * tj) =
                    make_float4(z[i][0] * dz1[i][0], z[i][1] * dz1[i][1], z[i][2] * dz1[i][2], z[i][3] * dz1[i][3]);
#pragma unroll 4
            for (int k = 0; k < kEpiTile; ++k) {
                const float4 h = *reinterpret_cast<const float4*>(sH1 + k * kEpiLd + 4 * tk);
                const float4 g = *reinterpret_cast<const float4*>(sG2 + k * kEpiLd + 4 * tj);
                const float hv[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    gw2[i][0] = fmaf(hv[i], g.x, gw2[i][0]);
                    gw2[i][1] = fmaf(hv[i], g.y, gw2[i][1]);
                    gw2[i][2] = fmaf(hv[i], g.z, gw2[i][2]);
                    gw2[i][3] = fmaf(hv[i], g.w, gw2[i][3]);
                }
            }
        }
        __syncthreads();
        // 5. g_b . b'(d) per position (4 threads each, fixed order);  g_W1 += b^T g_z1
        {
            const int kk = t >> 2, ng = t & 3;
            float part = 0.f;
            for (int n = ng; n < NB; n += 4) {
                float sdot = 0.f;
#pragma unroll 4
                for (int j = 0; j < kH; j += 4) {
                    const float4 g = *reinterpret_cast<const float4*>(sG1 + kk * kEpiLd + j);
                    const float4 w = *reinterpret_cast<const float4*>(sW1 + n * kH + j);
                    sdot = fmaf(g.x, w.x, fmaf(g.y, w.y, fmaf(g.z, w.z, fmaf(g.w, w.w, sdot))));
                }
                part = fmaf(sdot, sGb[kk * kMaxBasis + n], part);
            }
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (ng == 0) sGdl[kk] = part;
            const int jc = t & 63, n0 = t >> 6;
#pragma unroll 4
            for (int k = 0; k < kEpiTile; ++k) {
                const float g = sG1[k * kEpiLd + jc];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (n0 + 4 * i < NB) gw1[i] = fmaf(sB[k * kMaxBasis + n0 + 4 * i], g, gw1[i]);
            }
        }
        __syncthreads();
        // 6. dr
        if (t < kEpiTile && e >= 0) {
            const float gd_len = sGdl[t] + sGud[t];
            if (d > 1e-12f) {
                d0 = fmaf(gd_len, rx * inv_d, d0);
                d1v = fmaf(gd_len, ry * inv_d, d1v);
                d2v = fmaf(gd_len, rz * inv_d, d2v);
            }
            dr[(size_t)e * 3] = d0;
            dr[(size_t)e * 3 + 1] = d1v;
            dr[(size_t)e * 3 + 2] = d2v;
        }
    }
    float* o2 = gw2_part + (size_t)blockIdx.x * kH * kH;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float4*>(o2 + (4 * tk + i) * kH + 4 * tj) = make_float4(gw2[i][0], gw2[i][1], gw2[i][2], gw2[i][3]);
    float* o1 = gw1_part + (size_t)blockIdx.x * kMaxBasis * kH;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if ((t >> 6) + 4 * i < NB) o1[((t >> 6) + 4 * i) * kH + (t & 63)] = gw1[i];
}

// out[i] = sum_{b < nb} part[b * stride + i], in order of b (i < n).
__global__ void radial_sum_parts_kernel(const float* __restrict__ part, int nb, int64_t stride, int64_t n,
                                        float* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float s = 0.f;
    for (int b = 0; b < nb; ++b) s += part[(size_t)b * stride + i];
    out[i] = s;
}

// g_W3[k][pc] = 2^(sA - gexp) * sum over ranges of gw3_part[range][pc][k].
__global__ void radial_sum_gw3_kernel(const float* __restrict__ part, int nranges, int PC,
                                      const float* __restrict__ scal, float* __restrict__ gw3) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // over pc * 64 + k
    if (i >= (int64_t)PC * kH) return;
    const int pc = (int)(i / kH), k = (int)(i % kH);
    float s = 0.f;
    for (int b = 0; b < nranges; ++b) s += part[((size_t)b * PC + pc) * kH + k];
    gw3[(size_t)k * PC + pc] = s * ldexpf(1.f, inv_pow2_exponent(scal[0]) - g_scale_exponent(scal));
}

}  // namespace radial
}  // namespace eqc

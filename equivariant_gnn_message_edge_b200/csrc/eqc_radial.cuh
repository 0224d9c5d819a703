// Radial weights of the convolution produced on the chip (sm_100a).
//
// FlashCart (arXiv 2610.06409) App. B: a radial envelope makes every edge's
// contribution vanish smoothly at the cutoff, keeping the energy twice
// differentiable in the positions; App. E: the radial weights vanish with
// their first two derivatives at the cutoff.  e3j (arXiv 2609.35099) Table 3:
// the MACE(a) model has 8 radial (Bessel) functions and a 5 Angstrom cutoff.
// With d = |r_e| and x = min(d / rc, 1):
//   b_n(d) = sqrt(2 / rc) sin(n pi d / rc) / d               n = 1 .. NB
//   u(d)   = 1 - 28 x^6 + 48 x^7 - 21 x^8                     (p = 6 envelope)
//   h2     = silu(silu(b W1) W2)                              [64]
//   w[e, p, c] = u(d) * sum_k h2[k] W3[k, p*C + c]
// (no biases; silu(z) = z / (1 + exp(-z))).
//
// The first two layers are small per edge and run on the CUDA cores
// (radial_hidden_kernel).  The last layer is a dense contraction, [edges x
// 64] . [64 x P*C], and runs on the tensor cores: tcgen05.mma kind::f16 with
// fp32 accumulators in tensor memory, operands staged by TMA.  To keep fp32
// accuracy both operands are split into fp16 pairs, v * 2^s = hi + lo with
// hi = fp16(v * 2^s), lo = fp16(v * 2^s - hi), and
//   D = A_hi B_hi + A_hi B_lo + A_lo B_hi
// (the dropped A_lo B_lo is below 2^-22 of the product).  The powers of two
// put every operand's largest magnitude in [2^13, 2^14): one for all of W3,
// one per edge for h2; they are undone exactly in the per-edge factor
//   uscale[e] = u(d) * 2^-(s_W3 + s_h2(e)),   w = D * uscale.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "eqc_conv.cuh"

namespace eqc {
namespace radial {

constexpr int kH = 64;          // hidden width: the K of the last layer's contraction
constexpr int kMaxBasis = 16;   // Bessel functions
constexpr int kRowTile = 128;   // M of one MMA: rows of W3^T (path x channel)
constexpr int kEdgeTile = 64;   // N of one MMA: edges
constexpr int kTileRowBytes = kH * 2;   // one fp16 row of 64 values: 128 B, one swizzle atom wide

// ------------------------------------------------------------ small helpers

__device__ __forceinline__ float silu(float z) { return z / (1.f + expf(-z)); }

// 2^s with s such that m * 2^s lies in [2^13, 2^14) (s = 0 for m = 0).
__device__ __forceinline__ int pow2_exponent_for(float m) {
    if (!(m > 0.f)) return 0;
    int e;
    frexpf(m, &e);   // m = f * 2^e, f in [0.5, 1)
    return 14 - e;
}

__device__ __forceinline__ void split_f16(float v, __half& hi, __half& lo) {
    hi = __float2half_rn(v);
    lo = __float2half_rn(v - __half2float(hi));
}

__device__ __forceinline__ float envelope(float d, float rc) {
    const float x = fminf(d / rc, 1.f);
    const float x2 = x * x, x6 = x2 * x2 * x2;
    return fmaf(x6, fmaf(x, fmaf(-21.f, x, 48.f), -28.f), 1.f);
}

// ---------------------------------------------------------- tcgen05 pieces

// Shared-memory matrix descriptor of a tile stored as rows of 128 B with the
// 128-byte swizzle (what a TMA copy with CU_TENSOR_MAP_SWIZZLE_128B writes):
// 8-row groups 1024 B apart.  Read K-major (rows = M or N, the 128 B of a row
// = K) or MN-major (rows = K, the 128 B of a row = 64 values of M or N).  The
// tile must start on a 1024-byte boundary; a K step inside the row moves the
// start address (32 B per 16 fp16 values).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_byte_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_byte_addr >> 4) & 0x3FFFu);   // start address, 16 B units
    d |= (uint64_t)1u << 16;                             // leading byte offset (unused by this layout)
    d |= (uint64_t)(1024u >> 4) << 32;                   // stride byte offset: 8-row groups
    d |= (uint64_t)1u << 46;                             // descriptor version of sm_100
    d |= (uint64_t)2u << 61;                             // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16 with fp16 A and B, fp32 accumulators,
// an M x N tile; a_mn / b_mn: operand stored MN-major (else K-major).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn = false, bool b_mn = false) {
    return (1u << 4)                           // D format: f32
           | (0u << 7) | (0u << 10)            // A, B format: f16
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A . B^T for one K = 16 step; issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Tensor-memory allocation (one whole warp); the base address lands in *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 16 consecutive fp32 columns of this warp's 32 lanes (lane = thread).  The
// wait is part of the call and takes the registers as operands, so no use of
// them can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 2-D tensor-map copy of the box at (x, y) into shared memory, counted on `bar`.
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// Bounded wait of a single thread (the MMA issuer) on one phase of `bar`.
__device__ __forceinline__ bool mbar_wait_one(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_addr(bar);
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity), "r"(kWaitSuspendNs)
            : "memory");
        if (done) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// --------------------------------------------------------------- W3 prep

// A_hi / A_lo [PC][64] fp16 = split(W3^T * 2^s), s for the largest |W3|;
// inv_scale[0] = 2^-s.  One CTA of 1024 threads (W3 has 64 * P * C values).
__global__ void __launch_bounds__(1024)
    radial_prep_w3_kernel(const float* __restrict__ W3, int PC, __half* __restrict__ A_hi, __half* __restrict__ A_lo,
                          float* __restrict__ inv_scale) {
    __shared__ float red[32];
    const int tid = threadIdx.x;
    const int n = kH * PC;
    float m = 0.f;
    for (int i = tid; i < n; i += blockDim.x) m = fmaxf(m, fabsf(W3[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid < 32) {
        m = tid < (int)(blockDim.x >> 5) ? red[tid] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (tid == 0) red[0] = m;
    }
    __syncthreads();
    const int s = pow2_exponent_for(red[0]);
    const float sc = ldexpf(1.f, s);
    for (int i = tid; i < n; i += blockDim.x) {
        const int pc = i / kH, k = i - pc * kH;
        __half hi, lo;
        split_f16(W3[(size_t)k * PC + pc] * sc, hi, lo);
        A_hi[i] = hi;
        A_lo[i] = lo;
    }
    if (tid == 0) inv_scale[0] = ldexpf(1.f, -s);
}

// ------------------------------------------------------- hidden layers

// For output position k (edge e = perm[k], or k without perm): the two
// hidden layers on the CUDA cores, then h2 split into fp16 pairs with its own
// power of two (H_hi / H_lo [E][64]), and uscale[k] = u(d) * 2^-(s_W3 +
// s_h2).  One thread per edge; W1 and W2 are read from shared memory by all
// threads at once (broadcast).
__global__ void __launch_bounds__(128)
    radial_hidden_kernel(const float* __restrict__ r, const int* __restrict__ perm, int E,
                         const float* __restrict__ W1, const float* __restrict__ W2, int NB, float rc,
                         const float* __restrict__ w3_inv_scale, __half* __restrict__ H_hi,
                         __half* __restrict__ H_lo, float* __restrict__ uscale) {
    __shared__ __align__(16) float sW1[kMaxBasis * kH];
    __shared__ __align__(16) float sW2[kH * kH];
    for (int i = threadIdx.x; i < NB * kH; i += blockDim.x) sW1[i] = W1[i];
    for (int i = threadIdx.x; i < kH * kH; i += blockDim.x) sW2[i] = W2[i];
    __syncthreads();
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= E) return;
    const int e = perm ? perm[k] : k;
    const float rx = r[(size_t)e * 3], ry = r[(size_t)e * 3 + 1], rz = r[(size_t)e * 3 + 2];
    const float d = sqrtf(fmaf(rx, rx, fmaf(ry, ry, rz * rz)));
    const float inv_d = 1.f / fmaxf(d, 1e-12f);
    const float pref = sqrtf(2.f / rc);
    const float kd = 3.14159265358979323846f * d / rc;
    float h1[kH];
#pragma unroll
    for (int j = 0; j < kH; ++j) h1[j] = 0.f;
    for (int nb = 0; nb < NB; ++nb) {
        const float b = pref * sinf((float)(nb + 1) * kd) * inv_d;
#pragma unroll
        for (int j = 0; j < kH; ++j) h1[j] = fmaf(b, sW1[nb * kH + j], h1[j]);
    }
#pragma unroll
    for (int j = 0; j < kH; ++j) h1[j] = silu(h1[j]);
    float h2[kH];
#pragma unroll
    for (int j = 0; j < kH; ++j) h2[j] = 0.f;
#pragma unroll 4
    for (int q = 0; q < kH; ++q) {
        const float a = h1[q];
#pragma unroll
        for (int j = 0; j < kH; j += 4) {
            const float4 wv = *reinterpret_cast<const float4*>(&sW2[q * kH + j]);
            h2[j] = fmaf(a, wv.x, h2[j]);
            h2[j + 1] = fmaf(a, wv.y, h2[j + 1]);
            h2[j + 2] = fmaf(a, wv.z, h2[j + 2]);
            h2[j + 3] = fmaf(a, wv.w, h2[j + 3]);
        }
    }
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < kH; ++j) {
        h2[j] = silu(h2[j]);
        m = fmaxf(m, fabsf(h2[j]));
    }
    const int s = pow2_exponent_for(m);
    const float sc = ldexpf(1.f, s);
    uint4* dh = reinterpret_cast<uint4*>(H_hi + (size_t)k * kH);
    uint4* dl = reinterpret_cast<uint4*>(H_lo + (size_t)k * kH);
#pragma unroll
    for (int q = 0; q < kH / 8; ++q) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            __half h0, l0, h1v, l1v;
            split_f16(h2[8 * q + 2 * t] * sc, h0, l0);
            split_f16(h2[8 * q + 2 * t + 1] * sc, h1v, l1v);
            hw[t] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1v) << 16);
            lw[t] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1v) << 16);
        }
        dh[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        dl[q] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    uscale[k] = envelope(d, rc) * ldexpf(1.f, -s) * w3_inv_scale[0];
}

// ------------------------------------------- last layer to w (standalone)

// w[e, pc] = uscale[e] * sum_k A[pc, k] H[e, k] for one tile of 128 rows pc
// of W3^T and 64 edges (edge = position; H and uscale in edge order): TMA
// brings the four fp16 tiles, one thread issues the 12 MMAs (3 products x 4
// K steps) into 64 columns of tensor memory, and each warp reads its 32 rows
// back (row = lane) and stores them, 32 consecutive pc per edge (128 B).
// This writes w to memory: the convolution's fused radial path keeps it on
// the chip instead; this kernel is the unfused path and a check of the
// tensor-core stage on its own.
struct WSmem {
    static constexpr int A_BYTES = kRowTile * kTileRowBytes;   // 16 KB
    static constexpr int B_BYTES = kEdgeTile * kTileRowBytes;  // 8 KB
    static constexpr int BYTES = 2 * A_BYTES + 2 * B_BYTES + 1024 /* barriers */ + 1024 /* alignment */;
};

__global__ void __launch_bounds__(128)
    radial_w_kernel(const __grid_constant__ CUtensorMap map_a_hi, const __grid_constant__ CUtensorMap map_a_lo,
                    const __grid_constant__ CUtensorMap map_h_hi, const __grid_constant__ CUtensorMap map_h_lo,
                    const float* __restrict__ uscale, int E, int PC, float* __restrict__ w, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a_hi = base;
    uint8_t* a_lo = a_hi + WSmem::A_BYTES;
    uint8_t* b_hi = a_lo + WSmem::A_BYTES;
    uint8_t* b_lo = b_hi + WSmem::B_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(b_lo + WSmem::B_BYTES);   // [0] copies, [1] MMAs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
    __shared__ int ok_shared;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row0 = blockIdx.x * kRowTile, e0 = blockIdx.y * kEdgeTile;
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        ok_shared = 1;
    }
    if (warp == 0) tmem_alloc(tmem_slot, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        mbar_expect_tx(&bars[0], 2 * WSmem::A_BYTES + 2 * WSmem::B_BYTES);
        tma_2d(a_hi, &map_a_hi, 0, row0, &bars[0]);
        tma_2d(a_lo, &map_a_lo, 0, row0, &bars[0]);
        tma_2d(b_hi, &map_h_hi, 0, e0, &bars[0]);
        tma_2d(b_lo, &map_h_lo, 0, e0, &bars[0]);
        if (mbar_wait_one(&bars[0], 0)) {
            tc_fence_after();
            constexpr uint32_t id = idesc_f16(kRowTile, kEdgeTile);
            const uint64_t dah = sw128_desc(smem_addr(a_hi)), dal = sw128_desc(smem_addr(a_lo));
            const uint64_t dbh = sw128_desc(smem_addr(b_hi)), dbl = sw128_desc(smem_addr(b_lo));
#pragma unroll
            for (int kk = 0; kk < kH / 16; ++kk) {
                const uint64_t adv = (uint64_t)(kk * 32) >> 4;   // 32 B per K step, in 16 B units
                umma_f16(tmem, dah + adv, dbh + adv, id, kk > 0);
                umma_f16(tmem, dah + adv, dbl + adv, id, 1);
                umma_f16(tmem, dal + adv, dbh + adv, id, 1);
            }
            umma_commit(&bars[1]);
        } else {
            atomicOr(status, 4u);
            ok_shared = 0;
            // nothing was issued: complete the MMA barrier's phase so the
            // other threads do not wait out their limit
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&bars[1])) : "memory");
        }
    }
    __syncwarp();
    const bool done = mbar_wait(&bars[1], 0);
    tc_fence_after();
    if (!done && lane == 0) atomicOr(status, 4u);
    if (done && ok_shared) {
        const int pc = row0 + warp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int c0 = 0; c0 < kEdgeTile; c0 += 16) {
            float v[16];
            tmem_ld16(trow + c0, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int e = e0 + c0 + j;
                if (e < E && pc < PC) w[(size_t)e * PC + pc] = v[j] * uscale[e];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

}  // namespace radial
}  // namespace eqc

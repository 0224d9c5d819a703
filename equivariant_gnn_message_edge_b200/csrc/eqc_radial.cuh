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
// one per edge for h2; they are undone exactly, with the envelope, in the
// per-edge factor
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

// s such that m * 2^s lies in [2^13, 2^14), capped at 60; 60 for m = 0.  A
// row of zeros (or of values below 2^-46) gets the largest scale, so that
// the factor 2^-s, which the backward's dw tile carries for that row, stays
// within its bound (2^-s <= 2^-13 max|h2|) and 2^-s itself stays a normal
// float.
__device__ __forceinline__ int pow2_exponent_for(float m) {
    if (!(m > 0.f)) return 60;
    int e;
    frexpf(m, &e);   // m = f * 2^e, f in [0.5, 1)
    return 14 - e < 60 ? 14 - e : 60;
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

// 4 consecutive fp32 columns of this warp's 32 lanes (as tmem_ld16).
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]) : : "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

// 8 consecutive fp32 columns of this warp's 32 lanes (as tmem_ld16).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
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

}  // namespace radial
}  // namespace eqc

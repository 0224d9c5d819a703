// Host side of the on-chip radial weights (eqc_radial.cuh): workspace layout,
// tensor maps of the fp16 operand tiles and the launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "eqc_radial.h"
#include "eqc_radial.cuh"

namespace eqc {

void count_launch();

namespace radial {

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
// power of two s (H_hi / H_lo [E][64]), uscale[k] = u(d) 2^-(s_W3 + s) (so
// that w = D * uscale) and zscale[k] = 2^-(s_W3 + s) (may be null).  hmax
// (may be null) receives the largest |h2| of all edges (as the bits of a
// non-negative float, by atomicMax).  rec / ids (may be null) receive the
// position's record for the fused kernels: (r_e, uscale) and (gathered[e],
// own[e]), so they read positions in order with no dependent loads.  One
// thread per edge; W1 and W2 are read from shared memory by all threads.
__global__ void __launch_bounds__(128)
    radial_hidden_kernel(const float* __restrict__ r, const int* __restrict__ perm, int E,
                         const float* __restrict__ W1, const float* __restrict__ W2, int NB, float rc,
                         const float* __restrict__ w3_inv_scale, __half* __restrict__ H_hi,
                         __half* __restrict__ H_lo, float* __restrict__ uscale, float* __restrict__ zscale,
                         unsigned* __restrict__ hmax, const int* __restrict__ gathered,
                         const int* __restrict__ own, float4* __restrict__ rec, int2* __restrict__ ids) {
    __shared__ __align__(16) float sW1[kMaxBasis * kH];
    __shared__ __align__(16) float sW2[kH * kH];
    for (int i = threadIdx.x; i < NB * kH; i += blockDim.x) sW1[i] = W1[i];
    for (int i = threadIdx.x; i < kH * kH; i += blockDim.x) sW2[i] = W2[i];
    __syncthreads();
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    float m = 0.f;   // largest |h2| of this thread's edge
    if (k < E) {
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
        const float z = ldexpf(1.f, -s) * w3_inv_scale[0];
        const float us = envelope(d, rc) * z;
        uscale[k] = us;
        if (zscale) zscale[k] = z;
        if (rec) {   // the fused kernels' per-position record, in the order they walk
            rec[k] = make_float4(rx, ry, rz, us);
            ids[k] = make_int2(gathered[e], own[e]);
        }
    }
    if (hmax) {   // blockDim is a multiple of 32: every lane of the warp is here
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(hmax, __float_as_uint(m));
    }
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

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [rows][64] fp16 read in boxes of box_rows rows with the 128-byte swizzle
// (one box row = 128 B = one swizzle atom); rows past the end read as zero.
bool encode_f16_rows(CUtensorMap* map, const void* base, uint64_t rows, int box_rows) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc || !base || rows == 0 || box_rows <= 0 || box_rows > 256) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kH, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kTileRowBytes};
    const cuuint32_t box[2] = {(cuuint32_t)kH, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

Workspace carve(void* ws, int E, int PC) {
    Workspace w{};
    char* p = static_cast<char*>(ws);
    const size_t a = up256((size_t)PC * kH * 2), h = up256((size_t)(E > 0 ? E : 1) * kH * 2);
    w.a_hi = reinterpret_cast<__half*>(p);
    p += a;
    w.a_lo = reinterpret_cast<__half*>(p);
    p += a;
    w.inv_scale = reinterpret_cast<float*>(p);
    p += 256;
    w.h_hi = reinterpret_cast<__half*>(p);
    p += h;
    w.h_lo = reinterpret_cast<__half*>(p);
    p += h;
    w.uscale = reinterpret_cast<float*>(p);
    p += up256((size_t)(E > 0 ? E : 1) * 4);
    w.zscale = reinterpret_cast<float*>(p);
    p += up256((size_t)(E > 0 ? E : 1) * 4);
    w.rec = reinterpret_cast<float4*>(p);
    p += up256((size_t)(E > 0 ? E : 1) * 16);
    w.ids = reinterpret_cast<int2*>(p);
    p += up256((size_t)(E > 0 ? E : 1) * 8);
    w.bytes = (size_t)(p - static_cast<char*>(ws));
    return w;
}

size_t workspace_bytes(int E, int PC) { return carve(nullptr, E, PC).bytes; }

cudaError_t prepare(const Workspace& ws, const float* r, const int* perm, int E, const float* W1, const float* W2,
                    const float* W3, int NB, float rc, int PC, cudaStream_t st, unsigned* hmax, const int* gathered,
                    const int* own) {
    radial_prep_w3_kernel<<<1, 1024, 0, st>>>(W3, PC, ws.a_hi, ws.a_lo, ws.inv_scale);
    count_launch();
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || E == 0) return err;
    radial_hidden_kernel<<<(E + 127) / 128, 128, 0, st>>>(r, perm, E, W1, W2, NB, rc, ws.inv_scale, ws.h_hi,
                                                          ws.h_lo, ws.uscale, ws.zscale, hmax, gathered, own,
                                                          gathered ? ws.rec : nullptr, gathered ? ws.ids : nullptr);
    count_launch();
    return cudaGetLastError();
}

cudaError_t weights(const Workspace& ws, int E, int PC, float* w, unsigned* status, cudaStream_t st) {
    if (E == 0) return cudaSuccess;
    CUtensorMap ma_hi, ma_lo, mh_hi, mh_lo;
    if (!encode_f16_rows(&ma_hi, ws.a_hi, (uint64_t)PC, kRowTile) ||
        !encode_f16_rows(&ma_lo, ws.a_lo, (uint64_t)PC, kRowTile) ||
        !encode_f16_rows(&mh_hi, ws.h_hi, (uint64_t)E, kEdgeTile) ||
        !encode_f16_rows(&mh_lo, ws.h_lo, (uint64_t)E, kEdgeTile))
        return cudaErrorInvalidValue;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        err = cudaFuncSetAttribute(radial_w_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, WSmem::BYTES);
        if (err != cudaSuccess) return err;
        attr_done[dev] = true;
    }
    const dim3 grid((PC + kRowTile - 1) / kRowTile, (E + kEdgeTile - 1) / kEdgeTile);
    radial_w_kernel<<<grid, 128, WSmem::BYTES, st>>>(ma_hi, ma_lo, mh_hi, mh_lo, ws.uscale, E, PC, w, status);
    count_launch();
    return cudaGetLastError();
}

}  // namespace radial
}  // namespace eqc

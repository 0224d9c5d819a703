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
    w.bytes = (size_t)(p - static_cast<char*>(ws));
    return w;
}

size_t workspace_bytes(int E, int PC) { return carve(nullptr, E, PC).bytes; }

cudaError_t prepare(const Workspace& ws, const float* r, const int* perm, int E, const float* W1, const float* W2,
                    const float* W3, int NB, float rc, int PC, cudaStream_t st) {
    radial_prep_w3_kernel<<<1, 1024, 0, st>>>(W3, PC, ws.a_hi, ws.a_lo, ws.inv_scale);
    count_launch();
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || E == 0) return err;
    radial_hidden_kernel<<<(E + 127) / 128, 128, 0, st>>>(r, perm, E, W1, W2, NB, rc, ws.inv_scale, ws.h_hi,
                                                          ws.h_lo, ws.uscale);
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

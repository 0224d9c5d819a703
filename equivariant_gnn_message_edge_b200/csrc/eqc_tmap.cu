// Tensor maps of the row tensors the kernels stage with TMA (host side).
//
// The library does not link libcuda: cuTensorMapEncodeTiled is reached
// through the runtime's driver entry point query.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "eqc_dispatch.h"

namespace eqc {

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

bool encode_rows_map(CUtensorMap* map, const void* base, uint64_t count, int rows, int C, int tile_c) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || !base || count == 0 || rows <= 0 || rows > 256 || tile_c > 256) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)rows, (cuuint64_t)count};
    const cuuint64_t strides[2] = {(cuuint64_t)C * 4u, (cuuint64_t)rows * (cuuint64_t)C * 4u};
    const cuuint32_t box[3] = {(cuuint32_t)tile_c, (cuuint32_t)rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    // promote L2 fills to the box row width at most: a wider promotion would
    // fetch the neighbouring channel tile, which is not read until much later
    const int row_bytes = tile_c * 4;
    const CUtensorMapL2promotion promo = row_bytes >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                         : row_bytes >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                                            : CU_TENSOR_MAP_L2_PROMOTION_NONE;
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, promo,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace eqc

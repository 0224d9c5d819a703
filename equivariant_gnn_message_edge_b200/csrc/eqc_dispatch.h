// Dispatch table of kernel instances (host side, no device code).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace eqc {

// Tensor map of a row-major fp32 tensor [count][rows][C] read in boxes of
// [rows][tile_c] (one box per node or edge and channel tile).  False if the
// driver entry point is unavailable or rejects the layout.
bool encode_rows_map(CUtensorMap* map, const void* base, uint64_t count, int rows, int C, int tile_c);

struct FwdParams;
struct BwdParams;

struct KernelSet {
    int lin, lsh, lout, vec, mode, tile_c, g;
    // `bands` launches over consecutive ranges of the gathered node index
    cudaError_t (*fwd)(const FwdParams&, int tiles, int bands, cudaStream_t);
    cudaError_t (*bwd)(const BwdParams&, bool det, bool fused, int bands, cudaStream_t);
};

// Instances for one (L_in, L_sh); defined in eqc_inst_l<L_in>s<L_sh>.cu.
const KernelSet* instances_l0_s0(int lout, int vec);
const KernelSet* instances_l0_s1(int lout, int vec);
const KernelSet* instances_l0_s2(int lout, int vec);
const KernelSet* instances_l0_s3(int lout, int vec);
const KernelSet* instances_l1_s0(int lout, int vec);
const KernelSet* instances_l1_s1(int lout, int vec);
const KernelSet* instances_l1_s2(int lout, int vec);
const KernelSet* instances_l1_s3(int lout, int vec);
const KernelSet* instances_l2_s0(int lout, int vec);
const KernelSet* instances_l2_s1(int lout, int vec);
const KernelSet* instances_l2_s2(int lout, int vec);
const KernelSet* instances_l2_s3(int lout, int vec);
const KernelSet* instances_l3_s0(int lout, int vec);
const KernelSet* instances_l3_s1(int lout, int vec);
const KernelSet* instances_l3_s2(int lout, int vec);
const KernelSet* instances_l3_s3(int lout, int vec);

// Instances of the output variants (mode 1: both parities, 2: per-path, 3:
// both) for one L_in, every L_sh and L_out in 1..3, one channel width each;
// defined in eqc_inst_m<mode>_l<L_in>.cu.
#define EQC_DECLARE_MODE(m)                                  \
    const KernelSet* instances_m##m##_l0(int lsh, int lout); \
    const KernelSet* instances_m##m##_l1(int lsh, int lout); \
    const KernelSet* instances_m##m##_l2(int lsh, int lout); \
    const KernelSet* instances_m##m##_l3(int lsh, int lout);
EQC_DECLARE_MODE(1)
EQC_DECLARE_MODE(2)
EQC_DECLARE_MODE(3)
#undef EQC_DECLARE_MODE

// Channel width of the output-variant instances: 1 where an l = 3 block makes
// the unrolled per-edge code large, else 2.
constexpr int mode_vec(int lin, int lsh, int lout) { return (lin == 3 || lsh == 3 || lout == 3) ? 1 : 2; }

inline const KernelSet* find_mode_instance(int lin, int lsh, int lout, int mode) {
    using Fn = const KernelSet* (*)(int, int);
    static const Fn fns[3][4] = {
        {instances_m1_l0, instances_m1_l1, instances_m1_l2, instances_m1_l3},
        {instances_m2_l0, instances_m2_l1, instances_m2_l2, instances_m2_l3},
        {instances_m3_l0, instances_m3_l1, instances_m3_l2, instances_m3_l3},
    };
    if (mode < 1 || mode > 3 || lin < 0 || lin > 3) return nullptr;
    return fns[mode - 1][lin](lsh, lout);
}

inline const KernelSet* find_instance(int lin, int lsh, int lout, int vec) {
    using Fn = const KernelSet* (*)(int, int);
    static const Fn fns[4][4] = {
        {instances_l0_s0, instances_l0_s1, instances_l0_s2, instances_l0_s3},
        {instances_l1_s0, instances_l1_s1, instances_l1_s2, instances_l1_s3},
        {instances_l2_s0, instances_l2_s1, instances_l2_s2, instances_l2_s3},
        {instances_l3_s0, instances_l3_s1, instances_l3_s2, instances_l3_s3},
    };
    if (lin < 0 || lin > 3 || lsh < 0 || lsh > 3) return nullptr;
    return fns[lin][lsh](lout, vec);
}

// Double backward (natural-parity summed outputs): receiver pass, sender pass
// and r epilogue of one (L_in, L_sh, L_out) at one channel width.
struct DblParams;
struct DblKernelSet {
    int lin, lsh, lout, vec, tile_c, g;
    // recv: receiver CSR and senders; send: sender CSR and receivers
    cudaError_t (*run)(const DblParams& recv, const DblParams& send, cudaStream_t);
};

// Defined in eqc_dbl_l<L_in>.cu.
const DblKernelSet* dbl_instances_l0(int lsh, int lout);
const DblKernelSet* dbl_instances_l1(int lsh, int lout);
const DblKernelSet* dbl_instances_l2(int lsh, int lout);
const DblKernelSet* dbl_instances_l3(int lsh, int lout);

inline const DblKernelSet* find_dbl_instance(int lin, int lsh, int lout) {
    using Fn = const DblKernelSet* (*)(int, int);
    static const Fn fns[4] = {dbl_instances_l0, dbl_instances_l1, dbl_instances_l2, dbl_instances_l3};
    if (lin < 0 || lin > 3) return nullptr;
    return fns[lin](lsh, lout);
}

// Node-local channel-diagonal product (summed or per-path outputs) of one
// (L_u, L_v, L_out) at one channel width.
struct NpParams;
struct NpKernelSet {
    int lin, lsh, lout, vec, mode;
    cudaError_t (*fwd)(const NpParams&, cudaStream_t);
    cudaError_t (*bwd)(const NpParams&, cudaStream_t);
};

// Defined in eqc_np_l<L_u>.cu.
const NpKernelSet* np_instances_l0(int lv, int lout, bool per_path);
const NpKernelSet* np_instances_l1(int lv, int lout, bool per_path);
const NpKernelSet* np_instances_l2(int lv, int lout, bool per_path);
const NpKernelSet* np_instances_l3(int lv, int lout, bool per_path);

inline const NpKernelSet* find_np_instance(int lu, int lv, int lout, int mode) {
    using Fn = const NpKernelSet* (*)(int, int, bool);
    static const Fn fns[4] = {np_instances_l0, np_instances_l1, np_instances_l2, np_instances_l3};
    if (lu < 0 || lu > 3 || (mode != 0 && mode != 2)) return nullptr;
    return fns[lu](lv, lout, mode == 2);
}

// Harmonics-only kernels (depend on L_sh only); defined in eqc_api.cu.
cudaError_t launch_dr_epilogue(int lsh, const float* gy_part, int T, const float* r, float* dr, int E,
                               cudaStream_t st);
cudaError_t launch_sh(int lsh, const float* r, float* Y, int E, cudaStream_t st);

}  // namespace eqc

// Test-only build of the forward kernel whose row-staging waits cannot
// complete (not part of libeqconv; tests/test_gpu_wait_timeout.py loads it).
//
// Every stage fill here expects 16 bytes more than its copies carry, so no
// stage's phase ever completes, and the wait limit is cut to 2 ms.  The
// kernel must give up on the first wait, set status bit 4, wait (bounded) for
// the copies it still has in flight and return: the same code as the
// library's forward, with only these two constants changed.
#define EQC_WAIT_LIMIT_NS 2000000ull
#define EQC_TEST_FILL_DEFICIT 16

#include <cuda_runtime.h>

#include "../eqc_launch.cuh"

namespace eqc {
void count_launch() {}
}  // namespace eqc

using ProbeCfg = eqc::Cfg<1, 1, 1, 2>;   // irreps 0e+1o -> 0e+1o, L_sh = 1, 64-channel tiles

extern "C" __attribute__((visibility("default"))) int eqc_probe_forward_short_fill(
    const int* recv_ptr, const int* recv_perm, const int* senders, int N, int E, int C, const float* x,
    const float* r, const float* w, float* y, unsigned* status, void* stream) {
    eqc::FwdParams prm{x, r, w, y, recv_ptr, recv_perm, senders, N, C, E, 0, N, 0, status};
    const int tiles = (C + ProbeCfg::TILE_C - 1) / ProbeCfg::TILE_C;
    const cudaError_t e = eqc::Launch<ProbeCfg>::fwd(prm, tiles, 1, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? 0 : (int)e;
}

extern "C" __attribute__((visibility("default"))) int eqc_probe_paths() { return ProbeCfg::NP; }

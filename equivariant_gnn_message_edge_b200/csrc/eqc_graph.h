// Edge layout builder (host entry points; kernels in eqc_graph.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>

namespace eqc {

size_t graph_workspace_bytes(int N, int E);

cudaError_t graph_build(int N, int E, const int* senders, const int* receivers, int* recv_ptr, int* recv_perm,
                        int* send_ptr, int* send_perm, void* ws, unsigned* status, cudaStream_t st);

// Size of the library's fixed scratch array for graph_build_noalloc.
constexpr size_t kGraphScratchBytes = size_t(8) << 20;

// graph_build with scratch taken from the fixed array (no allocation);
// *too_large is set, and nothing is launched, when (N, E) needs more scratch.
cudaError_t graph_build_noalloc(int N, int E, const int* senders, const int* receivers, int* recv_ptr,
                                int* recv_perm, int* send_ptr, int* send_perm, unsigned* status, cudaStream_t st,
                                bool* too_large);

}  // namespace eqc

// Edge layout builder (host entry points; kernels in eqc_graph.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>

namespace eqc {

size_t graph_workspace_bytes(int N, int E);

cudaError_t graph_build(int N, int E, const int* senders, const int* receivers, int* recv_ptr, int* recv_perm,
                        int* send_ptr, int* send_perm, void* ws, unsigned* status, cudaStream_t st);

}  // namespace eqc

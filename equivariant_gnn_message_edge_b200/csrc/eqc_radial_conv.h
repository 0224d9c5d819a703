// Host interface of the convolution with on-chip radial weights (no device code).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>

namespace eqc {
namespace radial {

struct RadFwdArgs {
    const float* x;          // [N][D_in][C]
    const float* r;          // [E][3]
    const int* recv_ptr;
    const int* recv_perm;
    const int* senders;
    const int* receivers;
    const float* W1;         // [NB][64]
    const float* W2;         // [64][64]
    const float* W3;         // [64][P*C]
    int NB;
    float rc;
    float* y;                // [N][D_out][C] of the plan (summed or per-path layout)
    bool per_path;           // the plan's output layout
    void* workspace;
    size_t workspace_bytes;
    int N, E, C;
    unsigned* status;
};

struct RadBwdArgs {
    const float* x;          // [N][D_in][C]
    const float* r;          // [E][3]
    const float* gy;         // [N][D_out][C] of the plan (summed or per-path layout)
    const int* send_ptr;
    const int* send_perm;
    const int* senders;
    const int* receivers;
    const float* W1;
    const float* W2;
    const float* W3;
    int NB;
    float rc;
    float* dx;               // [N][D_in][C]
    float* dr;               // [E][3]
    float* gW1;              // [NB][64]
    float* gW2;              // [64][64]
    float* gW3;              // [64][P*C]
    bool per_path;
    void* workspace;
    size_t workspace_bytes;
    int N, E, C;
    unsigned* status;
};

struct RadConvSet {
    int lin, lsh, lout;
    int P, D_pp;             // paths; rows of the per-path layout
    size_t (*fwd_workspace)(int N, int E, int C, bool per_path);
    cudaError_t (*fwd)(const RadFwdArgs&, cudaStream_t);
    size_t (*bwd_workspace)(int N, int E, int C);
    cudaError_t (*bwd)(const RadBwdArgs&, cudaStream_t);
};

// The compiled (L_in, L_sh, L_out) combinations (natural-parity prefixes);
// nullptr for others.
const RadConvSet* find_radial_conv(int lin, int lsh, int lout);

}  // namespace radial
}  // namespace eqc

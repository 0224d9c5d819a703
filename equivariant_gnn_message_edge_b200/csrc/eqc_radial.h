// Host interface of the on-chip radial weights (no device code).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstddef>

namespace eqc {
namespace radial {

constexpr int kMaxBasisHost = 16;   // Bessel functions (eqc_radial.cuh kMaxBasis)

// Pieces of the caller's workspace (all 256-byte aligned):
//   a_hi, a_lo  [PC][64] fp16   W3^T split into fp16 pairs, scaled by 2^s_W3
//   inv_scale   [1]             2^-s_W3
//   h_hi, h_lo  [E][64]  fp16   h2 of every edge (or position) split, scaled per row
//   uscale      [E]             u(d) 2^-(s_W3 + s_h2)
//   zscale      [E]             2^-(s_W3 + s_h2)
//   rec, ids    [E]             per-position records of the fused kernels
struct Workspace {
    __half* a_hi;
    __half* a_lo;
    float* inv_scale;
    __half* h_hi;
    __half* h_lo;
    float* uscale;
    float* zscale;
    float4* rec;     // [E] (r_e, uscale) by position
    int2* ids;       // [E] (gathered node, own node) by position
    size_t bytes;
};

Workspace carve(void* ws, int E, int PC);
size_t workspace_bytes(int E, int PC);

// W3 split (one CTA) and the hidden layers of every edge, in the order of
// `perm` (position k holds edge perm[k]; perm == nullptr: edge order):
// H = split(h2 * 2^s), uscale = u(d) 2^-(s_W3 + s), so w = (W3^T H^T) * uscale;
// zscale = 2^-(s_W3 + s).  hmax (may be null; zeroed by the caller) receives
// max |h2| as float bits.  With `gathered` and `own` (edge arrays), rec and
// ids receive each position's (r, uscale) and (gathered[e], own[e]).
cudaError_t prepare(const Workspace& ws, const float* r, const int* perm, int E, const float* W1, const float* W2,
                    const float* W3, int NB, float rc, int PC, cudaStream_t st, unsigned* hmax = nullptr,
                    const int* gathered = nullptr, const int* own = nullptr);

// w [E][PC] from a prepared workspace (edge order), on the tensor cores.
cudaError_t weights(const Workspace& ws, int E, int PC, float* w, unsigned* status, cudaStream_t st);

}  // namespace radial
}  // namespace eqc

/*
 * eqconv.h - C ABI of libeqconv, the sm_100a (NVIDIA B200) implementation of
 * the E(3)-equivariant message-passing convolution of MACE-style interatomic
 * potentials.
 *
 * The operation (e3j: an Efficient and Open-Source Backend for Euclidean
 * Equivariant Operations on GPU and TPU, abstract and Table 1; FlashCart: Fast
 * Cartesian Tensor Products for Equivariant Interatomic Potentials, App. B,
 * §4 and App. D):
 *
 *   y[i, l3 m3, c] = sum_{e: recv(e) = i} sum_{p = (l1, l2, l3)} w[e, p, c]
 *                    sum_{m1, m2} C_p[m1, m2, m3] x[send(e), l1 m1, c] Y_{l2 m2}(r_e / |r_e|)
 *
 * with C_p the orthonormal real-basis Clebsch-Gordan coupling of path p
 * (Condon-Shortley phase, first nonzero entry positive) and Y the real
 * spherical harmonics, component-normalised (sum_m Y_lm^2 = 2l+1), z polar,
 * m > 0 ~ cos(m phi), m < 0 ~ sin(|m| phi).  Paths are the admissible
 * (l1, l2, l3): |l1 - l2| <= l3 <= l1 + l2 and natural parity, ordered by
 * (l1, l2, l3); paths that land on the same l3 are summed (by default: see
 * EQCONV_OUT_ALL_PARITY and EQCONV_OUT_PER_PATH for both-parity outputs and
 * per-path output blocks).
 *
 * Besides the forward and the backward the library has the double backward
 * (eqconv_double_backward, the VJP of the backward, for training on forces)
 * and the node-local channel-diagonal product of two node features
 * (eqconv_node_product*, one step of the correlation ladder).
 *
 * Layout (FlashCart App. D, Figure D1: rank blocks, then components, then
 * channels): every tensor is fp32, row-major, channels innermost.
 *   x      [N][D_in][C]      D_in  = (L_in + 1)^2
 *   y, gy  [N][D_out][C]     D_out = (L_out + 1)^2
 *   w, dw  [E][P][C]
 *   r, dr  [E][3]            edge vectors (the op depends on r / |r| only)
 *   senders, receivers [E]   int32
 *
 * Supported: irreps_in / irreps_out are natural-parity prefixes "0e+1o+2e+3o"
 * cut at L_in / L_out; L_in, L_sh, L_out <= 3; 4 <= C <= 4096, C % 4 == 0;
 * N, E < 2^31.  All device pointers must be 16-byte aligned.
 *
 * Memory and streams: every tensor and workspace is caller-owned device
 * memory (e.g. PyTorch tensors).  The plan owns its coupling tables and one
 * device status word (allocated at plan creation on the current device).  All
 * device work is enqueued on the given stream; no call synchronises the host
 * except eqconv_get_device_error.  Outputs are fully overwritten.
 *
 * Errors: every call returns an eqconv status; nothing throws across the ABI.
 * Out-of-range sender/receiver indices never cause out-of-bounds accesses:
 * the kernels skip such edges and set the plan's device status word, which
 * eqconv_get_device_error reports as EQCONV_ERR_DEVICE_CHECK.
 */
#ifndef EQCONV_H
#define EQCONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EQCONV_API __attribute__((visibility("default")))
#else
#define EQCONV_API
#endif

/* ABI-identical to cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* eqconv_stream_t;

enum {
    EQCONV_OK = 0,
    EQCONV_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, bad irreps */
    EQCONV_ERR_UNSUPPORTED = 2,   /* L > 3, C % 4 != 0, non-prefix irreps, no paths */
    EQCONV_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
    EQCONV_ERR_WORKSPACE = 4,     /* workspace null or smaller than required */
    EQCONV_ERR_DEVICE_CHECK = 5   /* a kernel saw an out-of-range index (see above) */
};

/* flags for eqconv_backward */
#define EQCONV_DETERMINISTIC 1u   /* sender-ordered pass, no atomics: bitwise run-to-run identical */

typedef struct eqconv_plan_s* eqconv_plan_t;

/* Edge layout.  The caller fills N, E, senders and receivers and provides the
 * four output arrays; eqconv_graph_build fills them (FlashCart, arXiv
 * 2610.06409, §4 and App. D: the forward runs over receiver-sorted edges so
 * that each program sums a receiver's incoming edges locally; the
 * deterministic VJP walks the edges in sender order so that each sender's
 * input gradient is summed by one program):
 *   recv_ptr[N+1]  = [0, cumsum(in-degree)]    recv_perm[E] = stable argsort(receivers)
 *   send_ptr[N+1]  = [0, cumsum(out-degree)]   send_perm[E] = stable argsort(senders)
 * All device pointers, caller-owned; the struct itself is read on the host. */
typedef struct eqconv_graph_s {
    int32_t N, E;
    const int32_t* senders;
    const int32_t* receivers;
    int32_t* recv_ptr;
    int32_t* recv_perm;
    int32_t* send_ptr;
    int32_t* send_perm;
} eqconv_graph_t;

/* Plan: parses the irreps, enumerates the paths, builds the real CG tables
 * (Racah formula, evaluated at compile time of the library) and selects the
 * kernel instance.  Host only, not hot.  *out receives the handle. */
EQCONV_API int eqconv_plan_create(eqconv_plan_t* out, const char* irreps_in, int L_sh,
                       const char* irreps_out, int C);

/* Output variants (bits of out_mode in eqconv_plan_create_ex).
 * FlashCart (arXiv 2610.06409), App. B: a path may also join irreps whose
 * parities multiply to the opposite of (-1)^l3 (odd l1 + l2 + l3: the
 * antisymmetric couplings, such as 1 x 1 -> 1, the cross product); App. D:
 * the channel-diagonal product may keep every path's output or sum the paths
 * that land on the same irrep.
 *   EQCONV_OUT_ALL_PARITY: outputs of both parities.  irreps_out must then be
 *     the both-parity prefix "0e+1o+1e+2e+2o+3o+3e" up to L_out (for each
 *     l >= 1 the natural-parity irrep first; 0o is absent: no path from
 *     natural-parity inputs reaches it), D_out = 2 (L_out+1)^2 - 1, and the
 *     odd paths feed the second block of each l.  Their coupling is the
 *     imaginary part of the real-basis CG sum (eqconv_cg_table).
 *   EQCONV_OUT_PER_PATH: no summation over paths.  Every path p writes its
 *     own block of 2 l3 + 1 rows, in path order, starting at row
 *     eqconv_plan_path_rows()[p]; D_out = sum over paths of (2 l3 + 1) (the
 *     "mid" irreps that MACE feeds to its next linear layer).  irreps_out
 *     still names the allowed output irreps as a natural-parity prefix (or
 *     with EQCONV_OUT_ALL_PARITY, a both-parity prefix) and only selects
 *     paths.  gy has the same per-path layout; dx, dw and dr are as usual.
 * Both bits may be combined.  The variants exist for L_sh and L_out in 1..3
 * (L_in 0..3) with one channel width per plan (1 where an l = 3 block is
 * present, else 2); other combinations return EQCONV_ERR_UNSUPPORTED. */
#define EQCONV_OUT_ALL_PARITY 1u
#define EQCONV_OUT_PER_PATH 2u

/* eqconv_plan_create with an output variant (out_mode: 0 or the bits above;
 * 0 is eqconv_plan_create). */
EQCONV_API int eqconv_plan_create_ex(eqconv_plan_t* out, const char* irreps_in, int L_sh,
                                     const char* irreps_out, int C, unsigned out_mode);

/* First output row of every path (P ints): l3^2 for natural-parity summed
 * outputs, the block of the path's (l3, parity) for EQCONV_OUT_ALL_PARITY,
 * the path's own block for EQCONV_OUT_PER_PATH. */
EQCONV_API int eqconv_plan_path_rows(eqconv_plan_t plan, int* out_rows);

/* Channel vector width of the forward / backward kernels (1, 2 or 4 channels
 * per lane, i.e. channel tiles of 32, 64 or 128 channels; width 1 exists only
 * for plans with an l = 3 block and falls back to 2 otherwise).  Defaults
 * (measured best on B200 at C = 128): 2 for the forward; for the backward 4
 * (deterministic, C >= 128) or 2 (atomic), and 1 for both modes when the plan
 * has an l = 3 block.  bwd_vec sets both backward modes.  A tuning knob;
 * results agree within rounding across widths (deterministic mode stays
 * bitwise reproducible for a fixed width). */
EQCONV_API int eqconv_plan_set_vec(eqconv_plan_t plan, int fwd_vec, int bwd_vec);

/* L2 budget (bytes) of one gather band.  The forward and the atomic backward
 * gather sender rows x[s], the deterministic backward gathers receiver rows
 * gy[i], about 45 times per row.  When N x (rows gathered) x (channel tile)
 * x 4 B exceeds the budget, the op runs as B launches over consecutive ranges
 * of the gathered node index, each touching only that range's rows, so they
 * stay in L2; y (or deterministic dx) is written by the first band and
 * accumulated by the next ones in fixed order.  Default (no call): 40 MiB
 * for the atomic backward (rows every SM reads stay in B200's L2 up to about
 * that size) and no banding for the forward and the deterministic backward,
 * which measured faster unbanded; a call sets the budget of all three, and 0
 * disables banding.  A tuning knob: results agree within rounding for any
 * budget, and deterministic mode is bitwise reproducible for a fixed budget. */
EQCONV_API int eqconv_plan_set_gather_budget(eqconv_plan_t plan, size_t bytes);

/* Sizes of the plan; paths_l1l2l3 (3*P ints, may be NULL) receives the paths. */
EQCONV_API int eqconv_plan_info(eqconv_plan_t plan, int* P, int* D_in, int* D_sh, int* D_out,
                     int* paths_l1l2l3);

/* Host only, no device needed.  The natural-parity paths of (irreps_in, L_sh,
 * irreps_out) in kernel order: *P receives the count and paths_l1l2l3 (room
 * for max_paths triples, may be NULL) the (l1, l2, l3) triples. */
EQCONV_API int eqconv_enumerate_paths(const char* irreps_in, int L_sh, const char* irreps_out,
                                      int* P, int* paths_l1l2l3, int max_paths);

/* Host only.  eqconv_enumerate_paths for an output variant (out_mode as in
 * eqconv_plan_create_ex): also gives every path's first output row
 * (out_rows, room for max_paths ints, may be NULL) and the output row count
 * (*D_out, may be NULL).  Does not check that kernels exist for the variant. */
EQCONV_API int eqconv_enumerate_paths_ex(const char* irreps_in, int L_sh, const char* irreps_out,
                                         unsigned out_mode, int* P, int* paths_l1l2l3, int* out_rows,
                                         int* D_out, int max_paths);

/* Host only, no device needed.  The real-basis CG tensor the kernels use for
 * the path (l1, l2, l3), fp64 row-major [2l1+1][2l2+1][2l3+1]: the real part
 * of the basis-change sum for even l1 + l2 + l3, its imaginary part for odd
 * (both-parity outputs).  out_len must be at least that size.
 * EQCONV_ERR_UNSUPPORTED for triples outside the triangle rule or l > 3. */
EQCONV_API int eqconv_cg_table(int l1, int l2, int l3, double* out, int out_len);

/* Device workspace bytes needed by eqconv_graph_build for (N, E). */
EQCONV_API size_t eqconv_graph_workspace_bytes(int N, int E);

/* Builds recv_ptr/recv_perm/send_ptr/send_perm on `stream` (stable LSD radix
 * sort + histogram + exclusive scan; bit-exact with a stable argsort): the
 * receiver-sorted and sender-sorted edge orders of FlashCart §4 / App. D.
 * N, E, senders and receivers are read from *g (host struct, device arrays);
 * the workspace is caller-owned device memory of at least
 * eqconv_graph_workspace_bytes(N, E) bytes (EQCONV_ERR_WORKSPACE otherwise).
 * Out-of-range senders/receivers set the device status word and are counted
 * nowhere (the outputs are then unspecified but in-bounds). */
EQCONV_API int eqconv_graph_build(eqconv_plan_t plan, const eqconv_graph_t* g, void* workspace,
                       size_t workspace_bytes, eqconv_stream_t stream);

/* Same result as eqconv_graph_build, for callers that cannot allocate device
 * memory: a plugin running inside another program's simulation step where
 * the host program owns every device allocation, or code that must not call
 * cudaMalloc because cudaMalloc can block the device.  It takes no workspace
 * and allocates nothing.  Its scratch is a fixed 8 MiB device array inside
 * the library, which every GPU that loads the library holds until the
 * process exits.  (The pages have no counterpart to this entry point.)
 *   - Limit: eqconv_graph_workspace_bytes(N, E) must be <= 8 MiB (about
 *     16.5 B per edge + 4 B per node; e.g. E <= 480k edges at N <= 100k).
 *     Larger graphs return EQCONV_ERR_WORKSPACE and launch nothing;
 *     eqconv_last_error then states the bytes needed.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is cached per device together
 *     with the ID of the context it belongs to: after cudaDeviceReset the
 *     next call sees a new context and looks the address up again.
 *   - Every call shares the one array: calls that overlap on the GPU (on two
 *     streams, or from two threads) race and corrupt each other's result.
 *     The scratch keeps the last call's contents; each call clears what it
 *     needs zeroed itself. */
EQCONV_API int eqconv_graph_build_noalloc(eqconv_plan_t plan, const eqconv_graph_t* g,
                                          eqconv_stream_t stream);

/* Forward: y [N][D_out][C] by the formula at the top of this file (e3j,
 * arXiv 2609.35099, abstract and Table 1: the convolution of MACE-style
 * potentials; FlashCart, arXiv 2610.06409, App. B for the paths and §4 /
 * App. D for the scheme: receiver-sorted, one program per receiver and
 * channel tile summing its incoming edges locally and storing each output
 * once, no atomics and no per-edge message tensor).  One fused kernel launch
 * (more when gather bands are set); deterministic.  x, w and y must be
 * 16-byte aligned; y is overwritten.  `flags` is reserved (pass 0). */
EQCONV_API int eqconv_forward(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x,
                   const float* r, const float* w, float* y, unsigned flags,
                   eqconv_stream_t stream);

/* Device workspace bytes needed by eqconv_backward in either mode (0 when C
 * fits one channel tile of both modes: the dr reduction is then done
 * in-kernel; otherwise per-tile partials of dr's harmonic gradient). */
EQCONV_API size_t eqconv_backward_workspace_bytes(eqconv_plan_t plan, int E);

/* Backward (vector-Jacobian product) given gy [N][D_out][C]: writes
 *   dx[j, l1 m1, c] = sum_{e: send(e)=j} sum_p w[e,p,c] sum_{m2,m3} C_p Y_{l2 m2}(r_e) gy[recv(e), l3 m3, c]
 *   dw[e, p, c]     = sum_{m1,m2,m3} C_p x[send(e), l1 m1, c] Y_{l2 m2}(r_e) gy[recv(e), l3 m3, c]
 *   dr[e]           = (dY(r_e/|r_e|)/dr_e)^T gY[e],
 *                     gY[e, l2 m2] = sum_c sum_{p with this l2} w[e,p,c] sum_{m1,m3} C_p x gy
 * (FlashCart, arXiv 2610.06409, §2: forces are the gradient of the energy
 * with respect to positions, so dr carries them; §4 and App. D: the VJP's
 * shared input gradient dx is accumulated either with atomic adds in
 * receiver order or, in sender order, deterministically; weight gradients
 * are stored directly).
 * flags & EQCONV_DETERMINISTIC: one pass over the sender CSR, dx summed in
 * registers, no atomics, bitwise reproducible; otherwise one pass over the
 * receiver CSR with dx accumulated by atomic adds (dx is zeroed by the
 * library first).  The workspace (eqconv_backward_workspace_bytes) is needed
 * only when C spans several channel tiles.  All outputs are overwritten. */
EQCONV_API int eqconv_backward(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x,
                    const float* r, const float* w, const float* gy, float* dx, float* dw,
                    float* dr, void* workspace, size_t workspace_bytes, unsigned flags,
                    eqconv_stream_t stream);

/* Device workspace bytes eqconv_double_backward needs for E edges (the
 * per-channel-tile partials of two harmonic-gradient vectors, [E][T][2 G]
 * fp32 with G = (L_sh+1)^2 - 1); 0 for plans without a double backward. */
EQCONV_API size_t eqconv_double_backward_workspace_bytes(eqconv_plan_t plan, int E);

/* Double backward: the VJP of eqconv_backward, for training on forces
 * (FlashCart, arXiv 2610.06409, §2 and §3 / App. C: the VJP-of-VJP of a
 * weighted bilinear product follows from bilinearity; App. D: it sums
 * receiver contributions to the incoming-gradient derivative).
 * Given the inputs of eqconv_backward (x, r, w, gy) and cotangents
 * ga [N][D_in][C] of dx, gb [E][P][C] of dw and gq [E][3] of dr, writes the
 * gradient of S = <ga, dx> + <gb, dw> + <gq, dr> with respect to every input:
 *   g_x  [N][D_in][C]  = sum over out-edges of  gb_p A_p(Y)^T gy_i + w_p A_p(rho)^T gy_i
 *   g_w  [E][P][C]     = ga_s . A_p(Y)^T gy_i + x_s . A_p(rho)^T gy_i
 *   g_gy [N][D_out][C] = sum over in-edges of  w_p (A_p(Y) ga_s + A_p(rho) x_s) + gb_p A_p(Y) x_s
 *   g_r  [E][3]        = (dY/dr)^T gYv + H(r; gY1) gq
 * with rho = (dY/dr) gq, A_p(v) = sum_m2 C_p[., m2, .] v[l2 m2], gYv the
 * harmonic gradient of (ga, w) plus that of (x, gb), gY1 that of (x, w), and
 * H the Hessian of the harmonics.  Zero-length edges contribute no rho and
 * no g_r.  Deterministic (bitwise reproducible): three launches on
 * `stream` (a receiver pass, a sender pass and a per-edge epilogue), no
 * atomics.  All outputs are overwritten.
 *   - Plans made with an output variant (out_mode != 0) return
 *     EQCONV_ERR_UNSUPPORTED.
 *   - Pointers as in eqconv_backward (16-byte aligned rows); the workspace
 *     must hold eqconv_double_backward_workspace_bytes(plan, E) bytes. */
EQCONV_API int eqconv_double_backward(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x,
                                      const float* r, const float* w, const float* gy, const float* ga,
                                      const float* gb, const float* gq, float* g_x, float* g_w, float* g_gy,
                                      float* g_r, void* workspace, size_t workspace_bytes,
                                      eqconv_stream_t stream);

/* ---- Node-local channel-diagonal product ----------------------------------
 * FlashCart (arXiv 2610.06409) §5, App. B and App. D: the correlation ladder
 * builds higher-order features by repeated pairwise products at each atom;
 * each step couples same-index channels of two node features along the
 * admissible paths and keeps every path's output (a learned linear map mixes
 * paths and channels afterwards) or sums weighted paths.
 *   y[i, o3(p)+m3, c] = sum_p w[p,c] sum_{m1,m2} C_p[m1,m2,m3] u[i, l1 m1, c] v[i, l2 m2, c]
 * u [N][D_u][C] (irreps_u a natural-parity prefix), v [N][(L_v+1)^2][C]
 * (degrees 0..L_v, natural parity, like the harmonics of the convolution),
 * w [P][C] per-path, per-channel weights (NULL: all ones), y [N][D_out][C].
 * Paths, their order, the CG tables and the output layouts (summed, or
 * EQCONV_OUT_PER_PATH) are exactly those of a convolution plan with
 * L_sh = L_v; eqconv_plan_info / eqconv_plan_path_rows describe them.
 * Both-parity outputs are not offered for this op (out_mode 0 or
 * EQCONV_OUT_PER_PATH).  A node-product plan is not a convolution plan: the
 * convolution entry points reject it with EQCONV_ERR_INVALID_ARG. */
EQCONV_API int eqconv_node_product_plan_create(eqconv_plan_t* out, const char* irreps_u, int L_v,
                                               const char* irreps_out, int C, unsigned out_mode);

/* y = the product above, on `stream`; one launch.  Rows 16-byte aligned. */
EQCONV_API int eqconv_node_product(eqconv_plan_t plan, int N, const float* u, const float* v,
                                   const float* w, float* y, eqconv_stream_t stream);

/* Device workspace bytes eqconv_node_product_backward needs when dw is
 * requested (per-warp partials of dw, [warps][P][C] fp32). */
EQCONV_API size_t eqconv_node_product_workspace_bytes(eqconv_plan_t plan, int N);

/* Backward given gy [N][D_out][C]:
 *   du[i, l1 m1, c] = sum_p w[p,c] sum_{m2,m3} C_p v[i, l2 m2, c] gy[i, o3+m3, c]
 *   dv[i, l2 m2, c] = sum_p w[p,c] sum_{m1,m3} C_p u[i, l1 m1, c] gy[i, o3+m3, c]
 *   dw[p, c]        = sum_i sum C_p u v gy          (dw may be NULL: not computed)
 * Deterministic: each warp sums dw over a fixed node set and a second launch
 * adds the warps' partials in order.  All outputs are overwritten. */
EQCONV_API int eqconv_node_product_backward(eqconv_plan_t plan, int N, const float* u, const float* v,
                                            const float* w, const float* gy, float* du, float* dv,
                                            float* dw, void* workspace, size_t workspace_bytes,
                                            eqconv_stream_t stream);

/* ---- Symmetric contraction, correlation order 2 ---------------------------
 * e3j (arXiv 2609.35099), abstract and Table 3: MACE(a)'s product basis has
 * correlation order 2; FlashCart (arXiv 2610.06409) §5 / App. B: the
 * correlation ladder of channel-diagonal products of an atom's own
 * features, weighted per path, channel and element.  For A [N][(L_A+1)^2][C]
 * (irreps_A a natural-parity prefix) and species [N] (int32, 0..S-1):
 *   B[i, L M, c] = W1[z_i, L, c] A[i, L M, c]                          (L <= min(L_A, L_out))
 *                + sum_q W2[z_i, q, c] sum_{m1,m2} C_q[m1,m2,M] A[i,l1 m1,c] A[i,l2 m2,c]
 * with q = (l1, l2, L) over l1 <= l2 <= L_A, L <= L_out, the triangle rule
 * and l1 + l2 + L even, ordered by (l1, l2, L) (eqconv_plan_info gives them:
 * P = their count, D_in = (L_A+1)^2, D_out = (L_out+1)^2).
 * W1 [S][min(L_A, L_out)+1][C], W2 [S][P][C], B [N][D_out][C], fp32.
 * L_A, L_out <= 3; 1 <= S <= 16; C % 4 == 0.  A symmetric-contraction plan
 * is not a convolution plan.  Out-of-range species set the status word (bit
 * 1); those nodes get B = 0. */
EQCONV_API int eqconv_symmetric_contraction_plan_create(eqconv_plan_t* out, const char* irreps_A,
                                                        const char* irreps_out, int C, int n_species);

/* B = the contraction above; one launch on `stream`.  Pointers 16-byte aligned. */
EQCONV_API int eqconv_symmetric_contraction(eqconv_plan_t plan, int N, const float* A, const int32_t* species,
                                            const float* W1, const float* W2, float* B, eqconv_stream_t stream);

/* Device workspace bytes eqconv_symmetric_contraction_backward needs (the
 * per-warp weight-gradient partials). */
EQCONV_API size_t eqconv_symmetric_contraction_workspace_bytes(eqconv_plan_t plan, int N);

/* Backward given gB [N][D_out][C]:
 *   dA = W1 gB + sum_q W2 (C_q A_l2 gB on block l1 + C_q A_l1 gB on block l2)
 *   dW1[s, L, c] = sum over nodes of species s of A_L . gB_L
 *   dW2[s, q, c] = sum over nodes of species s of C_q A A gB
 * Deterministic: each warp sums its fixed node set per species in shared
 * memory, a second launch adds the warps' partials in order.  All outputs
 * overwritten. */
EQCONV_API int eqconv_symmetric_contraction_backward(eqconv_plan_t plan, int N, const float* A, const int32_t* species,
                                                     const float* W1, const float* W2, const float* gB, float* dA,
                                                     float* dW1, float* dW2, void* workspace, size_t workspace_bytes,
                                                     eqconv_stream_t stream);

/* ---- Radial weights from edge lengths ------------------------------------
 * FlashCart (arXiv 2610.06409) App. B: a radial envelope makes every edge's
 * contribution vanish smoothly at the cutoff; App. E: the weights vanish with
 * their first two derivatives there.  e3j (arXiv 2609.35099) Table 3: 8
 * radial (Bessel) functions, 5 Angstrom cutoff.  With d = |r_e|,
 * x = min(d / r_cut, 1) and no biases:
 *   b_n(d)     = sqrt(2 / r_cut) sin(n pi d / r_cut) / max(d, 1e-12)   n = 1..n_basis
 *   u(d)       = 1 - 28 x^6 + 48 x^7 - 21 x^8
 *   w[e, p, c] = u(d) * sum_k h2[k] W3[k][p*C + c],
 *   h2 = silu(silu(b W1) W2),   silu(z) = z / (1 + exp(-z))
 * W1 [n_basis][64], W2 [64][64], W3 [64][P*C] fp32 row-major (hidden width
 * EQCONV_RADIAL_HIDDEN); 1 <= n_basis <= 16; C % 32 == 0.  The last layer
 * runs on the tensor cores with every operand split into two scaled fp16
 * halves (about 22 bits of each operand kept; fp32 accumulation).
 * The workspace (eqconv_radial_workspace_bytes, 16-byte aligned) holds the
 * split W3, the edges' split h2 and per-edge factors; caller-owned. */
#define EQCONV_RADIAL_HIDDEN 64

EQCONV_API size_t eqconv_radial_workspace_bytes(eqconv_plan_t plan, int E);

/* w [E][P][C] of the formula above, written to memory (the unfused radial
 * path; eqconv_forward_radial keeps w on the chip instead).  Three launches
 * on `stream`: the W3 split, the hidden layers, the last layer. */
EQCONV_API int eqconv_radial_weights(eqconv_plan_t plan, int E, const float* r, const float* W1, const float* W2,
                                     const float* W3, int n_basis, float r_cut, float* w, void* workspace,
                                     size_t workspace_bytes, eqconv_stream_t stream);

/* Device workspace bytes eqconv_forward_radial needs for (N, E); 0 when the
 * plan has no fused radial path. */
EQCONV_API size_t eqconv_forward_radial_workspace_bytes(eqconv_plan_t plan, int N, int E);

/* The convolution's forward with w[e, p, c] produced on the chip from the
 * edge lengths by the radial MLP above (W1, W2, W3, n_basis, r_cut as in
 * eqconv_radial_weights): y = forward(x, r, w(|r|)) without w ever in
 * memory (e3j Table 3 / FlashCart App. B, App. E for the weights; FlashCart
 * §4 / App. D for the receiver-sorted scheme).  Plans: natural-parity
 * prefixes with (L_in, L_sh, L_out) = (1,1,1), (1,2,2), (2,2,2) or (3,3,3),
 * summed or EQCONV_OUT_PER_PATH layout, C % 32 == 0; others return
 * EQCONV_ERR_UNSUPPORTED.  Launches on `stream`: the W3 split, the hidden
 * layers (by receiver position), the fused kernel (one CTA per receiver
 * range, 32-channel slice and group of up to 12 paths: tensor-core last
 * layer into tensor memory, read there by one warp per path) and, for a
 * summed plan, the sum of the per-path blocks in path order.  Deterministic.
 * Out-of-range senders set the status word; the result is then unspecified
 * (reads stay in bounds).  The workspace
 * (eqconv_forward_radial_workspace_bytes) is caller-owned device memory. */
EQCONV_API int eqconv_forward_radial(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r,
                                     const float* W1, const float* W2, const float* W3, int n_basis, float r_cut,
                                     float* y, void* workspace, size_t workspace_bytes, eqconv_stream_t stream);

/* Device workspace bytes eqconv_backward_radial needs for (N, E); 0 when
 * the plan has no fused radial path. */
EQCONV_API size_t eqconv_backward_radial_workspace_bytes(eqconv_plan_t plan, int N, int E);

/* Backward of eqconv_forward_radial given gy (the plan's output layout):
 *   dx  [N][D_in][C]   as eqconv_backward's, with w = w(|r|)
 *   dr  [E][3]         (dY/dr)^T gY + (d/dd <dw, w(d)>) r / |r|: both routes
 *                      of the edge vector (FlashCart §2: forces are the
 *                      energy's gradient in the positions)
 *   gW1 [n_basis][64], gW2 [64][64], gW3 [64][P*C]: gradients of <gy, y>
 *                      with respect to the MLP weights
 * w and dw never exist in memory: w is recomputed on the tensor cores, the
 * sender-ordered pass (deterministic) keeps dw on the chip and feeds it to
 * two tensor-core contractions (sum over edges of (u h2) x dw for gW3; W3 .
 * dw per edge for the MLP's backward); a per-edge epilogue finishes the MLP
 * backward and dr; the weight gradients are summed in a fixed order.
 * Same plans and arguments as eqconv_forward_radial; outputs overwritten;
 * bitwise reproducible run to run.  The workspace
 * (eqconv_backward_radial_workspace_bytes) is caller-owned device memory. */
EQCONV_API int eqconv_backward_radial(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r,
                                      const float* W1, const float* W2, const float* W3, int n_basis, float r_cut,
                                      const float* gy, float* dx, float* dr, float* gW1, float* gW2, float* gW3,
                                      void* workspace, size_t workspace_bytes, eqconv_stream_t stream);

/* The spherical harmonics the kernels use, Y [E][(L_sh+1)^2] (a test hook
 * for the in-kernel harmonics; not on the hot path). */
EQCONV_API int eqconv_spherical_harmonics(eqconv_plan_t plan, int E, const float* r, float* Y,
                               eqconv_stream_t stream);

/* Synchronises `stream`, reads and clears the plan's device status word;
 * *status receives EQCONV_OK or EQCONV_ERR_DEVICE_CHECK (the return value
 * reports whether the query itself worked, so a failed synchronisation is
 * not mistaken for a device check).  Status bits: 1 an out-of-range node
 * index was skipped, 4 a bounded wait for a row copy gave up. */
EQCONV_API int eqconv_get_device_error(eqconv_plan_t plan, eqconv_stream_t stream, int* status);

EQCONV_API void eqconv_plan_destroy(eqconv_plan_t plan);

EQCONV_API const char* eqconv_status_string(int status);

/* Text of the last CUDA failure an entry point of the calling thread
 * reported as EQCONV_ERR_CUDA (where, error name, description).  Owned by the
 * library; valid until the thread's next failing call. */
EQCONV_API const char* eqconv_last_error(void);

/* Number of kernels this library has launched in this process (all devices). */
EQCONV_API unsigned long long eqconv_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* EQCONV_H */

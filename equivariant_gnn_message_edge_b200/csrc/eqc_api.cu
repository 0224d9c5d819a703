// C ABI of libeqconv (declarations and contracts in include/eqconv.h).
//
// The plan validates the irreps, enumerates the natural-parity paths
// (FlashCart, arXiv 2610.06409, App. B: triangle rule, natural parity) and
// selects the compiled kernel instance; forward / backward validate their
// arguments and enqueue the fused kernels of eqc_conv.cuh on the caller's
// stream.  Nothing here allocates per call.
#include <cuda_runtime.h>

#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <cctype>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <utility>
#include <vector>

#include "eqc_conv.cuh"
#include "eqc_dbl.cuh"
#include "eqc_nodeprod.cuh"
#include "eqc_dispatch.h"
#include "eqc_graph.h"
#include "eqc_radial.h"
#include "eqc_radial_conv.h"
#include "eqc_symc.cuh"
#include "eqc_symc.h"
#include "eqconv.h"

namespace eqc {

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Last CUDA failure seen by an entry point of this thread (for diagnostics).
static thread_local char g_last_error[256] = "no error";
static void note_error(const char* where, cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

template <int LSH>
static cudaError_t dr_epi(const float* gy_part, int T, const float* r, float* dr, int E, cudaStream_t st) {
    if (E <= 0) return cudaSuccess;
    eqconv_dr_epilogue<LSH><<<(E + 255) / 256, 256, 0, st>>>(gy_part, T, r, dr, E);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dr_epilogue(int lsh, const float* gy_part, int T, const float* r, float* dr, int E,
                               cudaStream_t st) {
    switch (lsh) {
        case 0: return dr_epi<0>(gy_part, T, r, dr, E, st);
        case 1: return dr_epi<1>(gy_part, T, r, dr, E, st);
        case 2: return dr_epi<2>(gy_part, T, r, dr, E, st);
        case 3: return dr_epi<3>(gy_part, T, r, dr, E, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int LSH>
static cudaError_t sh_k(const float* r, float* Y, int E, cudaStream_t st) {
    if (E <= 0) return cudaSuccess;
    eqconv_sh_kernel<LSH><<<(E + 255) / 256, 256, 0, st>>>(r, Y, E);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_sh(int lsh, const float* r, float* Y, int E, cudaStream_t st) {
    switch (lsh) {
        case 0: return sh_k<0>(r, Y, E, st);
        case 1: return sh_k<1>(r, Y, E, st);
        case 2: return sh_k<2>(r, Y, E, st);
        case 3: return sh_k<3>(r, Y, E, st);
        default: return cudaErrorInvalidValue;
    }
}

__global__ void k_zero_f4(float4* p, int64_t n4) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n4) p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace eqc

struct eqconv_plan_s {
    int lin, lsh, lout, C;
    int fwd_vec, det_vec, atomic_vec;
    size_t gather_budget;   // bytes of gathered rows one band may touch (0: one band)
    bool budget_set;        // false: per-mode defaults (bands for the atomic backward only)
    int mode;               // output variant bits (eqc::kModeAllParity, eqc::kModePerPath)
    int P, D_in, D_sh, D_out;
    int paths[eqc::kMaxPaths][3];
    int path_rows[eqc::kMaxPaths];
    int device;
    unsigned* d_status;
    const eqc::KernelSet* fwd_ks;
    const eqc::KernelSet* det_ks;      // deterministic backward
    const eqc::KernelSet* atomic_ks;   // atomic backward
    const eqc::DblKernelSet* dbl_ks;   // double backward (summed natural-parity outputs only)
    bool node_product;                 // a node-local product plan (no convolution)
    const eqc::NpKernelSet* np_ks;     // node-local product
    const eqc::SymKernelSet* symc_ks;  // symmetric contraction (then node_product is true too)
    int n_species;
};

namespace {

// Irreps string -> list of (l, parity +1/-1); "1x" multiplicities and spaces
// are accepted.  False if malformed.
bool parse_irreps(const char* s, std::vector<std::pair<int, int>>& out) {
    out.clear();
    if (!s) return false;
    std::string t;
    for (const char* c = s; *c; ++c)
        if (!std::isspace((unsigned char)*c)) t.push_back(*c);
    if (t.empty()) return false;
    size_t i = 0;
    while (i <= t.size()) {
        size_t j = t.find('+', i);
        if (j == std::string::npos) j = t.size();
        std::string tok = t.substr(i, j - i);
        if (tok.size() >= 2 && tok[0] == '1' && tok[1] == 'x') tok = tok.substr(2);
        if (tok.size() < 2) return false;
        const char par = tok.back();
        if (par != 'e' && par != 'o') return false;
        const std::string num = tok.substr(0, tok.size() - 1);
        if (num.empty() || num.size() > 2) return false;
        for (char ch : num)
            if (!std::isdigit((unsigned char)ch)) return false;
        out.emplace_back(std::stoi(num), par == 'e' ? 1 : -1);
        if (j == t.size()) break;
        i = j + 1;
    }
    return true;
}

// The canonical irreps list of degree 0..L: natural parity (0e, 1o, 2e, ...)
// or both parities (0e, 1o, 1e, 2e, 2o, 3o, 3e, ...).
std::vector<std::pair<int, int>> prefix_irreps(int L, bool all_parity) {
    std::vector<std::pair<int, int>> v;
    for (int l = 0; l <= L; ++l) {
        const int nat = (l % 2 == 0) ? 1 : -1;
        v.emplace_back(l, nat);
        if (all_parity && l > 0) v.emplace_back(l, -nat);
    }
    return v;
}

// L when `s` is the canonical prefix 0..L (natural or both parities); -1 if
// malformed, -2 if well formed but not such a prefix (or L > 3).
int parse_prefix(const char* s, bool all_parity) {
    std::vector<std::pair<int, int>> v;
    if (!parse_irreps(s, v)) return -1;
    for (int L = 0; L <= eqc::kMaxL; ++L)
        if (v == prefix_irreps(L, all_parity)) return L;
    return -2;
}

int parse_natural_prefix(const char* s) { return parse_prefix(s, false); }

// Validates (irreps_in, L_sh, irreps_out, out_mode) and enumerates the paths.
int plan_paths(const char* irreps_in, int L_sh, const char* irreps_out, unsigned out_mode, int& lin, int& lout,
               eqc::PathList& PL) {
    if (out_mode & ~(EQCONV_OUT_ALL_PARITY | EQCONV_OUT_PER_PATH)) return EQCONV_ERR_INVALID_ARG;
    const int mode = (int)out_mode;
    lin = parse_natural_prefix(irreps_in);
    lout = parse_prefix(irreps_out, (mode & eqc::kModeAllParity) != 0);
    if (lin == -1 || lout == -1 || L_sh < 0) return EQCONV_ERR_INVALID_ARG;
    if (lin == -2 || lout == -2 || L_sh > eqc::kMaxL) return EQCONV_ERR_UNSUPPORTED;
    PL = eqc::make_paths(lin, L_sh, lout, mode);
    if (PL.n == 0) return EQCONV_ERR_UNSUPPORTED;
    return EQCONV_OK;
}

// Channel vector widths measured best on B200 at C = 128: 64-channel tiles for
// the forward and the atomic backward (their gathered rows stay in L2 and more
// warps fit), 128-channel tiles for the deterministic backward (fewer
// coupling-matrix builds per edge).  With an l = 3 block the backward's
// unrolled per-edge code outgrows the instruction cache; 32-channel tiles
// halve it and measured fastest for both backward modes.
int default_fwd_vec(int) { return 2; }
int default_det_vec(int C, bool l3) { return l3 ? 1 : (C >= 128 ? 4 : 2); }
int default_atomic_vec(bool l3) { return l3 ? 1 : 2; }

int tiles_for(int C, int tile_c) { return (C + tile_c - 1) / tile_c; }

// L2 budget of one gather band.  Rows gathered by every SM stay in L2 on B200
// while their set is about 40 MB (151 MB of x at lmax 2, C = 128 missed on
// about half the gathers).  Measured on B200 (lmax 2, C = 128): bands cut the
// DRAM bytes of every pass, but only the atomic backward gets faster (its dx
// atomics stay in L2); the forward breaks even and the deterministic backward
// slows down (each band gives a warp few edges to pipeline and dx is re-read),
// so by default only the atomic backward is banded.
constexpr size_t kDefaultGatherBudget = size_t(40) << 20;

// Number of bands so that one band's gathered slice (rows of D components x
// the channel tile) fits the budget.
int bands_for(eqconv_plan_t plan, int N, int D, int tile_c, bool atomic_bwd) {
    const size_t budget = plan->budget_set ? plan->gather_budget : (atomic_bwd ? kDefaultGatherBudget : 0);
    if (budget == 0 || N <= 1) return 1;
    const size_t slice = (size_t)N * (size_t)D * (size_t)(tile_c < plan->C ? tile_c : plan->C) * sizeof(float);
    size_t b = (slice + budget - 1) / budget;
    if (b < 1) b = 1;
    if (b > 64) b = 64;
    if (b > (size_t)N) b = (size_t)N;
    return (int)b;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device(eqconv_plan_t plan) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return EQCONV_ERR_CUDA;
    return dev == plan->device ? EQCONV_OK : EQCONV_ERR_INVALID_ARG;
}

int check_graph(const eqconv_graph_t* g) {
    if (!g || g->N < 0 || g->E < 0) return EQCONV_ERR_INVALID_ARG;
    if (!g->recv_ptr || !g->send_ptr) return EQCONV_ERR_INVALID_ARG;
    if (g->E > 0 && (!g->senders || !g->receivers || !g->recv_perm || !g->send_perm)) return EQCONV_ERR_INVALID_ARG;
    return EQCONV_OK;
}

int cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return EQCONV_OK;
    eqc::note_error(where, e);
    return EQCONV_ERR_CUDA;
}

}  // namespace

extern "C" {

int eqconv_plan_create(eqconv_plan_t* out, const char* irreps_in, int L_sh, const char* irreps_out, int C) {
    return eqconv_plan_create_ex(out, irreps_in, L_sh, irreps_out, C, 0u);
}

namespace {
int create_plan(eqconv_plan_t* out, const char* irreps_in, int L_sh, const char* irreps_out, int C,
                unsigned out_mode, bool node_product);
}

int eqconv_plan_create_ex(eqconv_plan_t* out, const char* irreps_in, int L_sh, const char* irreps_out, int C,
                          unsigned out_mode) {
    return create_plan(out, irreps_in, L_sh, irreps_out, C, out_mode, false);
}

int eqconv_node_product_plan_create(eqconv_plan_t* out, const char* irreps_u, int L_v, const char* irreps_out, int C,
                                    unsigned out_mode) {
    return create_plan(out, irreps_u, L_v, irreps_out, C, out_mode, true);
}

}  // extern "C"

namespace {
int create_plan(eqconv_plan_t* out, const char* irreps_in, int L_sh, const char* irreps_out, int C,
                unsigned out_mode, bool node_product) {
    if (!out) return EQCONV_ERR_INVALID_ARG;
    *out = nullptr;
    int lin = 0, lout = 0;
    eqc::PathList PL{};
    const int rc = plan_paths(irreps_in, L_sh, irreps_out, out_mode, lin, lout, PL);
    if (rc != EQCONV_OK) return rc;
    if (C <= 0) return EQCONV_ERR_INVALID_ARG;
    if (C % 4 != 0 || C < 4 || C > 4096) return EQCONV_ERR_UNSUPPORTED;
    const int mode = (int)out_mode;
    eqconv_plan_s* p = new (std::nothrow) eqconv_plan_s();
    if (!p) return EQCONV_ERR_CUDA;
    p->lin = lin;
    p->lsh = L_sh;
    p->lout = lout;
    p->C = C;
    p->mode = mode;
    p->P = PL.n;
    p->D_in = (lin + 1) * (lin + 1);
    p->D_sh = (L_sh + 1) * (L_sh + 1);
    p->D_out = PL.dout;
    for (int i = 0; i < PL.n; ++i) {
        p->paths[i][0] = PL.l1[i];
        p->paths[i][1] = PL.l2[i];
        p->paths[i][2] = PL.l3[i];
        p->path_rows[i] = PL.o3[i];
    }
    p->gather_budget = 0;
    p->budget_set = false;
    if (mode == 0) {
        p->fwd_vec = default_fwd_vec(C);
        const bool l3 = lin == 3 || L_sh == 3 || lout == 3;
        p->det_vec = default_det_vec(C, l3);
        p->atomic_vec = default_atomic_vec(l3);
        p->fwd_ks = eqc::find_instance(lin, L_sh, lout, p->fwd_vec);
        p->det_ks = eqc::find_instance(lin, L_sh, lout, p->det_vec);
        p->atomic_ks = eqc::find_instance(lin, L_sh, lout, p->atomic_vec);
    } else {
        p->fwd_vec = p->det_vec = p->atomic_vec = eqc::mode_vec(lin, L_sh, lout);
        p->fwd_ks = p->det_ks = p->atomic_ks = eqc::find_mode_instance(lin, L_sh, lout, mode);
    }
    p->dbl_ks = mode == 0 ? eqc::find_dbl_instance(lin, L_sh, lout) : nullptr;
    p->node_product = node_product;
    p->np_ks = node_product ? eqc::find_np_instance(lin, L_sh, lout, mode) : nullptr;
    const bool ok = node_product ? p->np_ks != nullptr : (p->fwd_ks && p->det_ks && p->atomic_ks);
    if (!ok) {
        delete p;
        return EQCONV_ERR_UNSUPPORTED;
    }
    if (cudaGetDevice(&p->device) != cudaSuccess || cudaMalloc(&p->d_status, sizeof(unsigned)) != cudaSuccess) {
        delete p;
        return EQCONV_ERR_CUDA;
    }
    if (cudaMemset(p->d_status, 0, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(p->d_status);
        delete p;
        return EQCONV_ERR_CUDA;
    }
    *out = p;
    return EQCONV_OK;
}
}  // namespace

extern "C" {

int eqconv_plan_set_vec(eqconv_plan_t plan, int fwd_vec, int bwd_vec) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    if (plan->node_product) return EQCONV_ERR_UNSUPPORTED;
    const auto ok = [](int v) { return v == 1 || v == 2 || v == 4; };
    if (!ok(fwd_vec) || !ok(bwd_vec)) return EQCONV_ERR_UNSUPPORTED;
    if (plan->mode != 0) {
        // output variants are compiled at one width
        const int v = eqc::mode_vec(plan->lin, plan->lsh, plan->lout);
        return (fwd_vec == v && bwd_vec == v) ? EQCONV_OK : EQCONV_ERR_UNSUPPORTED;
    }
    const eqc::KernelSet* f = eqc::find_instance(plan->lin, plan->lsh, plan->lout, fwd_vec);
    const eqc::KernelSet* b = eqc::find_instance(plan->lin, plan->lsh, plan->lout, bwd_vec);
    if (!f || !b) return EQCONV_ERR_UNSUPPORTED;
    plan->fwd_vec = fwd_vec;
    plan->det_vec = plan->atomic_vec = bwd_vec;
    plan->fwd_ks = f;
    plan->det_ks = plan->atomic_ks = b;
    return EQCONV_OK;
}

int eqconv_plan_set_gather_budget(eqconv_plan_t plan, size_t bytes) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    plan->gather_budget = bytes;
    plan->budget_set = true;
    return EQCONV_OK;
}

int eqconv_plan_info(eqconv_plan_t plan, int* P, int* D_in, int* D_sh, int* D_out, int* paths_l1l2l3) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    if (P) *P = plan->P;
    if (D_in) *D_in = plan->D_in;
    if (D_sh) *D_sh = plan->D_sh;
    if (D_out) *D_out = plan->D_out;
    if (paths_l1l2l3)
        for (int i = 0; i < plan->P; ++i)
            for (int k = 0; k < 3; ++k) paths_l1l2l3[3 * i + k] = plan->paths[i][k];
    return EQCONV_OK;
}

int eqconv_plan_path_rows(eqconv_plan_t plan, int* out_rows) {
    if (!plan || !out_rows) return EQCONV_ERR_INVALID_ARG;
    for (int i = 0; i < plan->P; ++i) out_rows[i] = plan->path_rows[i];
    return EQCONV_OK;
}

int eqconv_enumerate_paths(const char* irreps_in, int L_sh, const char* irreps_out, int* P, int* paths_l1l2l3,
                           int max_paths) {
    return eqconv_enumerate_paths_ex(irreps_in, L_sh, irreps_out, 0u, P, paths_l1l2l3, nullptr, nullptr, max_paths);
}

int eqconv_enumerate_paths_ex(const char* irreps_in, int L_sh, const char* irreps_out, unsigned out_mode, int* P,
                              int* paths_l1l2l3, int* out_rows, int* D_out, int max_paths) {
    if (!P) return EQCONV_ERR_INVALID_ARG;
    int lin = 0, lout = 0;
    eqc::PathList PL{};
    const int rc = plan_paths(irreps_in, L_sh, irreps_out, out_mode, lin, lout, PL);
    if (rc == EQCONV_ERR_UNSUPPORTED && lin >= 0 && lout >= 0 && L_sh <= eqc::kMaxL && PL.n == 0) {
        *P = 0;   // well-formed, no admissible path
        if (D_out) *D_out = 0;
        return EQCONV_OK;
    }
    if (rc != EQCONV_OK) return rc;
    *P = PL.n;
    if (D_out) *D_out = PL.dout;
    if ((paths_l1l2l3 || out_rows) && max_paths < PL.n) return EQCONV_ERR_INVALID_ARG;
    for (int i = 0; i < PL.n; ++i) {
        if (paths_l1l2l3) {
            paths_l1l2l3[3 * i] = PL.l1[i];
            paths_l1l2l3[3 * i + 1] = PL.l2[i];
            paths_l1l2l3[3 * i + 2] = PL.l3[i];
        }
        if (out_rows) out_rows[i] = PL.o3[i];
    }
    return EQCONV_OK;
}

int eqconv_cg_table(int l1, int l2, int l3, double* out, int out_len) {
    if (!out) return EQCONV_ERR_INVALID_ARG;
    if (l1 < 0 || l2 < 0 || l3 < 0 || l1 > eqc::kMaxL || l2 > eqc::kMaxL || l3 > eqc::kMaxL)
        return EQCONV_ERR_UNSUPPORTED;
    if (l3 < eqc::iabs(l1 - l2) || l3 > l1 + l2) return EQCONV_ERR_UNSUPPORTED;
    const int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
    if (out_len < d1 * d2 * d3) return EQCONV_ERR_INVALID_ARG;
    const eqc::CG3 t = eqc::make_real_cg(l1, l2, l3);
    for (int a = 0; a < d1; ++a)
        for (int b = 0; b < d2; ++b)
            for (int c = 0; c < d3; ++c) out[(a * d2 + b) * d3 + c] = t.v[a][b][c];
    return EQCONV_OK;
}

size_t eqconv_graph_workspace_bytes(int N, int E) {
    if (N < 0 || E < 0) return 0;
    return eqc::graph_workspace_bytes(N, E);
}

int eqconv_graph_build(eqconv_plan_t plan, const eqconv_graph_t* g, void* workspace, size_t workspace_bytes,
                       eqconv_stream_t stream) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    const size_t need = eqc::graph_workspace_bytes(g->N, g->E);
    if (!workspace || workspace_bytes < need) return EQCONV_ERR_WORKSPACE;
    return cuda_status(eqc::graph_build(g->N, g->E, g->senders, g->receivers, g->recv_ptr, g->recv_perm, g->send_ptr,
                                        g->send_perm, workspace, plan->d_status, (cudaStream_t)stream),
                       "graph_build");
}

int eqconv_graph_build_noalloc(eqconv_plan_t plan, const eqconv_graph_t* g, eqconv_stream_t stream) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    bool too_large = false;
    const cudaError_t err =
        eqc::graph_build_noalloc(g->N, g->E, g->senders, g->receivers, g->recv_ptr, g->recv_perm, g->send_ptr,
                                 g->send_perm, plan->d_status, (cudaStream_t)stream, &too_large);
    if (too_large) {
        snprintf(eqc::g_last_error, sizeof(eqc::g_last_error),
                 "graph_build_noalloc: N=%d, E=%d needs %zu bytes of scratch; the fixed scratch holds %zu",
                 g->N, g->E, eqc::graph_workspace_bytes(g->N, g->E), eqc::kGraphScratchBytes);
        return EQCONV_ERR_WORKSPACE;
    }
    return cuda_status(err, "graph_build_noalloc");
}

int eqconv_forward(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r, const float* w,
                   float* y, unsigned flags, eqconv_stream_t stream) {
    (void)flags;
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    if (plan->node_product) return EQCONV_ERR_INVALID_ARG;   // not a convolution plan
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    if (g->N == 0) return EQCONV_OK;
    if (!x || !y || (g->E > 0 && (!r || !w))) return EQCONV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(w)) return EQCONV_ERR_INVALID_ARG;
    eqc::FwdParams prm{x, r, w, y, g->recv_ptr, g->recv_perm, g->senders, g->N, plan->C, g->E, 0, g->N, 0,
                       plan->d_status};
    const int T = tiles_for(plan->C, plan->fwd_ks->tile_c);
    const int bands = bands_for(plan, g->N, plan->D_in, plan->fwd_ks->tile_c, false);
    return cuda_status(plan->fwd_ks->fwd(prm, T, bands, (cudaStream_t)stream), "forward");
}

static size_t bwd_ws_bytes(eqconv_plan_t plan, const eqc::KernelSet* ks, int E) {
    const int T = tiles_for(plan->C, ks->tile_c);
    const int G = plan->D_sh - 1;
    if (T == 1 || G == 0) return 0;
    return (size_t)E * T * G * sizeof(float);
}

size_t eqconv_backward_workspace_bytes(eqconv_plan_t plan, int E) {
    if (!plan || E < 0) return 0;
    const size_t a = bwd_ws_bytes(plan, plan->det_ks, E), b = bwd_ws_bytes(plan, plan->atomic_ks, E);
    return a > b ? a : b;
}

int eqconv_backward(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r, const float* w,
                    const float* gy, float* dx, float* dw, float* dr, void* workspace, size_t workspace_bytes,
                    unsigned flags, eqconv_stream_t stream) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    if (plan->node_product) return EQCONV_ERR_INVALID_ARG;   // not a convolution plan
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    if (g->N == 0) return EQCONV_OK;
    if (!x || !gy || !dx || (g->E > 0 && (!r || !w || !dw || !dr))) return EQCONV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gy) || !aligned16(dx) || !aligned16(w) || !aligned16(dw))
        return EQCONV_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    const bool det = (flags & EQCONV_DETERMINISTIC) != 0;
    const eqc::KernelSet* ks = det ? plan->det_ks : plan->atomic_ks;
    const int T = tiles_for(plan->C, ks->tile_c);
    const int G = plan->D_sh - 1;
    const bool fused = (T == 1) || (G == 0);
    const size_t need = bwd_ws_bytes(plan, ks, g->E);
    if (need > 0 && (!workspace || workspace_bytes < need)) return EQCONV_ERR_WORKSPACE;
    if (!det) {
        const int64_t n4 = (int64_t)g->N * plan->D_in * plan->C / 4;
        eqc::k_zero_f4<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(reinterpret_cast<float4*>(dx), n4);
        eqc::count_launch();
        const cudaError_t ze = cudaGetLastError();
        if (ze != cudaSuccess) return cuda_status(ze, "backward zero dx");
    }
    if (g->E == 0) {
        if (det) {
            const int64_t n4 = (int64_t)g->N * plan->D_in * plan->C / 4;
            eqc::k_zero_f4<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(reinterpret_cast<float4*>(dx), n4);
            eqc::count_launch();
            const cudaError_t ze = cudaGetLastError();
            if (ze != cudaSuccess) return cuda_status(ze, "backward zero dx");
        }
        return EQCONV_OK;
    }
    eqc::BwdParams prm{};
    prm.x = x;
    prm.r = r;
    prm.w = w;
    prm.gy = gy;
    prm.dx = dx;
    prm.dw = dw;
    prm.dr = dr;
    prm.gy_part = static_cast<float*>(workspace);
    prm.ptr = det ? g->send_ptr : g->recv_ptr;
    prm.perm = det ? g->send_perm : g->recv_perm;
    prm.other = det ? g->receivers : g->senders;
    prm.N = g->N;
    prm.C = plan->C;
    prm.T = T;
    prm.E = g->E;
    prm.status = plan->d_status;
    const int bands = bands_for(plan, g->N, det ? plan->D_out : plan->D_in, ks->tile_c, !det);
    cudaError_t err = ks->bwd(prm, det, fused, bands, st);
    if (err != cudaSuccess) return cuda_status(err, det ? "backward (deterministic)" : "backward (atomic)");
    if (!fused) err = eqc::launch_dr_epilogue(plan->lsh, prm.gy_part, T, r, dr, g->E, st);
    return cuda_status(err, "dr epilogue");
}

size_t eqconv_double_backward_workspace_bytes(eqconv_plan_t plan, int E) {
    if (!plan || E < 0 || !plan->dbl_ks) return 0;
    const int T = tiles_for(plan->C, plan->dbl_ks->tile_c);
    return (size_t)E * (size_t)T * 2u * (size_t)(plan->D_sh - 1) * sizeof(float);
}

int eqconv_double_backward(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r,
                           const float* w, const float* gy, const float* ga, const float* gb, const float* gq,
                           float* g_x, float* g_w, float* g_gy, float* g_r, void* workspace, size_t workspace_bytes,
                           eqconv_stream_t stream) {
    if (!plan) return EQCONV_ERR_INVALID_ARG;
    if (plan->node_product) return EQCONV_ERR_INVALID_ARG;   // not a convolution plan
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    if (!plan->dbl_ks) return EQCONV_ERR_UNSUPPORTED;
    if (g->N == 0) return EQCONV_OK;
    if (!x || !gy || !ga || !g_x || !g_gy) return EQCONV_ERR_INVALID_ARG;
    if (g->E > 0 && (!r || !w || !gb || !gq || !g_w || !g_r)) return EQCONV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gy) || !aligned16(ga) || !aligned16(g_x) || !aligned16(g_gy) ||
        !aligned16(w) || !aligned16(gb) || !aligned16(g_w))
        return EQCONV_ERR_INVALID_ARG;
    const size_t need = eqconv_double_backward_workspace_bytes(plan, g->E);
    if (need > 0 && (!workspace || workspace_bytes < need)) return EQCONV_ERR_WORKSPACE;
    eqc::DblParams prm{};
    prm.x = x;
    prm.a = ga;
    prm.r = r;
    prm.q = gq;
    prm.w = w;
    prm.b = gb;
    prm.gy = gy;
    prm.g_x = g_x;
    prm.g_w = g_w;
    prm.g_gy = g_gy;
    prm.g_r = g_r;
    prm.part = static_cast<float*>(workspace);
    prm.N = g->N;
    prm.C = plan->C;
    prm.T = tiles_for(plan->C, plan->dbl_ks->tile_c);
    prm.E = g->E;
    prm.status = plan->d_status;
    // the receiver pass walks the receiver CSR, the sender pass the sender CSR
    eqc::DblParams recv = prm, send = prm;
    recv.ptr = g->recv_ptr;
    recv.perm = g->recv_perm;
    recv.other = g->senders;
    send.ptr = g->send_ptr;
    send.perm = g->send_perm;
    send.other = g->receivers;
    return cuda_status(plan->dbl_ks->run(recv, send, (cudaStream_t)stream), "double backward");
}

int eqconv_symmetric_contraction_plan_create(eqconv_plan_t* out, const char* irreps_A, const char* irreps_out, int C,
                                             int n_species) {
    if (!out) return EQCONV_ERR_INVALID_ARG;
    *out = nullptr;
    const int la = parse_natural_prefix(irreps_A), lout = parse_natural_prefix(irreps_out);
    if (la == -1 || lout == -1 || C <= 0 || n_species < 1) return EQCONV_ERR_INVALID_ARG;
    if (la == -2 || lout == -2 || C % 4 != 0 || C > 4096 || n_species > eqc::kSymMaxSpecies)
        return EQCONV_ERR_UNSUPPORTED;
    const eqc::SymKernelSet* ks = eqc::find_symc(la, lout);
    if (!ks || ks->np == 0) return EQCONV_ERR_UNSUPPORTED;
    eqconv_plan_s* p = new (std::nothrow) eqconv_plan_s();
    if (!p) return EQCONV_ERR_CUDA;
    p->lin = la;
    p->lsh = la;
    p->lout = lout;
    p->C = C;
    p->mode = 0;
    p->P = ks->np;
    p->D_in = ks->d_a;
    p->D_sh = ks->d_a;
    p->D_out = ks->d_out;
    for (int i = 0; i < ks->np; ++i) {
        for (int k = 0; k < 3; ++k) p->paths[i][k] = ks->paths[i][k];
        p->path_rows[i] = ks->paths[i][2] * ks->paths[i][2];
    }
    p->node_product = true;   // not a convolution plan
    p->symc_ks = ks;
    p->n_species = n_species;
    if (cudaGetDevice(&p->device) != cudaSuccess || cudaMalloc(&p->d_status, sizeof(unsigned)) != cudaSuccess) {
        delete p;
        return EQCONV_ERR_CUDA;
    }
    if (cudaMemset(p->d_status, 0, sizeof(unsigned)) != cudaSuccess) {
        cudaFree(p->d_status);
        delete p;
        return EQCONV_ERR_CUDA;
    }
    *out = p;
    return EQCONV_OK;
}

int eqconv_symmetric_contraction(eqconv_plan_t plan, int N, const float* A, const int32_t* species, const float* W1,
                                 const float* W2, float* B, eqconv_stream_t stream) {
    if (!plan || N < 0) return EQCONV_ERR_INVALID_ARG;
    if (!plan->symc_ks) return EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    if (N == 0) return EQCONV_OK;
    if (!A || !species || !W1 || !W2 || !B || !aligned16(A) || !aligned16(B) || !aligned16(W1) || !aligned16(W2))
        return EQCONV_ERR_INVALID_ARG;
    eqc::SymParams prm{};
    prm.A = A;
    prm.species = species;
    prm.W1 = W1;
    prm.W2 = W2;
    prm.B = B;
    prm.N = N;
    prm.C = plan->C;
    prm.S = plan->n_species;
    prm.status = plan->d_status;
    return cuda_status(plan->symc_ks->fwd(prm, (cudaStream_t)stream), "symmetric contraction");
}

size_t eqconv_symmetric_contraction_workspace_bytes(eqconv_plan_t plan, int N) {
    if (!plan || !plan->symc_ks || N < 0) return 0;
    return plan->symc_ks->workspace(N, plan->C, plan->n_species);
}

int eqconv_symmetric_contraction_backward(eqconv_plan_t plan, int N, const float* A, const int32_t* species,
                                          const float* W1, const float* W2, const float* gB, float* dA, float* dW1,
                                          float* dW2, void* workspace, size_t workspace_bytes,
                                          eqconv_stream_t stream) {
    if (!plan || N < 0) return EQCONV_ERR_INVALID_ARG;
    if (!plan->symc_ks) return EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    if (!W1 || !W2 || !dW1 || !dW2) return EQCONV_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    if (N == 0) {
        const size_t s = (size_t)plan->n_species * plan->C * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dW1, 0, s * plan->symc_ks->l1n, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dW2, 0, s * plan->symc_ks->np, st);
        return cuda_status(e, "symmetric contraction backward, no nodes");
    }
    if (!A || !species || !gB || !dA || !aligned16(A) || !aligned16(gB) || !aligned16(dA) || !aligned16(W1) ||
        !aligned16(W2))
        return EQCONV_ERR_INVALID_ARG;
    const size_t need = plan->symc_ks->workspace(N, plan->C, plan->n_species);
    if (!workspace || workspace_bytes < need) return EQCONV_ERR_WORKSPACE;
    eqc::SymParams prm{};
    prm.A = A;
    prm.species = species;
    prm.W1 = W1;
    prm.W2 = W2;
    prm.gB = gB;
    prm.dA = dA;
    prm.dw_part = static_cast<float*>(workspace);
    prm.N = N;
    prm.C = plan->C;
    prm.S = plan->n_species;
    prm.status = plan->d_status;
    return cuda_status(plan->symc_ks->bwd(prm, dW1, dW2, st), "symmetric contraction backward");
}

size_t eqconv_node_product_workspace_bytes(eqconv_plan_t plan, int N) {
    if (!plan || N < 0 || !plan->np_ks) return 0;
    const int need = (N + eqc::kNpWarps - 1) / eqc::kNpWarps;
    const int blocks = need < 2 * 148 ? (need > 0 ? need : 1) : 2 * 148;
    return (size_t)blocks * eqc::kNpWarps * (size_t)plan->P * (size_t)plan->C * sizeof(float);
}

int eqconv_node_product(eqconv_plan_t plan, int N, const float* u, const float* v, const float* w, float* y,
                        eqconv_stream_t stream) {
    if (!plan || N < 0) return EQCONV_ERR_INVALID_ARG;
    if (!plan->np_ks) return plan->node_product ? EQCONV_ERR_UNSUPPORTED : EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    if (N == 0) return EQCONV_OK;
    if (!u || !v || !y || !aligned16(u) || !aligned16(v) || !aligned16(y) || (w && !aligned16(w)))
        return EQCONV_ERR_INVALID_ARG;
    eqc::NpParams prm{};
    prm.u = u;
    prm.v = v;
    prm.w = w;
    prm.y = y;
    prm.N = N;
    prm.C = plan->C;
    return cuda_status(plan->np_ks->fwd(prm, (cudaStream_t)stream), "node product");
}

int eqconv_node_product_backward(eqconv_plan_t plan, int N, const float* u, const float* v, const float* w,
                                 const float* gy, float* du, float* dv, float* dw, void* workspace,
                                 size_t workspace_bytes, eqconv_stream_t stream) {
    if (!plan || N < 0) return EQCONV_ERR_INVALID_ARG;
    if (!plan->np_ks) return plan->node_product ? EQCONV_ERR_UNSUPPORTED : EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    if (!u || !v || !gy || !du || !dv) return EQCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(v) || !aligned16(gy) || !aligned16(du) || !aligned16(dv) ||
        (w && !aligned16(w)) || (dw && !aligned16(dw)))
        return EQCONV_ERR_INVALID_ARG;
    const size_t need = dw ? eqconv_node_product_workspace_bytes(plan, N) : 0;
    if (need > 0 && (!workspace || workspace_bytes < need)) return EQCONV_ERR_WORKSPACE;
    eqc::NpParams prm{};
    prm.u = u;
    prm.v = v;
    prm.w = w;
    prm.gy = gy;
    prm.du = du;
    prm.dv = dv;
    prm.dw = dw;
    prm.dw_part = dw ? static_cast<float*>(workspace) : nullptr;
    prm.N = N;
    prm.C = plan->C;
    return cuda_status(plan->np_ks->bwd(prm, (cudaStream_t)stream), "node product backward");
}

size_t eqconv_radial_workspace_bytes(eqconv_plan_t plan, int E) {
    if (!plan || E < 0 || plan->node_product) return 0;
    return eqc::radial::workspace_bytes(E, plan->P * plan->C);
}

int eqconv_radial_weights(eqconv_plan_t plan, int E, const float* r, const float* W1, const float* W2,
                          const float* W3, int n_basis, float r_cut, float* w, void* workspace,
                          size_t workspace_bytes, eqconv_stream_t stream) {
    if (!plan || plan->node_product || E < 0) return EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    if (n_basis < 1 || n_basis > eqc::radial::kMaxBasisHost || !(r_cut > 0.f)) return EQCONV_ERR_INVALID_ARG;
    if (!W1 || !W2 || !W3 || (E > 0 && (!r || !w))) return EQCONV_ERR_INVALID_ARG;
    if (plan->C % 32 != 0) return EQCONV_ERR_UNSUPPORTED;
    const int PC = plan->P * plan->C;
    const size_t need = eqc::radial::workspace_bytes(E, PC);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return EQCONV_ERR_WORKSPACE;
    const cudaStream_t st = (cudaStream_t)stream;
    const eqc::radial::Workspace ws = eqc::radial::carve(workspace, E, PC);
    cudaError_t err = eqc::radial::prepare(ws, r, nullptr, E, W1, W2, W3, n_basis, r_cut, PC, st);
    if (err != cudaSuccess) return cuda_status(err, "radial weights (hidden layers)");
    return cuda_status(eqc::radial::weights(ws, E, PC, w, plan->d_status, st), "radial weights (last layer)");
}

static const eqc::radial::RadConvSet* radial_set(eqconv_plan_t plan) {
    if (!plan || plan->node_product || (plan->mode & eqc::kModeAllParity)) return nullptr;
    return eqc::radial::find_radial_conv(plan->lin, plan->lsh, plan->lout);
}

size_t eqconv_forward_radial_workspace_bytes(eqconv_plan_t plan, int N, int E) {
    const eqc::radial::RadConvSet* rs = radial_set(plan);
    if (!rs || N < 0 || E < 0) return 0;
    return rs->fwd_workspace(N, E, plan->C, (plan->mode & eqc::kModePerPath) != 0);
}

int eqconv_forward_radial(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r,
                          const float* W1, const float* W2, const float* W3, int n_basis, float r_cut, float* y,
                          void* workspace, size_t workspace_bytes, eqconv_stream_t stream) {
    if (!plan || plan->node_product) return EQCONV_ERR_INVALID_ARG;
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    const eqc::radial::RadConvSet* rs = radial_set(plan);
    if (!rs || plan->C % 32 != 0) return EQCONV_ERR_UNSUPPORTED;
    if (n_basis < 1 || n_basis > eqc::radial::kMaxBasisHost || !(r_cut > 0.f)) return EQCONV_ERR_INVALID_ARG;
    if (g->N == 0) return EQCONV_OK;
    if (!x || !y || !W1 || !W2 || !W3 || (g->E > 0 && !r)) return EQCONV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return EQCONV_ERR_INVALID_ARG;
    const bool per_path = (plan->mode & eqc::kModePerPath) != 0;
    const size_t need = rs->fwd_workspace(g->N, g->E, plan->C, per_path);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return EQCONV_ERR_WORKSPACE;
    eqc::radial::RadFwdArgs a{};
    a.x = x;
    a.r = r;
    a.recv_ptr = g->recv_ptr;
    a.recv_perm = g->recv_perm;
    a.senders = g->senders;
    a.receivers = g->receivers;
    a.W1 = W1;
    a.W2 = W2;
    a.W3 = W3;
    a.NB = n_basis;
    a.rc = r_cut;
    a.y = y;
    a.per_path = per_path;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.N = g->N;
    a.E = g->E;
    a.C = plan->C;
    a.status = plan->d_status;
    return cuda_status(rs->fwd(a, (cudaStream_t)stream), "forward (radial)");
}

size_t eqconv_backward_radial_workspace_bytes(eqconv_plan_t plan, int N, int E) {
    const eqc::radial::RadConvSet* rs = radial_set(plan);
    if (!rs || N < 0 || E < 0 || plan->C % 32 != 0) return 0;
    return rs->bwd_workspace(N, E, plan->C);
}

int eqconv_backward_radial(eqconv_plan_t plan, const eqconv_graph_t* g, const float* x, const float* r,
                           const float* W1, const float* W2, const float* W3, int n_basis, float r_cut,
                           const float* gy, float* dx, float* dr, float* gW1, float* gW2, float* gW3,
                           void* workspace, size_t workspace_bytes, eqconv_stream_t stream) {
    if (!plan || plan->node_product) return EQCONV_ERR_INVALID_ARG;
    int rc = check_graph(g);
    if (rc != EQCONV_OK) return rc;
    if ((rc = check_device(plan)) != EQCONV_OK) return rc;
    const eqc::radial::RadConvSet* rs = radial_set(plan);
    if (!rs || plan->C % 32 != 0) return EQCONV_ERR_UNSUPPORTED;
    if (n_basis < 1 || n_basis > eqc::radial::kMaxBasisHost || !(r_cut > 0.f)) return EQCONV_ERR_INVALID_ARG;
    if (!W1 || !W2 || !W3 || !gW1 || !gW2 || !gW3) return EQCONV_ERR_INVALID_ARG;
    if (g->N == 0) {
        const cudaStream_t st = (cudaStream_t)stream;
        cudaError_t e = cudaMemsetAsync(gW1, 0, (size_t)n_basis * 64 * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gW2, 0, (size_t)64 * 64 * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(gW3, 0, (size_t)64 * plan->P * plan->C * 4, st);
        return cuda_status(e, "backward (radial), no nodes");
    }
    if (!x || !gy || !dx || (g->E > 0 && (!r || !dr))) return EQCONV_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gy) || !aligned16(dx)) return EQCONV_ERR_INVALID_ARG;
    const size_t need = rs->bwd_workspace(g->N, g->E, plan->C);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return EQCONV_ERR_WORKSPACE;
    eqc::radial::RadBwdArgs a{};
    a.x = x;
    a.r = r;
    a.gy = gy;
    a.send_ptr = g->send_ptr;
    a.send_perm = g->send_perm;
    a.senders = g->senders;
    a.receivers = g->receivers;
    a.W1 = W1;
    a.W2 = W2;
    a.W3 = W3;
    a.NB = n_basis;
    a.rc = r_cut;
    a.dx = dx;
    a.dr = dr;
    a.gW1 = gW1;
    a.gW2 = gW2;
    a.gW3 = gW3;
    a.per_path = (plan->mode & eqc::kModePerPath) != 0;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.N = g->N;
    a.E = g->E;
    a.C = plan->C;
    a.status = plan->d_status;
    return cuda_status(rs->bwd(a, (cudaStream_t)stream), "backward (radial)");
}

int eqconv_spherical_harmonics(eqconv_plan_t plan, int E, const float* r, float* Y, eqconv_stream_t stream) {
    if (!plan || E < 0 || (E > 0 && (!r || !Y))) return EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    return cuda_status(eqc::launch_sh(plan->lsh, r, Y, E, (cudaStream_t)stream), "spherical harmonics");
}

int eqconv_get_device_error(eqconv_plan_t plan, eqconv_stream_t stream, int* status) {
    if (!plan || !status) return EQCONV_ERR_INVALID_ARG;
    int rc = check_device(plan);
    if (rc != EQCONV_OK) return rc;
    unsigned h = 0;
    const cudaError_t se = cudaStreamSynchronize((cudaStream_t)stream);
    if (se != cudaSuccess) return cuda_status(se, "get_device_error sync");
    if (cudaMemcpy(&h, plan->d_status, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
        return EQCONV_ERR_CUDA;
    if (h != 0 && cudaMemset(plan->d_status, 0, sizeof(unsigned)) != cudaSuccess) return EQCONV_ERR_CUDA;
    *status = h ? EQCONV_ERR_DEVICE_CHECK : EQCONV_OK;
    return EQCONV_OK;
}

void eqconv_plan_destroy(eqconv_plan_t plan) {
    if (!plan) return;
    int cur = -1;
    const bool switch_dev = cudaGetDevice(&cur) == cudaSuccess && cur != plan->device;
    if (switch_dev) cudaSetDevice(plan->device);
    cudaFree(plan->d_status);
    if (switch_dev) cudaSetDevice(cur);
    delete plan;
}

const char* eqconv_status_string(int status) {
    switch (status) {
        case EQCONV_OK: return "EQCONV_OK";
        case EQCONV_ERR_INVALID_ARG: return "EQCONV_ERR_INVALID_ARG: null/misaligned pointer, bad size or bad irreps";
        case EQCONV_ERR_UNSUPPORTED: return "EQCONV_ERR_UNSUPPORTED: L > 3, C % 4 != 0, non-prefix irreps or no path";
        case EQCONV_ERR_CUDA: return "EQCONV_ERR_CUDA: a CUDA call or kernel launch failed";
        case EQCONV_ERR_WORKSPACE: return "EQCONV_ERR_WORKSPACE: workspace missing or too small";
        case EQCONV_ERR_DEVICE_CHECK: return "EQCONV_ERR_DEVICE_CHECK: a kernel saw an out-of-range index";
        default: return "unknown eqconv status";
    }
}

unsigned long long eqconv_launch_count(void) { return eqc::g_launches.load(std::memory_order_relaxed); }

const char* eqconv_last_error(void) { return eqc::g_last_error; }

}  // extern "C"

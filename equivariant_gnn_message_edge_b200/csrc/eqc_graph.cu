// Edge layout builder: receiver and sender CSR offsets and stable permutations.
//
// FlashCart (arXiv 2610.06409) §4 / App. D: the forward keeps edges sorted by
// receiver and sums each receiver's incoming edges in one program; ordering
// edges by sender makes the sender-feature gradient deterministic.  For keys
// k[e] in [0, N):
//     ptr  = [0, cumsum(bincount(k))]        (histogram + exclusive scan)
//     perm = stable argsort(k)                (LSD radix sort, 8-bit digits)
// Integer work only; the result is bit-exact and independent of scheduling
// (integer atomics on counts, fixed-order ranks in the scatter).  No kernel
// waits on another block: every dependency is a kernel boundary.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "eqc_graph.h"

namespace eqc {

void count_launch();

namespace {

constexpr int kThreads = 256;
constexpr int kItems = 8;
constexpr int kTile = kThreads * kItems;  // 2048 keys per block
constexpr int kRadix = 256;

__global__ void k_zero_int(int* p, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) p[i] = 0;
}

__global__ void k_iota(int* p, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) p[i] = i;
}

// counts[key]++ for keys in range; others set status bit 2.  Lanes of a warp
// holding the same key add once (sorted keys would otherwise serialise on one
// counter).
__global__ void k_key_hist(const int* keys, int E, int N, int* counts, unsigned* status) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool inb = i < E;
    const int k = inb ? keys[i] : 0;
    const bool valid = inb && (unsigned)k < (unsigned)N;
    if (inb && !valid) atomicOr(status, 2u);
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? k : -1 - lane);
    if (valid && __ffs(peers) - 1 == lane) atomicAdd(&counts[k], __popc(peers));
}

// Block-level exclusive scan of kTile ints; writes block totals.
__global__ void k_scan_tiles(const int* in, int* out, int n, int* totals) {
    __shared__ int warp_sums[kThreads / 32];
    const int base = blockIdx.x * kTile + threadIdx.x * kItems;
    int v[kItems];
    int s = 0;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
        v[j] = (base + j < n) ? in[base + j] : 0;
        s += v[j];
    }
    // inclusive scan of per-thread sums within the warp
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    int warp_off = 0, block_total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        const int ws = warp_sums[w];
        if (w < warp) warp_off += ws;
        block_total += ws;
    }
    int run = warp_off + inc - s;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
        if (base + j < n) out[base + j] = run;
        run += v[j];
    }
    if (threadIdx.x == 0 && totals) totals[blockIdx.x] = block_total;
}

__global__ void k_add_tile_offsets(int* out, int n, const int* offsets) {
    const int base = blockIdx.x * kTile + threadIdx.x * kItems;
    const int add = offsets[blockIdx.x];
#pragma unroll
    for (int j = 0; j < kItems; ++j)
        if (base + j < n) out[base + j] += add;
}

// hist[d * ntiles + tile] = number of keys of the tile with digit d
__global__ void k_radix_hist(const int* keys, int E, int shift, int* hist, int ntiles) {
    __shared__ int h[kRadix];
    h[threadIdx.x] = 0;
    __syncthreads();
    const int base = blockIdx.x * kTile;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
        const int i = base + j * kThreads + threadIdx.x;
        if (i < E) atomicAdd(&h[((unsigned)keys[i] >> shift) & (kRadix - 1)], 1);
    }
    __syncthreads();
    hist[threadIdx.x * ntiles + blockIdx.x] = h[threadIdx.x];
}

// Stable scatter: items are ranked in index order within the tile (round by
// round, warp by warp, lane by lane), so equal digits keep their input order.
__global__ void k_radix_scatter(const int* keys_in, const int* vals_in, int* keys_out, int* vals_out, int E,
                                int shift, const int* offsets, int ntiles) {
    __shared__ int base_pos[kRadix];
    __shared__ int wcount[kThreads / 32][kRadix];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    base_pos[tid] = offsets[tid * ntiles + blockIdx.x];
    const unsigned lt_mask = (1u << lane) - 1u;
    const int tile0 = blockIdx.x * kTile;
    for (int j = 0; j < kItems; ++j) {
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) wcount[w][tid] = 0;
        __syncthreads();
        const int i = tile0 + j * kThreads + tid;
        const bool valid = i < E;
        int key = 0, val = 0, d = 0;
        if (valid) {
            key = keys_in[i];
            val = vals_in ? vals_in[i] : i;
            d = ((unsigned)key >> shift) & (kRadix - 1);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? d : (kRadix + lane));
        const int rank = __popc(peers & lt_mask);
        if (valid && rank == 0) wcount[warp][d] = __popc(peers);
        __syncthreads();
        if (valid) {
            int pos = base_pos[d] + rank;
            for (int w = 0; w < warp; ++w) pos += wcount[w][d];
            keys_out[pos] = key;
            vals_out[pos] = val;
        }
        __syncthreads();
        int tot = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) tot += wcount[w][tid];
        base_pos[tid] += tot;
        __syncthreads();
    }
}

inline int cdiv(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

size_t scan_aux_ints(int64_t n) {
    size_t s = 0;
    while (n > kTile) {
        n = cdiv(n, kTile);
        s += (size_t)n + 1;
    }
    return s + 1;
}

cudaError_t scan_exclusive(const int* in, int* out, int n, int* aux, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int nb = cdiv(n, kTile);
    if (nb == 1) {
        k_scan_tiles<<<1, kThreads, 0, st>>>(in, out, n, nullptr);
        count_launch();
        return cudaGetLastError();
    }
    int* totals = aux;
    int* totals_scanned = aux;  // scanned in place through the recursion below
    k_scan_tiles<<<nb, kThreads, 0, st>>>(in, out, n, totals);
    count_launch();
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    err = scan_exclusive(totals, totals_scanned, nb, aux + nb + 1, st);
    if (err != cudaSuccess) return err;
    k_add_tile_offsets<<<nb, kThreads, 0, st>>>(out, n, totals_scanned);
    count_launch();
    return cudaGetLastError();
}

int radix_passes(int N) {
    if (N <= 1) return 0;
    unsigned v = (unsigned)(N - 1);
    int bits = 0;
    while (v) {
        ++bits;
        v >>= 1;
    }
    return (bits + 7) / 8;
}

struct WsLayout {
    size_t counts, keys_a, vals_a, keys_b, vals_b, hist, aux, total;
};

WsLayout layout(int N, int E) {
    auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
    const int ntiles = cdiv(E > 0 ? E : 1, kTile);
    const size_t nhist = (size_t)kRadix * ntiles;
    const int64_t scan_n = (int64_t)(nhist > (size_t)N + 1 ? nhist : (size_t)N + 1);
    WsLayout L{};
    size_t o = 0;
    L.counts = o;  o += up(sizeof(int) * ((size_t)N + 1));
    L.keys_a = o;  o += up(sizeof(int) * (size_t)E);
    L.vals_a = o;  o += up(sizeof(int) * (size_t)E);
    L.keys_b = o;  o += up(sizeof(int) * (size_t)E);
    L.vals_b = o;  o += up(sizeof(int) * (size_t)E);
    L.hist = o;    o += up(sizeof(int) * nhist);
    L.aux = o;     o += up(sizeof(int) * scan_aux_ints(scan_n));
    L.total = o;
    return L;
}

// ptr[N+1], perm[E] for keys[E] in [0, N)
cudaError_t build_csr(const int* keys, int N, int E, int* ptr, int* perm, char* ws, unsigned* status,
                      cudaStream_t st) {
    const WsLayout L = layout(N, E);
    int* counts = reinterpret_cast<int*>(ws + L.counts);
    int* aux = reinterpret_cast<int*>(ws + L.aux);
    cudaError_t err;
    // ptr
    k_zero_int<<<cdiv((int64_t)N + 1, 256), 256, 0, st>>>(counts, (int64_t)N + 1);
    count_launch();
    if (E > 0) {
        k_key_hist<<<cdiv(E, 256), 256, 0, st>>>(keys, E, N, counts, status);
        count_launch();
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if ((err = scan_exclusive(counts, ptr, N + 1, aux, st)) != cudaSuccess) return err;
    if (E == 0) return cudaSuccess;
    // perm
    const int passes = radix_passes(N);
    if (passes == 0) {
        k_iota<<<cdiv(E, 256), 256, 0, st>>>(perm, E);
        count_launch();
        return cudaGetLastError();
    }
    const int ntiles = cdiv(E, kTile);
    int* hist = reinterpret_cast<int*>(ws + L.hist);
    int* ka = reinterpret_cast<int*>(ws + L.keys_a);
    int* va = reinterpret_cast<int*>(ws + L.vals_a);
    int* kb = reinterpret_cast<int*>(ws + L.keys_b);
    int* vb = reinterpret_cast<int*>(ws + L.vals_b);
    const int* kin = keys;
    const int* vin = nullptr;  // identity values on the first pass
    for (int p = 0; p < passes; ++p) {
        const int shift = 8 * p;
        int* kout = (p & 1) ? kb : ka;
        int* vout = (p == passes - 1) ? perm : ((p & 1) ? vb : va);
        k_radix_hist<<<ntiles, kThreads, 0, st>>>(kin, E, shift, hist, ntiles);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        if ((err = scan_exclusive(hist, hist, kRadix * ntiles, aux, st)) != cudaSuccess) return err;
        k_radix_scatter<<<ntiles, kThreads, 0, st>>>(kin, vin, kout, vout, E, shift, hist, ntiles);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        kin = kout;
        vin = vout;
    }
    return cudaSuccess;
}

}  // namespace

size_t graph_workspace_bytes(int N, int E) { return layout(N, E).total; }

cudaError_t graph_build(int N, int E, const int* senders, const int* receivers, int* recv_ptr, int* recv_perm,
                        int* send_ptr, int* send_perm, void* ws, unsigned* status, cudaStream_t st) {
    cudaError_t err = build_csr(receivers, N, E, recv_ptr, recv_perm, static_cast<char*>(ws), status, st);
    if (err != cudaSuccess) return err;
    return build_csr(senders, N, E, send_ptr, send_perm, static_cast<char*>(ws), status, st);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of graph_build.
//
// Some callers cannot allocate device memory: for example a plugin called
// inside another program's simulation step, where the host program owns all
// device memory, or code that must not call cudaMalloc because it blocks the
// device.  For them the radix-sort scratch lives in this fixed array, which
// every GPU that loads the library holds until the process exits.  Host code
// must not pass `g_graph_scratch` itself to a kernel: on the host it is only
// a stand-in symbol, not a device address.  Its device address is looked up
// once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_graph_scratch[kGraphScratchBytes];

// Unique ID of the calling thread's current CUDA context (cuCtxGetId through
// the runtime's driver entry points, so the library does not link libcuda);
// 0 when there is no current context or the driver does not offer the call.
static unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

cudaError_t graph_build_noalloc(int N, int E, const int* senders, const int* receivers, int* recv_ptr,
                                int* recv_perm, int* send_ptr, int* send_perm, unsigned* status, cudaStream_t st,
                                bool* too_large) {
    *too_large = false;
    if (graph_workspace_bytes(N, E) > kGraphScratchBytes) {
        *too_large = true;
        return cudaSuccess;
    }
    static std::mutex mu;
    static void* addr[64] = {};
    static unsigned long long ctx_id[64] = {};   // context the cached address belongs to (0: none)
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        // The address belongs to the device's current context: after
        // cudaDeviceReset the primary context is a new one and the array has
        // a new address, so the cache is keyed by the context's unique ID and
        // looked up again when it changes (or when no ID can be read).
        const unsigned long long id = current_context_id();
        if (!addr[dev] || id == 0 || id != ctx_id[dev]) {
            void* a = nullptr;
            err = cudaGetSymbolAddress(&a, g_graph_scratch);
            if (err != cudaSuccess) {
                addr[dev] = nullptr;
                ctx_id[dev] = 0;
                return err;
            }
            addr[dev] = a;
            ctx_id[dev] = current_context_id();   // the lookup made the device's context current
        }
        scratch = addr[dev];
    }
    // Every word of scratch that must start at zero (the key counts) is
    // zeroed inside build_csr on each call; histograms and sort buffers are
    // fully overwritten before they are read.
    return graph_build(N, E, senders, receivers, recv_ptr, recv_perm, send_ptr, send_perm, scratch, status, st);
}

}  // namespace eqc

// route_static.cu -- mono_route_static: the routing of mono_route for callers
// that cannot allocate device memory.
//
// Some callers never get to allocate: a plugin whose host framework owns all
// device memory and offers no allocator, a serving loop that forbids
// allocation after start-up because cudaMalloc can synchronise the device and
// fragment a pre-planned pool, or code that runs where no workspace was set
// aside.  For them the routing tables (block summaries, addresses, posting
// lists, overflow counts, statistics) live in one library-owned array in
// global memory instead of a caller workspace.  The caller still provides Q,
// K, the codebooks and sel.
//
// The array is a file-scope __device__ object: every GPU that loads this
// library holds kStaticRouteScratchBytes of it until the process exits.  Host
// code cannot use the array's name as a device address, so the first call on
// each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it; that first call should therefore be made
// before any stream capture begins.  Every call on a device shares the one
// array and leaves its tables there: calls that overlap on the GPU (different
// streams, or other threads) race with each other and must be serialised by
// the caller.  The statistics counters are cleared by every call; mono_stats
// with a NULL workspace reads them (and the overflow counts) back from here.
// The cached address does not survive cudaDeviceReset.
#include <mutex>

#include "internal.cuh"

namespace mono {
namespace {

constexpr size_t kStaticRouteScratchBytes = 16u << 20;  // 16 MiB

__device__ __align__(256) unsigned char g_route_scratch[kStaticRouteScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// the routing regions of plan `p`, packed from offset 0; returns the bytes they need
size_t route_layout(const Plan &p, Plan *rp) {
    const mono_config &c = p.cfg;
    const size_t bh = (size_t)c.B * c.H, nb = (size_t)p.nb;
    *rp = p;
    for (int r = 0; r < kRegN; ++r) { rp->off[r] = 0; rp->bytes[r] = 0; }
    const int regions[] = {kRegKbar, kRegAddr, kRegPostIds, kRegPostAddr, kRegPostRank, kRegOverflow, kRegCounters,
                           kRegWalkLog};
    const size_t sizes[] = {bh * nb * c.d * 4, bh * nb * 4, bh * nb * 4, bh * nb * 4, bh * nb * 4, bh * 4,
                            (size_t)kCntN * 8, (size_t)kWalkLogCap * 4};
    size_t off = 0;
    for (int i = 0; i < 8; ++i) {
        rp->off[regions[i]] = off;
        rp->bytes[regions[i]] = sizes[i];
        off = align256(off + sizes[i]);
    }
    rp->ws_bytes = off;
    return off;
}

int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MONO_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || !ptr) return MONO_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return MONO_OK;
}

}  // namespace

int route_static_tables(const Plan &p, void **base, Plan *rp) {
    if (route_layout(p, rp) > kStaticRouteScratchBytes) return MONO_ERR_SCRATCH;
    return scratch_address(base);
}

}  // namespace mono

using namespace mono;

extern "C" {

size_t mono_route_static_capacity(void) { return kStaticRouteScratchBytes; }

int mono_route_static(const mono_plan_t *plan, const void *Q, const void *K, const float *codebooks,
                      const int32_t *forced, int32_t *sel, void *stream) {
    if (!plan) return MONO_ERR_NULL;
    const Plan &p = plan->p;
    if (p.cfg.B == 0 || p.cfg.S == 0) return MONO_OK;
    if (!Q || !K || !codebooks || (p.cfg.R > 0 && !sel)) return MONO_ERR_NULL;
    if (((uintptr_t)Q | (uintptr_t)K | (uintptr_t)codebooks | (uintptr_t)sel) % 16) return MONO_ERR_ALIGN;
    if (forced && (uintptr_t)forced % 4) return MONO_ERR_ALIGN;
    Plan rp;
    void *scratch = nullptr;
    int st = route_static_tables(p, &scratch, &rp);
    if (st != MONO_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (launch_summaries(rp, K, codebooks, scratch, s) != cudaSuccess) return MONO_ERR_CUDA;
    if (launch_lists(rp, scratch, s) != cudaSuccess) return MONO_ERR_CUDA;
    if (launch_queries(rp, Q, codebooks, forced, sel, scratch, s, false) != cudaSuccess) return MONO_ERR_CUDA;
    return MONO_OK;
}

}  // extern "C"

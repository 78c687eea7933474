// internal.cuh -- plan, workspace layout and device helpers shared by the
// kernels of the mixer library (not part of the public C-ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mono.h"

namespace mono {

constexpr int kMaxD = 128;
constexpr int kMaxM = 8;
constexpr int kMaxC = 64;
constexpr int kMaxT = 32;
constexpr int kMaxE = 32;
constexpr int kMaxR = 16;
constexpr int kMaxNb = 8192;
constexpr int kRopeLo = 64;  // positions per low rotation table

// Device error codes (first one recorded wins; see mono_stats).
enum DevErr : unsigned {
    kDevErrBadSel = 1,       // attention got a sel id outside [0, t/Bs - L]
    kDevErrCandOverflow = 2, // probe candidate list exceeded its bound (never expected)
    kDevErrTimeout = 3,      // a bounded wait ran out
    kDevErrBadAddr = 4,      // an address outside [0, C^M)
    kDevErrSmemAlign = 5,    // dynamic shared memory not 1024-byte aligned (TMA tiles need it)
};

// Counters at the start of the counter region (uint64 each).  kCntWalks counts
// the query-heads whose probe left the fast path for the general walk (near
// ties in the staged top-T, or a stage with too many surviving prefixes); the
// first kWalkLogCap of them are logged by flat index in the walk-log region.
// The routing statistics are the first kCntStats counters (reset together), the error word after them.
enum Counter { kCntQueriesLtR = 0, kCntRemoteSel = 1, kCntForcedIgnored = 2, kCntWalks = 3, kCntStats = 4, kCntErr = 4,
               kCntN = 8 };
constexpr int kWalkLogCap = 4096;
constexpr int kRedirectMaxA = 65536;  // largest C^M of redirect-on-overflow lists (per-address counts in shared memory)

enum Region {
    kRegKbar = MONO_WS_KBAR,
    kRegAddr = MONO_WS_ADDR,
    kRegPostIds = MONO_WS_POST_IDS,
    kRegPostAddr = MONO_WS_POST_ADDR,
    kRegPostRank = MONO_WS_POST_RANK,
    kRegOverflow = MONO_WS_OVERFLOW,
    kRegQ = MONO_WS_Q,
    kRegK = MONO_WS_K,
    kRegV = MONO_WS_V,
    kRegSel = MONO_WS_SEL,
    kRegO = MONO_WS_O,
    kRegWalkLog = MONO_WS_WALK_LOG,
    kRegCounters = MONO_WS_NREGIONS,
    kRegRope,
    kRegPairCount,   // [B,H,nb] int32 queries selecting each block (fast attention)
    kRegPairStart,   // [B,H,nb+1] int32 exclusive scan of the counts
    kRegPairFill,    // [B,H,nb] int32 fill cursors
    kRegPairs,       // [B*H*S*R] int32 (t*R + r) grouped by block
    kRegPartO,       // [B*H*S*R, d] bf16 remote partial outputs
    kRegPartML,      // [B*H*S*R] float2 (max, sum) of remote partials
    kRegWork,        // [B*H, max_work] int4 (block, first pair, pair count, 0) work items of the remote kernel
    kRegNWork,       // [B*H] int32 number of work items
    kRegN
};

struct Plan {
    mono_config cfg;
    int nb;        // S / Bs
    long long A;   // C^M
    int es;        // bytes per stored element (4 or 2)
    bool fast;     // tensor-core attention applies
    bool gemm_tc;  // tensor-core projections apply
    int max_work;  // upper bound on remote work items per (b, h)
    size_t off[kRegN];
    size_t bytes[kRegN];
    size_t ws_bytes;
};

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ void record_error(unsigned long long *counters, unsigned code) {
    atomicCAS(&counters[kCntErr], 0ull, (unsigned long long)code);
}

// Count a query-head that took the probe's general walk and log its flat index.
__device__ __forceinline__ void log_walk(unsigned long long *counters, int32_t *walk_log, long long flat) {
    const unsigned long long k = atomicAdd(&counters[kCntWalks], 1ull);
    if (k < (unsigned long long)kWalkLogCap) walk_log[k] = (int32_t)flat;
}

inline char *ws_ptr(const Plan &p, void *ws, int region) { return (char *)ws + p.off[region]; }

// Host-side count of kernel launches issued by this library (mono_kernel_launches).
void count_launches(int n);

// ---------------------------------------------------------------------------
// kernel launchers (each returns cudaGetLastError() of its launch)
// ---------------------------------------------------------------------------
cudaError_t launch_rope_tables(const Plan &p, void *ws, cudaStream_t s);
cudaError_t launch_project_simt(const Plan &p, const void *x, const void *Wq, const void *Wk, const void *Wv,
                                void *Q, void *K, void *V, const void *ws, cudaStream_t s);
cudaError_t launch_out_project_simt(const Plan &p, const void *O, const void *Wo, void *delta, cudaStream_t s);
cudaError_t launch_summaries(const Plan &p, const void *K, const float *cb, void *ws, cudaStream_t s);
cudaError_t launch_lists(const Plan &p, void *ws, cudaStream_t s);
// reset_stats: clear the routing statistics first (the lists launch has done it when the two run back to back,
// which lets the probe start while the lists kernel still runs)
cudaError_t launch_queries(const Plan &p, const void *Q, const float *cb, const int32_t *forced, int32_t *sel,
                           void *ws, cudaStream_t s, bool reset_stats = true);
cudaError_t launch_attend_simt(const Plan &p, const void *Q, const void *K, const void *V, const int32_t *sel,
                               void *O, void *ws, cudaStream_t s);
bool attend_tc_supported(const mono_config &c);
// cuTensorMapEncodeTiled from the driver (a PFN_cuTensorMapEncodeTiled_v12000), or null
void *tensor_map_encoder();
bool gemm_tc_supported(const mono_config &c);
cudaError_t launch_project_tc(const Plan &p, const void *x, const void *Wq, const void *Wk, const void *Wv, void *Q,
                              void *K, void *V, const void *ws, cudaStream_t s);
cudaError_t launch_out_project_tc(const Plan &p, const void *O, const void *Wo, void *delta, void *ws, cudaStream_t s);
// head-sharded output projection: fp32 rows scattered to the owners' staging buffers, then the owner's sum
cudaError_t launch_out_project_stage(const Plan &p, const void *O, const void *Wo, float *const *stage, int nranks,
                                     int rank, void *ws, cudaStream_t s);
cudaError_t launch_stage_reduce(const Plan &p, const float *stage, int nranks, void *out, cudaStream_t s);
// C_g[M,N] (fp32) (+)= sum_{src < nsrc} A_{g,src}(m,k) B_{g,src}(n,k) for g < ngroups (<= 3, nsrc * ngroups
// <= 6; A and B hold the operands group-major), bf16 operands on the tensor cores; an operand is K-major
// ([M|N rows][K]) or MN-major ([K rows][M|N]).  Pointers 16-byte aligned; row lengths multiples of 8 (supported() checks).
// K is split over several CTAs where the output tiles alone leave the SMs idle and slab (slab_bytes of fp32
// scratch) holds the partial tiles; they are summed in a fixed order, so the result is the same on every run.
bool gemm_grad_tc_supported(int M, int N, int K, bool a_mn, bool b_mn);
cudaError_t gemm_grad_tc(int M, int N, int K, int nsrc, int ngroups, const void *const *A, bool a_mn,
                         const void *const *B, bool b_mn, float *const *C, bool accumulate, float *slab,
                         size_t slab_bytes, unsigned long long *counters, cudaStream_t s);
// The routing regions that mono_route_static uses for plan `p` (offsets in
// rp->off relative to *base, the device address of its fixed array on the
// current device); MONO_ERR_SCRATCH if they do not fit.
int route_static_tables(const Plan &p, void **base, Plan *rp);
// the stages of the tensor-core attention: pair buckets, remote partials, local part + merge
enum AttendParts { kAttendPairs = 1, kAttendRemote = 2, kAttendLocal = 4, kAttendAll = 7 };
// With o32 and lse (backward recompute): the local kernel also writes each row of O in fp32 (token-major like O)
// and its natural log-sum-exp over the query's keys (scores scaled by 1/sqrt(d)); *stats tells whether the kernel
// for this shape did.
// backward, local keys of each query on the tensor cores: dq_loc [B*H, S, d] fp32 = sum over the local keys of
// P (dP - D) k (without the 1/sqrt(d) factor), from the forward's log-sum-exp and D per row and dO as two bf16
// terms [B*H, S, d]; shapes where bwd_local_dq_tc_supported
bool bwd_local_dq_tc_supported(const mono_config &c);
cudaError_t launch_bwd_local_dq_tc(const Plan &p, const void *Q, const void *K, const void *V, const void *dohi,
                                  const void *dolo, const float *lse, const float *dsum, float *dq_loc,
                                  unsigned long long *counters, cudaStream_t s);
// the same for dK and dV, key-major: dk_loc, dv_loc [B*H, S, d] fp32 = sum over the queries whose local window
// holds the key of dS q (without the 1/sqrt(d) factor) and P dO; shapes where bwd_local_dq_tc_supported
cudaError_t launch_bwd_local_dkdv_tc(const Plan &p, const void *Q, const void *K, const void *V, const void *dohi,
                                     const void *dolo, const float *lse, const float *dsum, float *dk_loc,
                                     float *dv_loc, unsigned long long *counters, cudaStream_t s);
// the remote blocks' part on the tensor cores, from the per-block lists of selecting pairs t * R + r (cnt,
// start, list as [B*H, nb] and [B*H, S*R], each list ascending): dq_pair [B*H, S*R, d] = each pair's dQ part,
// dk_loc and dv_loc rows of each block += (one CTA per block)
cudaError_t launch_bwd_remote_tc(const Plan &p, const void *Q, const void *K, const void *V, const void *dohi,
                                 const void *dolo, const float *lse, const float *dsum, const int32_t *cnt,
                                 const int32_t *start, const int32_t *list, float *dq_pair, float *dk_loc,
                                 float *dv_loc, unsigned long long *counters, cudaStream_t s);
cudaError_t launch_attend_tc(const Plan &p, const void *Q, const void *K, const void *V, const int32_t *sel, void *O,
                             void *ws, cudaStream_t s, int parts = kAttendAll, float *o32 = nullptr,
                             float *lse = nullptr, bool *stats = nullptr);

}  // namespace mono

// the opaque plan handle of the C-ABI
struct mono_plan_s {
    mono::Plan p;
};

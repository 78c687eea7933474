// attend_tc.cu -- selected-set attention on the tcgen05 tensor cores (bf16
// storage, fp32 accumulation and softmax).
//
// Source: aitechinspire.com Monodratic article, "Snapshot: key facts from the
// report": each query attends, with exact causal softmax, to the tokens of its
// R selected remote blocks plus its L guaranteed local blocks.
//
// The softmax over Sel(t) is split exactly into partial softmaxes that are
// merged at the end (the max/sum rescaling of online softmax):
//   * remote part, source-block-major: the (query, block) pairs are grouped by
//     block (count -> scan -> fill).  One CTA takes block j and up to 128 of
//     the queries that selected it.  It runs S = Q_sel K_j^T and O = P V_j on
//     the tensor cores and writes one partial (o normalised, in bf16, plus
//     (max, sum)) per pair.  Grouping by block turns the per-query gather
//     into dense 128-row MMAs.
//   * local part, query-tile-major: 128 consecutive queries share their local
//     key range (the query blocks plus the L-1 blocks before them).  A dense
//     masked tile gives S and O.  The same CTA then reads the R remote
//     partials of each query and merges them.
// Scores are kept in the log2 domain: s2 = <q,k> * log2(e)/sqrt(d).
#include "internal.cuh"
#include "tc.cuh"

namespace mono {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ bool sel_valid(int j, int t, int Bs, int L) { return j >= 0 && j <= t / Bs - L; }

// ---------------------------------------------------------------------------
// pair buckets.  Every (b, h) owns a segment of S*R pair slots and of
// wcap = nb + ceil(S*R/kChunk) work items, so the buckets of different heads
// never interact.  Each CTA of the count and fill kernels takes kQTile
// consecutive queries of one (b, h) and aggregates them in shared memory:
// one global atomic per distinct block per CTA instead of one per pair.
// ---------------------------------------------------------------------------
constexpr int kChunk = 128;   // queries per remote work item
constexpr int kQTile = 1024;  // queries per CTA of the count and fill kernels

// grid (ceil(S/kQTile), B*H), 256 threads, smem nb ints
__global__ void __launch_bounds__(256) k_pair_count(const int32_t *__restrict__ sel, int32_t *__restrict__ cnt,
                                                    int S, int R, int nb, int Bs, int L,
                                                    unsigned long long *__restrict__ counters) {
    extern __shared__ int s_h[];
    const long long bh = blockIdx.y;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s_h[j] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kQTile, t1 = min(S, t0 + kQTile);
    bool bad = false;
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x)
        for (int r = 0; r < R; ++r) {
            const int j = sel[((size_t)bh * S + t) * R + r];
            if (sel_valid(j, t, Bs, L)) atomicAdd(&s_h[j], 1);
            else bad |= j >= 0;
        }
    if (bad) record_error(counters, kDevErrBadSel);
    __syncthreads();
    for (int j = threadIdx.x; j < nb; j += blockDim.x)
        if (s_h[j]) atomicAdd(&cnt[bh * nb + j], s_h[j]);
}

// exclusive scan of one (b, h)'s bucket sizes, fill cursors reset, and one
// work item per chunk of <= kChunk queries.  grid B*H, 1024 threads.
__global__ void __launch_bounds__(1024) k_pair_scan(const int32_t *__restrict__ cnt, int32_t *__restrict__ start,
                                                    int32_t *__restrict__ fill, int2 *__restrict__ work,
                                                    int32_t *__restrict__ nwork, int nb, int wcap) {
    __shared__ int s_w[32], s_c[32];
    __shared__ int carry_p, carry_c;
    const long long bh = blockIdx.x;
    if (threadIdx.x == 0) { carry_p = 0; carry_c = 0; }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    for (int base = 0; base < nb; base += blockDim.x) {
        const int j = base + threadIdx.x;
        const int c = j < nb ? cnt[bh * nb + j] : 0;
        const int ch = (c + kChunk - 1) / kChunk;
        int xp = c, xc = ch;  // inclusive warp scans
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int yp = __shfl_up_sync(0xffffffffu, xp, o), yc = __shfl_up_sync(0xffffffffu, xc, o);
            if (lane >= o) { xp += yp; xc += yc; }
        }
        if (lane == 31) { s_w[warp] = xp; s_c[warp] = xc; }
        __syncthreads();
        if (warp == 0) {
            int wp = lane < nw ? s_w[lane] : 0, wc = lane < nw ? s_c[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int yp = __shfl_up_sync(0xffffffffu, wp, o), yc = __shfl_up_sync(0xffffffffu, wc, o);
                if (lane >= o) { wp += yp; wc += yc; }
            }
            s_w[lane] = wp;
            s_c[lane] = wc;
        }
        __syncthreads();
        const int off_p = carry_p + (warp ? s_w[warp - 1] : 0) + xp - c;
        const int off_c = carry_c + (warp ? s_c[warp - 1] : 0) + xc - ch;
        if (j < nb) {
            start[bh * nb + j] = off_p;
            fill[bh * nb + j] = 0;
            for (int k = 0; k < ch; ++k) work[bh * wcap + off_c + k] = make_int2(j, k);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            carry_p += s_w[nw - 1];
            carry_c += s_c[nw - 1];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) nwork[bh] = carry_c;
}

// grid (ceil(S/kQTile), B*H), 256 threads, smem 2*nb ints
__global__ void __launch_bounds__(256) k_pair_fill(const int32_t *__restrict__ sel, const int32_t *__restrict__ start,
                                                   int32_t *__restrict__ fill, int32_t *__restrict__ pairs, int S,
                                                   int R, int nb, int Bs, int L) {
    extern __shared__ int s_h[];
    int *s_base = s_h + nb;
    const long long bh = blockIdx.y;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s_h[j] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kQTile, t1 = min(S, t0 + kQTile);
    constexpr int kPer = (kQTile / 256) * kMaxR;   // pairs one thread can hold
    int my_j[kPer], my_rank[kPer], my_val[kPer];
    int n = 0;
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x)
        for (int r = 0; r < R; ++r) {
            const int j = sel[((size_t)bh * S + t) * R + r];
            if (!sel_valid(j, t, Bs, L)) continue;
            my_j[n] = j;
            my_rank[n] = atomicAdd(&s_h[j], 1);
            my_val[n] = t * R + r;
            ++n;
        }
    __syncthreads();
    for (int j = threadIdx.x; j < nb; j += blockDim.x)
        if (s_h[j]) s_base[j] = atomicAdd(&fill[bh * nb + j], s_h[j]);
    __syncthreads();
    int32_t *seg = pairs + (size_t)bh * S * R;
    for (int k = 0; k < n; ++k) {
        const int j = my_j[k];
        seg[start[bh * nb + j] + s_base[j] + my_rank[k]] = my_val[k];
    }
}

// ---------------------------------------------------------------------------
// shared helpers of the two attention kernels
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg16(const void *p) { return __ldg((const uint4 *)p); }

// rows [0, nrows) of a [*, D] bf16 matrix -> K-major tile (kdim = D); rows >= valid are zero.
// Asynchronous: every copy is in flight at once; complete with cp_async_wait_all.
template <int D>
__device__ __forceinline__ void load_rows(uint8_t *tile, const bf16 *src, int nrows, int valid, int tid, int nthr) {
    for (int idx = tid; idx < nrows * (D / 8); idx += nthr) {
        const int row = idx / (D / 8), c = idx % (D / 8);
        const bool ok = row < valid;
        tc::cp_async16(tile + tc::kmajor_chunk(row, c, D), ok ? (const void *)(src + (size_t)row * D + 8 * c) : src,
                       ok);
    }
}

// rows [0, nkeys) of V ([*, D]) -> MN-major tile for the B operand of O = P V
// (K = keys, N = dims); rows >= valid are zero.  Whole 16-byte chunks, no transpose.
template <int D>
__device__ __forceinline__ void load_v(uint8_t *tile, const bf16 *src, int nkeys, int valid, int tid, int nthr) {
    for (int idx = tid; idx < nkeys * (D / 8); idx += nthr) {
        const int key = idx / (D / 8), c = idx % (D / 8);
        const bool ok = key < valid;
        tc::cp_async16(tile + tc::mnmajor_chunk(key, c, nkeys),
                       ok ? (const void *)(src + (size_t)key * D + 8 * c) : src, ok);
    }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *(uint32_t *)&h;
}

__device__ __forceinline__ bool timed_out(const unsigned long long *counters) {
    return *(volatile const unsigned long long *)&counters[kCntErr] == kDevErrTimeout;
}

// ---------------------------------------------------------------------------
// remote partials: one CTA per (b, h, block j, chunk of <= 128 queries)
// ---------------------------------------------------------------------------
template <int D, int BS>
__global__ void __launch_bounds__(128) k_remote_tc(const bf16 *__restrict__ Q, const bf16 *__restrict__ K,
                                                   const bf16 *__restrict__ V, const int32_t *__restrict__ pairs,
                                                   const int32_t *__restrict__ start, const int32_t *__restrict__ cnt,
                                                   const int2 *__restrict__ work, const int32_t *__restrict__ nwork,
                                                   bf16 *__restrict__ part_o, float2 *__restrict__ part_ml,
                                                   unsigned long long *__restrict__ counters, int S, int R, int nb,
                                                   int wcap, float scale_log2) {
    // TMEM: S in columns [0, BS); O overwrites them once every thread has turned S into P
    constexpr int NCOLS = (BS > D ? BS : D) <= 64 ? 64 : 128;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t mbar;
    __shared__ uint32_t tmem_base;
    const long long bh = blockIdx.y;
    const int item = blockIdx.x;
    if (item >= nwork[bh] || timed_out(counters)) return;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int2 w = work[bh * wcap + item];
    const int j = w.x;
    const size_t bj = (size_t)bh * nb + j;
    const int p0 = start[bj] + w.y * kChunk;
    const int n = min(kChunk, cnt[bj] - w.y * kChunk);
    pairs += (size_t)bh * S * R;

    // P reuses Q's space when it fits: Q is only read by the first MMA, which has completed when P is written
    constexpr int QB = 128 * D * 2, KB = BS * D * 2, VB = BS * D * 2, PB = 128 * BS * 2;
    uint8_t *sQ = smem;                       // [128 x D]
    uint8_t *sK = sQ + QB;                    // [BS x D]
    uint8_t *sVt = sK + KB;                   // V_j, MN-major [BS keys x D]
    uint8_t *sP = PB <= QB ? sQ : sVt + VB;   // [128 x BS]

    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, NCOLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    // gather the selecting queries' rows, and block j's keys and values
    int pr = 0;
    if (tid < n) pr = pairs[p0 + tid];
    const int t = pr / R;
    {
        const bf16 *qrow = Q + ((size_t)bh * S + t) * D;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) tc::cp_async16(sQ + tc::kmajor_chunk(tid, c, D), qrow + 8 * c, tid < n);
    }
    const size_t kv0 = ((size_t)bh * S + (size_t)j * BS) * D;
    load_rows<D>(sK, K + kv0, BS, BS, tid, 128);
    load_v<D>(sVt, V + kv0, BS, BS, tid, 128);
    tc::cp_async_wait_all();
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);

    if (tid == 0) {
        const uint32_t id = tc::idesc_bf16(128, BS);
        const uint32_t aq = tc::smem_u32(sQ), bk = tc::smem_u32(sK);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
            tc::mma_bf16(tmem, tc::desc_kmajor(aq + 256 * k, D), tc::desc_kmajor(bk + 256 * k, D), id, k > 0);
        tc::commit(&mbar);
    }
    bool ok = tc::mbar_wait(&mbar, 0);
    tc::fence_after_sync();

    // softmax of this thread's row over the block's BS keys
    float v[32];
    float m = -INFINITY;
#pragma unroll
    for (int c0 = 0; c0 < BS; c0 += 32) {
        tc::tmem_ld32(trow + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, v[i]);
    }
    const float m2 = m * scale_log2;
    float l = 0.f;
#pragma unroll
    for (int c0 = 0; c0 < BS; c0 += 32) {
        tc::tmem_ld32(trow + c0, v);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float a = exp2f(fmaf(v[8 * q8 + 2 * u], scale_log2, -m2));
                const float b = exp2f(fmaf(v[8 * q8 + 2 * u + 1], scale_log2, -m2));
                l += a + b;
                pk[u] = pack2(a, b);
            }
            *(uint4 *)(sP + tc::kmajor_chunk(tid, (c0 >> 3) + q8, BS)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0 && ok) {
        const uint32_t id = tc::idesc_bf16(128, D, true);
        const uint32_t ap = tc::smem_u32(sP), bv = tc::smem_u32(sVt);
#pragma unroll
        for (int k = 0; k < BS / 16; ++k)
            tc::mma_bf16(tmem, tc::desc_kmajor(ap + 256 * k, BS), tc::desc_mnmajor(bv + 256 * k, BS), id, k > 0);
        tc::commit(&mbar);
    }
    if (ok) ok = tc::mbar_wait(&mbar, 1);
    tc::fence_after_sync();
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);

    // partial output of this (query, block) pair
    const size_t slot = (size_t)bh * S * R + pr;
    const float inv = 1.f / l;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
        tc::tmem_ld32(trow + c0, v);
        if (tid < n && ok) {
            uint4 *dst = (uint4 *)(part_o + slot * D + c0);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                dst[q8] = make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv), pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                     pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv), pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
        }
    }
    if (tid < n && ok) part_ml[slot] = make_float2(m2, l);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, NCOLS);
}

// ---------------------------------------------------------------------------
// local part + merge: one CTA per (b, h, tile of 128 queries)
// ---------------------------------------------------------------------------
template <int D, int BS, int NK>
__global__ void __launch_bounds__(128) k_local_merge_tc(const bf16 *__restrict__ Q, const bf16 *__restrict__ K,
                                                        const bf16 *__restrict__ V, const int32_t *__restrict__ sel,
                                                        const bf16 *__restrict__ part_o,
                                                        const float2 *__restrict__ part_ml, bf16 *__restrict__ O,
                                                        unsigned long long *__restrict__ counters, int S, int H, int R,
                                                        int L, float scale_log2) {
    constexpr int NCOLS = NK <= 128 ? 128 : 256;  // S: [0, NK); O reuses [0, D) after the softmax
    static_assert(NK <= 256 && NK % 32 == 0 && D <= NK, "tile shape");
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t mbar;
    __shared__ uint32_t tmem_base;
    if (timed_out(counters)) return;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int h = blockIdx.y, b = blockIdx.z;
    const long long bh = (long long)b * H + h;
    const int t0 = blockIdx.x * 128;
    const int nq = min(128, S - t0);
    const int kstart = max(0, t0 / BS - L + 1) * BS;
    const int kend = min(S, t0 + 128);
    const int nk = kend - kstart;

    constexpr int QB = 128 * D * 2, KB = NK * D * 2, VB = D * NK * 2, PB = 128 * NK * 2;
    uint8_t *sQ = smem, *sK = smem + QB, *sVt = smem + QB + KB;
    uint8_t *sP = (PB <= QB + KB) ? smem : smem + QB + KB + VB;  // P reuses Q/K once S is computed

    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, NCOLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::fence_mbar_init();
    }
    const bf16 *Qb = Q + ((size_t)bh * S) * D;
    const bf16 *Kb = K + ((size_t)bh * S) * D;
    const bf16 *Vb = V + ((size_t)bh * S) * D;
    load_rows<D>(sQ, Qb + (size_t)t0 * D, 128, nq, tid, 128);
    load_rows<D>(sK, Kb + (size_t)kstart * D, NK, nk, tid, 128);
    load_v<D>(sVt, Vb + (size_t)kstart * D, NK, nk, tid, 128);
    // this query's remote selections and their (max, sum); the partial rows are
    // prefetched to L2 so that the merge at the end does not wait on DRAM
    const int t = t0 + tid;
    const bool live = tid < nq;
    int jr[kMaxR];
    float2 ml[kMaxR];
    for (int r = 0; r < R; ++r) {
        jr[r] = -1;
        if (!live) continue;
        const size_t pq = ((size_t)bh * S + t) * R + r;
        const int j = sel[pq];
        if (sel_valid(j, t, BS, L)) {
            jr[r] = j;
            ml[r] = part_ml[pq];
            for (int c = 0; c < D * 2; c += 128) tc::prefetch_l2((const uint8_t *)(part_o + pq * D) + c);
        }
    }
    tc::cp_async_wait_all();
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    if (tid == 0) {
        const uint32_t id = tc::idesc_bf16(128, NK);
        const uint32_t aq = tc::smem_u32(sQ), bk = tc::smem_u32(sK);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
            tc::mma_bf16(tmem, tc::desc_kmajor(aq + 256 * k, D), tc::desc_kmajor(bk + 256 * k, D), id, k > 0);
        tc::commit(&mbar);
    }
    bool ok = tc::mbar_wait(&mbar, 0);
    tc::fence_after_sync();

    // masked softmax of row t over keys s in [lo(t), t].  In column terms the
    // valid keys are [vlo, vhi]; 32-column chunks entirely inside need no
    // per-element mask and chunks entirely outside need no exponential.
    const int lo = max(0, t / BS - L + 1) * BS;
    const int vlo = lo - kstart, vhi = t - kstart;
    float v[32];
    float m = -INFINITY;
#pragma unroll 1
    for (int c0 = 0; c0 < NK; c0 += 32) {
        tc::tmem_ld32(trow + c0, v);
        if (c0 + 31 < vlo || c0 > vhi) continue;
        if (c0 >= vlo && c0 + 31 <= vhi) {
#pragma unroll
            for (int i = 0; i < 32; ++i) m = fmaxf(m, v[i]);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i >= vlo && c0 + i <= vhi) m = fmaxf(m, v[i]);
        }
    }
    const float m2 = (m == -INFINITY) ? 0.f : m * scale_log2;
    float l = 0.f;
    // P may reuse the space of Q and K: they are only read by the first MMA,
    // which has completed (mbarrier) before any thread gets here.
#pragma unroll 1
    for (int c0 = 0; c0 < NK; c0 += 32) {
        tc::tmem_ld32(trow + c0, v);
        uint32_t pk[16];
        if (c0 + 31 < vlo || c0 > vhi) {
#pragma unroll
            for (int u = 0; u < 16; ++u) pk[u] = 0u;
        } else {
            const bool full = c0 >= vlo && c0 + 31 <= vhi;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = 2 * u;
                float a = exp2f(fmaf(v[i], scale_log2, -m2));
                float bb = exp2f(fmaf(v[i + 1], scale_log2, -m2));
                if (!full) {
                    a = (c0 + i >= vlo && c0 + i <= vhi) ? a : 0.f;
                    bb = (c0 + i + 1 >= vlo && c0 + i + 1 <= vhi) ? bb : 0.f;
                }
                l += a + bb;
                pk[u] = pack2(a, bb);
            }
        }
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8)
            *(uint4 *)(sP + tc::kmajor_chunk(tid, (c0 >> 3) + q8, NK)) =
                make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0 && ok) {
        const uint32_t id = tc::idesc_bf16(128, D, true);
        const uint32_t ap = tc::smem_u32(sP), bv = tc::smem_u32(sVt);
#pragma unroll
        for (int k = 0; k < NK / 16; ++k)
            tc::mma_bf16(tmem, tc::desc_kmajor(ap + 256 * k, NK), tc::desc_mnmajor(bv + 256 * k, NK), id, k > 0);
        tc::commit(&mbar);
    }
    if (ok) ok = tc::mbar_wait(&mbar, 1);
    tc::fence_after_sync();
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);

    // merge with the remote partials: out = (O_loc + sum_r l_r 2^(m_r - M) o_r 2^(m_loc... )) / ...
    float mm = m2;
    for (int r = 0; r < R; ++r)
        if (jr[r] >= 0) mm = fmaxf(mm, ml[r].x);
    const float wl = exp2f(m2 - mm);
    float den = l * wl;
    float wr[kMaxR];
    for (int r = 0; r < R; ++r) {
        wr[r] = 0.f;
        if (jr[r] >= 0) {
            wr[r] = ml[r].y * exp2f(ml[r].x - mm);
            den += wr[r];
        }
    }
    const float inv = 1.f / den;
    bf16 *orow = O + (((size_t)b * S + t) * H + h) * D;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
        tc::tmem_ld32(trow + c0, v);
        if (live && ok) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= wl;
            for (int r = 0; r < R; ++r) {
                if (jr[r] < 0) continue;
                const uint4 *src = (const uint4 *)(part_o + (((size_t)bh * S + t) * R + r) * D + c0);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    uint4 u4 = __ldg(src + q8);
                    const __nv_bfloat162 *h2 = (const __nv_bfloat162 *)&u4;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float2 f = __bfloat1622float2(h2[e]);
                        v[8 * q8 + 2 * e] = fmaf(wr[r], f.x, v[8 * q8 + 2 * e]);
                        v[8 * q8 + 2 * e + 1] = fmaf(wr[r], f.y, v[8 * q8 + 2 * e + 1]);
                    }
                }
            }
            uint4 *dst = (uint4 *)(orow + c0);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                dst[q8] = make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv), pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                     pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv), pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, NCOLS);
}

// ---------------------------------------------------------------------------
bool attend_tc_supported(const mono_config &c) {
    if (c.dtype != MONO_BF16 || (c.d != 64 && c.d != 128) || (c.Bs != 64 && c.Bs != 128)) return false;
    const int nk = 128 + (c.L - 1) * c.Bs;
    return nk <= 256;
}

template <int D, int BS, int NK>
static cudaError_t launch_tc_shape(const Plan &p, const bf16 *Q, const bf16 *K, const bf16 *V, const int32_t *sel,
                                   bf16 *O, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    unsigned long long *cnt_err = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.d));
    const int nbh = c.B * c.H * p.nb;
    cudaError_t e;
    if (c.R > 0) {
        int32_t *pc = (int32_t *)ws_ptr(p, ws, kRegPairCount);
        int32_t *ps = (int32_t *)ws_ptr(p, ws, kRegPairStart);
        int32_t *pf = (int32_t *)ws_ptr(p, ws, kRegPairFill);
        int32_t *pairs = (int32_t *)ws_ptr(p, ws, kRegPairs);
        int2 *work = (int2 *)ws_ptr(p, ws, kRegWork);
        int32_t *nwork = (int32_t *)ws_ptr(p, ws, kRegNWork);
        if ((e = cudaMemsetAsync(pc, 0, (size_t)nbh * 4, s)) != cudaSuccess) return e;
        const int nbhh = c.B * c.H;
        const int wcap = p.max_work;  // work items per (b, h)
        dim3 gq((c.S + kQTile - 1) / kQTile, nbhh);
        const size_t hs = (size_t)p.nb * 4;
        if (2 * hs > 48 * 1024) {
            if ((e = cudaFuncSetAttribute(k_pair_count, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hs)) ||
                (e = cudaFuncSetAttribute(k_pair_fill, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * hs))))
                return e;
        }
        k_pair_count<<<gq, 256, hs, s>>>(sel, pc, c.S, c.R, p.nb, c.Bs, c.L, cnt_err);
        k_pair_scan<<<nbhh, 1024, 0, s>>>(pc, ps, pf, work, nwork, p.nb, wcap);
        k_pair_fill<<<gq, 256, 2 * hs, s>>>(sel, ps, pf, pairs, c.S, c.R, p.nb, c.Bs, c.L);
        const size_t pbytes = (size_t)128 * BS * 2, qbytes = (size_t)128 * D * 2;
        const size_t smem = qbytes + (size_t)2 * BS * D * 2 + (pbytes <= qbytes ? 0 : pbytes);
        auto kr = k_remote_tc<D, BS>;
        if ((e = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        dim3 gr(wcap, nbhh);
        kr<<<gr, 128, smem, s>>>(Q, K, V, pairs, ps, pc, work, nwork, (bf16 *)ws_ptr(p, ws, kRegPartO),
                                 (float2 *)ws_ptr(p, ws, kRegPartML), cnt_err, c.S, c.R, p.nb, wcap, scale_log2);
        count_launches(4);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    constexpr int QB = 128 * D * 2, KB = NK * D * 2, VB = D * NK * 2, PB = 128 * NK * 2;
    const size_t smem = (size_t)QB + KB + VB + ((PB <= QB + KB) ? 0 : PB);
    auto kl = k_local_merge_tc<D, BS, NK>;
    if ((e = cudaFuncSetAttribute(kl, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    dim3 grid((c.S + 127) / 128, c.H, c.B);
    kl<<<grid, 128, smem, s>>>(Q, K, V, sel, (const bf16 *)ws_ptr(p, ws, kRegPartO),
                               (const float2 *)ws_ptr(p, ws, kRegPartML), O, cnt_err, c.S, c.H, c.R, c.L, scale_log2);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_attend_tc(const Plan &p, const void *Q, const void *K, const void *V, const int32_t *sel, void *O,
                             void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    const bf16 *q = (const bf16 *)Q, *k = (const bf16 *)K, *v = (const bf16 *)V;
    bf16 *o = (bf16 *)O;
    const int nk = 128 + (c.L - 1) * c.Bs;
    // NK = the local key range rounded up to a multiple of 32 (MMA N <= 256)
#define MONO_TC(DD, BB, NN) return launch_tc_shape<DD, BB, NN>(p, q, k, v, sel, o, ws, s)
    if (c.d == 64 && c.Bs == 64) {
        if (nk <= 128) MONO_TC(64, 64, 128);
        if (nk <= 192) MONO_TC(64, 64, 192);
        MONO_TC(64, 64, 256);
    }
    if (c.d == 128 && c.Bs == 64) {
        if (nk <= 128) MONO_TC(128, 64, 128);
        if (nk <= 192) MONO_TC(128, 64, 192);
        MONO_TC(128, 64, 256);
    }
    if (c.d == 64 && c.Bs == 128) {
        if (nk <= 128) MONO_TC(64, 128, 128);
        MONO_TC(64, 128, 256);
    }
    if (nk <= 128) MONO_TC(128, 128, 128);
    MONO_TC(128, 128, 256);
#undef MONO_TC
}

}  // namespace mono

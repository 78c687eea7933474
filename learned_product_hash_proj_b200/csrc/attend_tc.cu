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
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.cuh"
#include "tc.cuh"

// Which attention kernels mono_attend runs on the tensor cores (compile-time
// choices between equivalent paths; the results are the same bit for bit):
// the remote partials by the two-stage kernel instead of the warp-specialised
// one, and the remote and local parts fused into one kernel.
#ifndef MONO_REMOTE_TWO_STAGE
#define MONO_REMOTE_TWO_STAGE 0
#endif
#ifndef MONO_ATTEND_FUSED
#define MONO_ATTEND_FUSED 0
#endif

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
constexpr int kMaxGroup = 256;               // (b, h) slices per launch group
constexpr int kQTile = 1024;  // queries per CTA of the count and fill kernels

// Programmatic dependent launch along the attention's kernels: each kernel
// lets its successor's CTAs start at once, and each waits for its
// predecessor's results only before reading them (without a programmatic
// launch the wait returns at once).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
// work item {block, first pair, pair count, 0} per chunk of <= kChunk
// queries; also clears the slice's done counter (and its launch group's
// ticket) of the fused kernel.  grid B*H, 1024 threads.
__global__ void __launch_bounds__(1024) k_pair_scan(const int32_t *__restrict__ cnt, int32_t *__restrict__ start,
                                                    int32_t *__restrict__ fill, int4 *__restrict__ work,
                                                    int32_t *__restrict__ nwork, int *__restrict__ done,
                                                    int *__restrict__ tickets, int nb, int wcap, int group) {
    __shared__ int s_w[32], s_c[32];
    __shared__ int carry_p, carry_c;
    pdl_trigger();
    const long long bh = blockIdx.x;
    if (threadIdx.x == 0) {
        carry_p = 0;
        carry_c = 0;
        done[bh] = 0;
        if (bh % group == 0) tickets[bh / group] = 0;
    }
    pdl_wait();  // the counts are complete
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
            for (int k = 0; k < ch; ++k)
                work[bh * wcap + off_c + k] = make_int4(j, off_p + k * kChunk, min(kChunk, c - k * kChunk), 0);
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
    pdl_trigger();
    const long long bh = blockIdx.y;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s_h[j] = 0;
    pdl_wait();  // the bucket starts and cleared cursors
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

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *(uint32_t *)&h;
}

__device__ __forceinline__ bool timed_out(const unsigned long long *counters) {
    return *(volatile const unsigned long long *)&counters[kCntErr] == kDevErrTimeout;
}

// ---------------------------------------------------------------------------
// remote partials: persistent CTAs of 256 threads walk the work items
// {block j, first pair, pair count} of a group of (b, h) slices with a
// two-stage pipeline: while item k is computed, the tiles of item k+1 are in
// flight and the descriptor and pair ids of item k+2 are being loaded.  K_j
// and V_j arrive by TMA (128-byte swizzle, one thread issues them); the
// gathered query rows by cp.async.  Per item: S = Q_sel K_j^T and O = P V_j on
// tcgen05 (TMEM, 64 or 128 columns reused by every item), softmax in fp32,
// one partial per pair.  As in the local kernel, warps q and q+4 share TMEM
// lane quarter q and split the columns.
// ---------------------------------------------------------------------------
struct RemoteItem {
    long long bh;
    int j, p0, n;
};

// Q, K and V as [B*H, S, D] bf16 for TMA: 64-column (128-byte) boxes, 128-byte swizzle
struct AttnMaps {
    CUtensorMap q, k, v;
};

// dynamic shared memory of the remote kernel: two stages of {Q, K, V}, P (over
// the stage's Q when it fits there), then the small state
template <int D, int BS>
struct RemoteSmem {
    static constexpr int QB = 128 * D * 2, KB = BS * D * 2, VB = BS * D * 2, PB = 128 * BS * 2;
    static constexpr int STAGE = QB + KB + VB;
    static constexpr int P_OFF = PB <= QB ? -1 : 2 * STAGE;       // -1: P over the stage's Q
    static constexpr int RED_OFF = 2 * STAGE + (PB <= QB ? 0 : PB);  // float [2][128]
    static constexpr int PREF_OFF = RED_OFF + 1024;                // int [kMaxGroup + 1]
    static constexpr int BAR_OFF = PREF_OFF + ((kMaxGroup + 1) * 4 + 15) / 16 * 16;  // 3 mbarriers + TMEM base
    static constexpr int BYTES = BAR_OFF + 32;
};

template <int D, int BS>
__global__ void __launch_bounds__(256) k_remote_tc(const __grid_constant__ AttnMaps maps, const bf16 *__restrict__ Q,
                                                   const int32_t *__restrict__ pairs, const int4 *__restrict__ work,
                                                   const int32_t *__restrict__ nwork, bf16 *__restrict__ part_o,
                                                   float2 *__restrict__ part_ml,
                                                   unsigned long long *__restrict__ counters, int S, int R, int wcap,
                                                   float scale_log2, int bh0, int ng) {
    // TMEM: S in columns [0, BS); O overwrites them once every thread has turned S into P
    constexpr int NCOLS = (BS > D ? BS : D) <= 64 ? 64 : 128;
    constexpr int HALF = BS / 2, DH = D / 2;
    static_assert(HALF % 32 == 0 && DH % 32 == 0 && D % 64 == 0, "tile shape");
    using L = RemoteSmem<D, BS>;
    constexpr int QB = L::QB, KB = L::KB, STAGE = L::STAGE;
    extern __shared__ __align__(1024) uint8_t smem[];
    float(*s_red)[128] = (float(*)[128])(smem + L::RED_OFF);
    int *s_pref = (int *)(smem + L::PREF_OFF);
    uint64_t *bar_kv = (uint64_t *)(smem + L::BAR_OFF);  // [2]: K/V of each stage landed
    uint64_t *mbar = bar_kv + 2;                          // MMA completion
    uint32_t *tmem_base = (uint32_t *)(mbar + 1);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {  // uniform; TMA's 128-byte swizzle needs 1024-byte aligned tiles
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;

    if (tid == 0) {
        int acc = 0;
        for (int g = 0; g < ng; ++g) { s_pref[g] = acc; acc += nwork[bh0 + g]; }
        s_pref[ng] = acc;
        tc::mbar_init(&bar_kv[0], 1);
        tc::mbar_init(&bar_kv[1], 1);
        tc::mbar_init(mbar, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_base, NCOLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const int total = s_pref[ng];
    const int G = gridDim.x;

    auto descr = [&](int f) {
        int lo = 0, hi = ng;  // last g with s_pref[g] <= f
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_pref[mid] <= f) lo = mid;
            else hi = mid;
        }
        const long long bh = bh0 + lo;
        const int4 w = work[bh * wcap + (f - s_pref[lo])];
        RemoteItem it;
        it.bh = bh; it.j = w.x; it.p0 = w.y; it.n = w.z;
        return it;
    };
    auto pair_of = [&](const RemoteItem &it) { return row < it.n ? pairs[it.bh * S * R + it.p0 + row] : 0; };
    // the stage's tiles: K_j and V_j by TMA onto bar_kv[stage] (thread 0), the
    // selected query rows by cp.async (every thread, one group)
    auto issue = [&](int stage, const RemoteItem &it, int pr) {
        uint8_t *sQ = smem + stage * STAGE, *sK = sQ + QB, *sV = sK + KB;
        if (tid == 0) {
            tc::mbar_expect_tx(&bar_kv[stage], 2 * KB);
#pragma unroll
            for (int a = 0; a < D / 64; ++a) {
                tc::tma_load_3d(sK + a * (BS * 128), &maps.k, 64 * a, it.j * BS, (int)it.bh, &bar_kv[stage]);
                tc::tma_load_3d(sV + a * (BS * 128), &maps.v, 64 * a, it.j * BS, (int)it.bh, &bar_kv[stage]);
            }
        }
        const bf16 *qrow = Q + ((size_t)it.bh * S + pr / R) * D;
#pragma unroll
        for (int c = half * (D / 16); c < (half + 1) * (D / 16); ++c)
            tc::cp_async16(sQ + tc::kmajor_chunk(row, c, D), qrow + 8 * c, row < it.n);
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    int f = blockIdx.x;
    bool ok = true;
    // per stage: parity of the K/V loads issued and not yet seen complete, or -1
    // (thread 0 issues and waits; before leaving it waits for what is left)
    int pend[2] = {-1, -1};
    if (f < total) {
        RemoteItem it0 = descr(f);
        int pr0 = pair_of(it0);
        issue(0, it0, pr0);
        pend[0] = 0;
        int f1 = f + G;
        bool have1 = f1 < total;
        RemoteItem it1{};
        int pr1 = 0;
        if (have1) { it1 = descr(f1); pr1 = pair_of(it1); }
        for (int k = 0; ok; ++k) {
            const int stage = k & 1;
            const uint32_t kv_parity = (k >> 1) & 1;  // completions of bar_kv[stage] so far, mod 2
            if (have1) {
                issue(stage ^ 1, it1, pr1);
                if (stage) pend[0] = ((k + 1) >> 1) & 1;
                else pend[1] = ((k + 1) >> 1) & 1;
            }
            const int f2 = f1 + G;
            const bool have2 = have1 && f2 < total;
            RemoteItem it2{};
            if (have2) it2 = descr(f2);
            if (have1) asm volatile("cp.async.wait_group 1;" ::: "memory");
            else asm volatile("cp.async.wait_group 0;" ::: "memory");
            tc::fence_smem_to_async();
            const bool landed = tid != 0 || tc::mbar_wait(&bar_kv[stage], kv_parity);
            if (landed) {
                if (stage) pend[1] = -1;
                else pend[0] = -1;
            }
            tc::fence_before_sync();
            ok = __syncthreads_and(landed);
            tc::fence_after_sync();
            if (!ok) break;

            uint8_t *sQ = smem + stage * STAGE, *sK = sQ + QB, *sV = sK + KB;
            uint8_t *sP = L::P_OFF < 0 ? sQ : smem + L::P_OFF;
            if (tid == 0) {
                const uint32_t id = tc::idesc_bf16(128, BS);
                const uint32_t aq = tc::smem_u32(sQ), bk = tc::smem_u32(sK);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_bf16(tmem, tc::desc_kmajor(aq + 256 * kk, D),
                                 tc::desc_sw128(bk + (kk >> 2) * (BS * 128) + (kk & 3) * 32), id, kk > 0);
                tc::commit(mbar);
            }
            ok = __syncthreads_and(tc::mbar_wait(mbar, 0));   // CTA-uniform: the code below has barriers
            tc::fence_after_sync();
            float v[32];
            float m = -INFINITY;
#pragma unroll
            for (int c0 = half * HALF; c0 < half * HALF + HALF; c0 += 32) {
                tc::tmem_ld32(trow + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) m = fmaxf(m, v[i]);
            }
            s_red[half][row] = m;
            __syncthreads();
            m = fmaxf(s_red[0][row], s_red[1][row]);
            const float m2 = m * scale_log2;
            float l = 0.f;
#pragma unroll
            for (int c0 = half * HALF; c0 < half * HALF + HALF; c0 += 32) {
                tc::tmem_ld32(trow + c0, v);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    uint32_t pk[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float a = exp2f(fmaf(v[8 * q8 + 2 * u], scale_log2, -m2));
                        const float bb = exp2f(fmaf(v[8 * q8 + 2 * u + 1], scale_log2, -m2));
                        l += a + bb;
                        pk[u] = pack2(a, bb);
                    }
                    *(uint4 *)(sP + tc::kmajor_chunk(row, (c0 >> 3) + q8, BS)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            __syncthreads();  // every thread has read the maxima
            s_red[half][row] = l;
            tc::fence_smem_to_async();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            l = s_red[0][row] + s_red[1][row];
            // pair ids of item k+2 (its descriptor load has landed by now), consumed next iteration
            const int pr2 = have2 ? pair_of(it2) : 0;
            if (tid == 0 && ok) {
                const uint32_t id = tc::idesc_bf16(128, D, true);
                const uint32_t ap = tc::smem_u32(sP), bv = tc::smem_u32(sV);
#pragma unroll
                for (int kk = 0; kk < BS / 16; ++kk)
                    tc::mma_bf16(tmem, tc::desc_kmajor(ap + 256 * kk, BS), tc::desc_sw128_mn(bv + 2048 * kk, BS * 128),
                                 id, kk > 0);
                tc::commit(mbar);
            }
            ok = __syncthreads_and(ok && tc::mbar_wait(mbar, 1));
            tc::fence_after_sync();
            const bool live = row < it0.n;
            const size_t slot = (size_t)it0.bh * S * R + pr0;
            const float inv = 1.f / l;
#pragma unroll
            for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
                tc::tmem_ld32(trow + c0, v);
                if (live && ok) {
                    uint4 *dst = (uint4 *)(part_o + slot * D + c0);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        dst[q8] = make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv),
                                             pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                             pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv),
                                             pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
                }
            }
            if (live && ok && half == 0) part_ml[slot] = make_float2(m2, l);
            tc::fence_before_sync();
            __syncthreads();  // the stage's tiles and TMEM are free again
            tc::fence_after_sync();
            if (!have1) break;
            it0 = it1; pr0 = pr1;
            it1 = it2; pr1 = pr2;
            have1 = have2; f1 = f2;
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        // leave no TMA write in flight into this CTA's shared memory
        if (tid == 0) {
            if (pend[0] >= 0 && !tc::mbar_wait(&bar_kv[0], (uint32_t)pend[0])) ok = false;
            if (pend[1] >= 0 && !tc::mbar_wait(&bar_kv[1], (uint32_t)pend[1])) ok = false;
        }
    }
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, NCOLS);
}

// ---------------------------------------------------------------------------
// remote partials, warp-specialised: one persistent CTA per SM walks the
// work items {block j, first pair, pair count} of a group of (b, h) slices
// through an NST-deep ring of stages.
//   warp 0             producer: per item, the selecting queries' rows by
//                      cp.async (every lane, 16-byte pieces, arriving on the
//                      stage's "full" barrier as they land) and their pair
//                      ids into the stage; K_j and V_j by TMA (lane 0).  The
//                      work item and pair ids of the next items are read
//                      one and two steps ahead;
//   warp 1 (one lane)  MMA issuer: S = Q K_j^T of items i+1 .. i+NG-1 is
//                      issued before O = P V_j of item i, so that every
//                      softmax group has an item while the tensor core works;
//   NG groups of 4     softmax groups that take items in turn (4 where the
//   warps              tensor memory holds that many items, else 2), one
//                      thread per query row: the softmax of S in fp32, P
//                      (bf16) written back over S in tensor memory and read
//                      from there by the P V MMA, then the normalised partial
//                      (bf16) and its (max, sum) for the merge.
// A stage is released ("empty") by the MMA issuer once both MMAs of its item
// have completed and by the four warps of the group once they have read the
// item's pair ids.  Tensor memory: 512 columns, 512/NG per group (S and P
// first, O in the last D columns).  Every wait is bounded; a role that gives
// up sets a shared abort flag that ends the others' waits, and the producer
// and the MMA issuer wait for their own copies and MMAs in flight before the
// CTA exits.
// ---------------------------------------------------------------------------
template <int D, int BS>
struct RemoteWs {
    static constexpr int QB = 128 * D * 2, KB = BS * D * 2, IDS = 128 * 4 + 16;
    static constexpr int STAGE = QB + 2 * KB + 1024;  // Q, K, V, then pair ids and item (kept 1024-aligned)
    static constexpr int NST = (200 * 1024) / STAGE > 6 ? 6 : (200 * 1024) / STAGE;
    // softmax groups: as many as the 512 tensor-memory columns hold (S/P and O of one item each)
    static constexpr int NG = (BS + D <= 128) ? 4 : 2;
    static constexpr int TG = 512 / NG;              // columns per group
    static constexpr int O_COL = TG - D;
    static constexpr int THREADS = 64 + NG * 128;
    static constexpr int PREF_OFF = NST * STAGE;                                     // int [kMaxGroup + 1]
    static constexpr int BAR_OFF = PREF_OFF + ((kMaxGroup + 1) * 4 + 15) / 16 * 16;
    // mbarriers: full[NST], empty[NST], s_full[NG], p_full[NG], o_full[NG], t_free[NG], drain; TMEM base, abort
    static constexpr int NBAR = 2 * NST + 4 * NG + 1;
    static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
    static constexpr bool supported = NST >= NG + 1 && BS + D <= TG && D % 64 == 0 && BS % 32 == 0 && IDS <= 1024;
};

template <int D, int BS>
__global__ void __launch_bounds__(RemoteWs<D, BS>::THREADS, 1)
    k_remote_ws(const __grid_constant__ AttnMaps maps, const bf16 *__restrict__ Q, const int32_t *__restrict__ pairs,
                const int4 *__restrict__ work, const int32_t *__restrict__ nwork, bf16 *__restrict__ part_o,
                float2 *__restrict__ part_ml, unsigned long long *__restrict__ counters, int S, int R, int wcap,
                float scale_log2, int bh0, int ng) {
    using Lay = RemoteWs<D, BS>;
    static_assert(Lay::supported, "tile shape");
    constexpr int QB = Lay::QB, KB = Lay::KB, STAGE = Lay::STAGE, NST = Lay::NST, NG = Lay::NG, TG = Lay::TG;
    constexpr int CH = D * 2 / 16;  // 16-byte pieces of a query row
    extern __shared__ __align__(1024) uint8_t smem[];
    int *s_pref = (int *)(smem + Lay::PREF_OFF);
    uint64_t *bars = (uint64_t *)(smem + Lay::BAR_OFF);
    uint64_t *full = bars, *empty = bars + NST, *s_full = bars + 2 * NST, *p_full = s_full + NG,
             *o_full = s_full + 2 * NG, *t_free = s_full + 3 * NG, *drain = s_full + 4 * NG;
    uint32_t *tmem_base = (uint32_t *)(bars + Lay::NBAR);
    volatile int *abort_flag = (volatile int *)(tmem_base + 1);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // a stage: Q rows (K-major, no swizzle), K_j and V_j (TMA, 128-byte swizzle), pair ids [128], item (bh, n)
    auto stage_q = [&](int s) { return smem + s * STAGE; };
    auto stage_ids = [&](int s) { return (int *)(smem + s * STAGE + QB + 2 * KB); };

    if (tid == 0) {
        int acc = 0;
        for (int g = 0; g < ng; ++g) { s_pref[g] = acc; acc += nwork[bh0 + g]; }
        s_pref[ng] = acc;
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(&full[s], 32 + 1);  // every producer lane's copies + the K/V transaction
            tc::mbar_init(&empty[s], 1 + 4);  // the MMA issuer + the group's four warps
        }
        for (int g = 0; g < NG; ++g) {
            tc::mbar_init(&s_full[g], 1);
            tc::mbar_init(&p_full[g], 4);
            tc::mbar_init(&o_full[g], 1);
            tc::mbar_init(&t_free[g], 4);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const int total = s_pref[ng];
    const int G = gridDim.x;
    const int n = blockIdx.x < total ? (total - 1 - blockIdx.x) / G + 1 : 0;  // items of this CTA
    bool ok = true;
    auto fail = [&]() {
        ok = false;
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ---------------- producer (the whole warp) ----------------
        // Software-pipelined: while item i's copies are issued, the pair ids of item i+1 (whose work item was
        // read one step earlier) and the work item of i+2 are in flight, so no step waits on a chain of loads.
        auto slice_of = [&](int f, int &g) {
            int lo = 0, hi = ng;  // last slice with s_pref[lo] <= f
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (s_pref[mid] <= f) lo = mid;
                else hi = mid;
            }
            g = lo;
        };
        auto load_item = [&](int i, int &g, int4 &w) {
            const int f = blockIdx.x + i * G;
            slice_of(f, g);
            w = work[(size_t)(bh0 + g) * wcap + (f - s_pref[g])];
        };
        auto load_ids = [&](int g, const int4 &w, int (&pr)[4]) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int row = lane + 32 * k;
                pr[k] = row < w.z ? pairs[(size_t)(bh0 + g) * S * R + w.y + row] : -1;
            }
        };
        int last_v[NST];
#pragma unroll
        for (int s = 0; s < NST; ++s) last_v[s] = -1;
        int g0 = 0, g1 = 0;
        int4 w0 = make_int4(0, 0, 0, 0), w1 = w0;
        int pr0[4] = {-1, -1, -1, -1};
        if (n > 0) { load_item(0, g0, w0); load_ids(g0, w0, pr0); }
        if (n > 1) load_item(1, g1, w1);
        for (int i = 0; i < n && ok; ++i) {
            const int s = i % NST, v = i / NST;
            if (v > 0 && !__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&empty[s], (v - 1) & 1, abort_flag))) {
                fail();
                break;
            }
            const long long bh = bh0 + g0;
            const int j = w0.x, cnt = w0.z;
            uint8_t *sQ = stage_q(s), *sK = sQ + QB, *sV = sK + KB;
            int *ids = stage_ids(s);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int row = lane + 32 * k;
                const bool live = row < cnt;
                ids[row] = pr0[k];
                const bf16 *qrow = Q + ((size_t)bh * S + (live ? pr0[k] / R : 0)) * D;
#pragma unroll
                for (int c = 0; c < CH; ++c) tc::cp_async16(sQ + tc::kmajor_chunk(row, c, D), qrow + 8 * c, live);
            }
            if (lane == 0) {
                ids[128] = g0;
                ids[129] = cnt;
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(&full[s]))
                         : "memory");
            __syncwarp();
            if (lane == 0) {
                tc::mbar_expect_tx(&full[s], 2 * KB);
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    tc::tma_load_3d(sK + a * (BS * 128), &maps.k, 64 * a, j * BS, (int)bh, &full[s]);
                    tc::tma_load_3d(sV + a * (BS * 128), &maps.v, 64 * a, j * BS, (int)bh, &full[s]);
                }
            }
            last_v[s] = v;
            // the next items' loads, consumed in the next steps
            int pr1[4] = {-1, -1, -1, -1};
            if (i + 1 < n) load_ids(g1, w1, pr1);
            int g2 = 0;
            int4 w2 = make_int4(0, 0, 0, 0);
            if (i + 2 < n) load_item(i + 2, g2, w2);
            g0 = g1; w0 = w1;
#pragma unroll
            for (int k = 0; k < 4; ++k) pr0[k] = pr1[k];
            g1 = g2; w1 = w2;
        }
        // every copy issued has landed before the CTA may exit
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0)
            for (int s = 0; s < NST; ++s)
                if (last_v[s] >= 0 && !tc::mbar_wait(&full[s], last_v[s] & 1)) ok = false;
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t id1 = tc::idesc_bf16(128, BS), id2 = tc::idesc_bf16(128, D, true);
            auto mma1 = [&](int i) -> bool {
                const int s = i % NST, v = i / NST, g = i % NG, u = i / NG;
                if (!tc::mbar_wait_or_abort(&full[s], v & 1, abort_flag)) return false;
                if (u > 0 && !tc::mbar_wait_or_abort(&t_free[g], (u - 1) & 1, abort_flag)) return false;
                tc::fence_smem_to_async();
                tc::fence_after_sync();
                const uint32_t aq = tc::smem_u32(stage_q(s)), bk = aq + QB;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_bf16(tmem + g * TG, tc::desc_kmajor(aq + 256 * kk, D),
                                 tc::desc_sw128(bk + (kk >> 2) * (BS * 128) + (kk & 3) * 32), id1, kk > 0);
                tc::commit(&s_full[g]);
                return true;
            };
            auto mma2 = [&](int i) -> bool {
                const int s = i % NST, g = i % NG, u = i / NG;
                if (!tc::mbar_wait_or_abort(&p_full[g], u & 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t bv = tc::smem_u32(stage_q(s)) + QB + KB;
#pragma unroll
                for (int kk = 0; kk < BS / 16; ++kk)
                    tc::mma_bf16_ts(tmem + g * TG + Lay::O_COL, tmem + g * TG + 8 * kk,
                                    tc::desc_sw128_mn(bv + 2048 * kk, BS * 128), id2, kk > 0);
                tc::commit(&o_full[g]);
                tc::commit(&empty[s]);
                return true;
            };
            // S of the next NG-1 items is issued before O of this one, so every softmax group has work
            for (int i = 0; i < NG - 1 && i < n && ok; ++i)
                if (!mma1(i)) fail();
            for (int i = 0; i < n && ok; ++i) {
                if (i + NG - 1 < n && !mma1(i + NG - 1)) { fail(); break; }
                if (!mma2(i)) { fail(); break; }
            }
            // every MMA issued has completed before the CTA may exit
            tc::commit(drain);
            if (!tc::mbar_wait(drain, 0)) ok = false;
        }
    } else {
        // ---------------- softmax groups ----------------
        const int g = (warp - 2) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t tS = tmem + g * TG + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tO = tS + Lay::O_COL;
        for (int i = g; i < n && ok; i += NG) {
            const int s = i % NST, v = i / NST, u = i / NG;
            // (the decisions to go on are warp-uniform: the TMEM accesses below are warp-collective)
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&full[s], v & 1, abort_flag))) { fail(); break; }
            const int *ids = stage_ids(s);
            const int pr = ids[row];
            const long long bh = bh0 + ids[128];
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[s]);  // this warp is done with the stage
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&s_full[g], u & 1, abort_flag))) { fail(); break; }
            tc::fence_after_sync();
            // softmax of the row over the block's BS keys (all visible: the block lies before the query)
            float vv[32];
            float m = -INFINITY;
#pragma unroll
            for (int c0 = 0; c0 < BS; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tS + c0, vv);
#pragma unroll
                for (int k = 0; k < 32; ++k) m = fmaxf(m, vv[k]);
            }
            const float m2 = m * scale_log2;
            float l = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < BS; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tS + c0, vv);
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float a = exp2f(fmaf(vv[2 * k], scale_log2, -m2));
                    const float bb = exp2f(fmaf(vv[2 * k + 1], scale_log2, -m2));
                    l += a + bb;
                    pk[k] = pack2(a, bb);
                }
                // P over the columns of S already read (column c0/2 .. c0/2 + 15 of this row)
                __syncwarp();
                tc::tmem_st16(tS + (c0 >> 1), pk);
            }
            __syncwarp();
            tc::tmem_st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&p_full[g]);
            const float inv = 1.f / l;
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&o_full[g], u & 1, abort_flag))) { fail(); break; }
            tc::fence_after_sync();
            const bool live = pr >= 0;
            const size_t slot = (size_t)bh * S * R + (live ? pr : 0);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tO + c0, vv);
                if (live) {
                    uint4 *dst = (uint4 *)(part_o + slot * D + c0);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        dst[q8] = make_uint4(pack2(vv[8 * q8] * inv, vv[8 * q8 + 1] * inv),
                                             pack2(vv[8 * q8 + 2] * inv, vv[8 * q8 + 3] * inv),
                                             pack2(vv[8 * q8 + 4] * inv, vv[8 * q8 + 5] * inv),
                                             pack2(vv[8 * q8 + 6] * inv, vv[8 * q8 + 7] * inv));
                }
            }
            if (live) part_ml[slot] = make_float2(m2, l);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&t_free[g]);
        }
    }
    if (!ok) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// local part + merge: persistent CTAs of 256 threads walk the 128-query tiles
// of a group of (b, h) slices.  Per tile: S over the tile's local key range
// (<= 256 keys) and O = P V on tcgen05, the masked softmax in fp32, and the
// exact merge with the tile's remote partials.  The Q, K and V tiles arrive
// by TMA (128-byte swizzle; one thread issues them): the next tile's Q as
// soon as this tile's S has been computed, its K and V once O has.  TMEM lane
// quarter q (rows 32q .. 32q+31) is read by warps q and q+4, each taking half
// of the columns; their partial row max and sum meet in shared memory (in the
// K tile, which is free between the two MMAs).
// ---------------------------------------------------------------------------
template <int D, int NK>
struct LocalSmem {
    static constexpr int QB = 128 * D * 2, KB = NK * D * 2, VB = NK * D * 2, PB = 128 * NK * 2;
    static constexpr int Q_OFF = 0, K_OFF = QB, V_OFF = QB + KB, P_OFF = QB + KB + VB;
    static constexpr int BAR_OFF = P_OFF + PB;  // 3 mbarriers + TMEM base
    static constexpr int BYTES = BAR_OFF + 32;
};
template <int D, int NK>
constexpr size_t local_smem() {
    return LocalSmem<D, NK>::BYTES;
}

template <int D, int BS, int NK, int RMAX>
__global__ void __launch_bounds__(256) k_local_merge_tc(const __grid_constant__ AttnMaps maps,
                                                        const int32_t *__restrict__ sel,
                                                        const bf16 *__restrict__ part_o,
                                                        const float2 *__restrict__ part_ml, bf16 *__restrict__ O,
                                                        unsigned long long *__restrict__ counters, int S, int H, int R,
                                                        int L, float scale_log2, int bh0, int ng) {
    constexpr int NCOLS = NK <= 128 ? 128 : 256;  // S: [0, NK); O reuses [0, D) after the softmax
    constexpr int HALF = NK / 2, DH = D / 2;
    static_assert(NK <= 256 && HALF % 32 == 0 && DH % 32 == 0 && D <= NK && D % 64 == 0, "tile shape");
    using Lay = LocalSmem<D, NK>;
    constexpr int QB = Lay::QB, KB = Lay::KB;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *sQ = smem + Lay::Q_OFF, *sK = smem + Lay::K_OFF, *sV = smem + Lay::V_OFF, *sP = smem + Lay::P_OFF;
    float(*s_red)[128] = (float(*)[128])sK;
    uint64_t *bar_q = (uint64_t *)(smem + Lay::BAR_OFF), *bar_kv = bar_q + 1, *mbar = bar_q + 2;
    uint32_t *tmem_base = (uint32_t *)(bar_q + 3);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {  // uniform; TMA's 128-byte swizzle needs 1024-byte aligned tiles
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int ntiles = (S + 127) / 128;
    const int total = ng * ntiles;
    const int G = gridDim.x;

    if (warp == 0) {
        tc::tmem_alloc(tmem_base, NCOLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar_q, 1);
        tc::mbar_init(bar_kv, 1);
        tc::mbar_init(mbar, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);

    // TMA of tile f's Q tile / K and V tiles (thread 0).  Rows past the end of
    // the (b, h) slice read as zero.
    auto issue_q = [&](int f) {
        const int bh = bh0 + f / ntiles, t0 = (f % ntiles) * 128;
        tc::mbar_expect_tx(bar_q, QB);
#pragma unroll
        for (int a = 0; a < D / 64; ++a) tc::tma_load_3d(sQ + a * (128 * 128), &maps.q, 64 * a, t0, bh, bar_q);
    };
    auto issue_kv = [&](int f) {
        const int bh = bh0 + f / ntiles, t0 = (f % ntiles) * 128;
        const int kstart = max(0, t0 / BS - L + 1) * BS;
        tc::mbar_expect_tx(bar_kv, 2 * KB);
#pragma unroll
        for (int a = 0; a < D / 64; ++a) {
            tc::tma_load_3d(sK + a * (NK * 128), &maps.k, 64 * a, kstart, bh, bar_kv);
            tc::tma_load_3d(sV + a * (NK * 128), &maps.v, 64 * a, kstart, bh, bar_kv);
        }
    };

    bool ok = true;
    int f = blockIdx.x;
    // this row's selections of the next tile, loaded one tile ahead
    // (R <= RMAX; arrays indexed by compile-time slot so they stay in registers)
    constexpr int kPre = DH <= 32 ? (RMAX < 2 ? RMAX : 2) : 0;  // slots whose partial rows go to registers early
    int selv[RMAX];
    auto load_sel = [&](int ff) {
        const long long bbh = bh0 + ff / ntiles;
        const int tt = (ff % ntiles) * 128 + row;
#pragma unroll
        for (int r = 0; r < RMAX; ++r) selv[r] = (r < R && tt < S) ? sel[((size_t)bbh * S + tt) * R + r] : -1;
    };
    // thread 0: the tile count k of the Q and of the K/V loads issued and not
    // yet seen complete, or -1 (waited for before leaving)
    int pend_q = -1, pend_kv = -1;
    if (f < total) {
        if (tid == 0) {
            issue_q(f);
            issue_kv(f);
            pend_q = pend_kv = 0;
        }
        load_sel(f);
    }
    for (int k = 0; f < total && ok; ++k, f += G) {
        const bool have1 = f + G < total;
        // this tile's geometry; this row's remote selections, their (max, sum)
        // and partial rows are requested now and used by the merge at the end
        const long long bh = bh0 + f / ntiles;
        const int b = (int)(bh / H), h = (int)(bh % H);
        const int t0 = (f % ntiles) * 128;
        const int nq = min(128, S - t0);
        const int kstart = max(0, t0 / BS - L + 1) * BS;
        const int t = t0 + row;
        const bool live = row < nq;
        int jr[RMAX];
        float2 ml[RMAX];
        uint4 pre[kPre > 0 ? kPre : 1][DH / 8];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            jr[r] = -1;
            ml[r] = make_float2(0.f, 0.f);
            if (r >= R || !live || !sel_valid(selv[r], t, BS, L)) continue;
            const size_t pq = ((size_t)bh * S + t) * R + r;
            jr[r] = selv[r];
            ml[r] = part_ml[pq];
            if (r < kPre) {
#pragma unroll
                for (int q8 = 0; q8 < DH / 8; ++q8)
                    pre[r < kPre ? r : 0][q8] = __ldg((const uint4 *)(part_o + pq * D + half * DH) + q8);
            } else {
                tc::prefetch_l2(part_o + pq * D + half * DH);
            }
        }
        if (have1) load_sel(f + G);
        bool landed = true;
        if (tid == 0) {
            const uint32_t par = k & 1;  // each barrier completes once per tile
            const bool lq = tc::mbar_wait(bar_q, par);
            if (lq) pend_q = -1;
            const bool lkv = lq && tc::mbar_wait(bar_kv, par);
            if (lkv) pend_kv = -1;
            landed = lq && lkv;
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(landed);
        tc::fence_after_sync();
        if (!ok) break;
        if (tid == 0) {
            const uint32_t id = tc::idesc_bf16(128, NK);
            const uint32_t aq = tc::smem_u32(sQ), bk = tc::smem_u32(sK);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                tc::mma_bf16(tmem, tc::desc_sw128(aq + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                             tc::desc_sw128(bk + (kk >> 2) * (NK * 128) + (kk & 3) * 32), id, kk > 0);
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, 0));
        tc::fence_after_sync();
        if (tid == 0 && have1 && ok) {
            issue_q(f + G);  // S is computed: the Q tile is free
            pend_q = k + 1;
        }

        // masked softmax of row t over keys s in [lo(t), t]; in column terms
        // [vlo, vhi].  32-column chunks entirely inside need no per-element
        // mask, chunks entirely outside no exponential.
        const int lo = max(0, t / BS - L + 1) * BS;
        const int vlo = lo - kstart, vhi = t - kstart;
        const int cbeg = half * HALF;
        float v[32];
        float m = -INFINITY;
#pragma unroll 1
        for (int c0 = cbeg; c0 < cbeg + HALF; c0 += 32) {
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
        s_red[half][row] = m;
        __syncthreads();
        m = fmaxf(s_red[0][row], s_red[1][row]);
        const float m2 = (m == -INFINITY) ? 0.f : m * scale_log2;
        float l = 0.f;
#pragma unroll 1
        for (int c0 = cbeg; c0 < cbeg + HALF; c0 += 32) {
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
                *(uint4 *)(sP + tc::kmajor_chunk(row, (c0 >> 3) + q8, NK)) =
                    make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
        }
        __syncthreads();  // every thread has read the maxima
        s_red[half][row] = l;
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        l = s_red[0][row] + s_red[1][row];
        if (tid == 0 && ok) {
            const uint32_t id = tc::idesc_bf16(128, D, true);
            const uint32_t ap = tc::smem_u32(sP), bv = tc::smem_u32(sV);
#pragma unroll
            for (int kk = 0; kk < NK / 16; ++kk)
                tc::mma_bf16(tmem, tc::desc_kmajor(ap + 256 * kk, NK), tc::desc_sw128_mn(bv + 2048 * kk, NK * 128),
                             id, kk > 0);
            tc::commit(mbar);
        }
        ok = __syncthreads_and(ok && tc::mbar_wait(mbar, 1));
        tc::fence_after_sync();
        if (tid == 0 && have1 && ok) {
            tc::fence_smem_to_async();  // the row exchange in the K tile is read; TMA may overwrite it
            issue_kv(f + G);            // O is computed: the K and V tiles are free
            pend_kv = k + 1;
        }

        // merge with the remote partials (max/sum rescaling), this thread's half of the columns
        float mm = m2;
#pragma unroll
        for (int r = 0; r < RMAX; ++r)
            if (jr[r] >= 0) mm = fmaxf(mm, ml[r].x);
        const float wl = exp2f(m2 - mm);
        float den = l * wl;
        float wr[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            wr[r] = 0.f;
            if (jr[r] >= 0) {
                wr[r] = ml[r].y * exp2f(ml[r].x - mm);
                den += wr[r];
            }
        }
        const float inv = 1.f / den;
        bf16 *orow = O + (((size_t)b * S + t) * H + h) * D;
#pragma unroll
        for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
            tc::tmem_ld32(trow + c0, v);
            if (live && ok) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= wl;
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    if (jr[r] < 0) continue;
                    const uint4 *src = (const uint4 *)(part_o + (((size_t)bh * S + t) * R + r) * D + c0);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint4 u4;
                        if (kPre > 0 && r < kPre) u4 = pre[r < kPre ? r : 0][((c0 - half * DH) >> 3) + q8];
                        else u4 = __ldg(src + q8);
                        const __nv_bfloat162 *h2 = (const __nv_bfloat162 *)&u4;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float2 fv = __bfloat1622float2(h2[e]);
                            v[8 * q8 + 2 * e] = fmaf(wr[r], fv.x, v[8 * q8 + 2 * e]);
                            v[8 * q8 + 2 * e + 1] = fmaf(wr[r], fv.y, v[8 * q8 + 2 * e + 1]);
                        }
                    }
                }
                uint4 *dst = (uint4 *)(orow + c0);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    dst[q8] = make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv),
                                         pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                         pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv),
                                         pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
            }
        }
        tc::fence_before_sync();
        __syncthreads();  // P and TMEM are free again
        tc::fence_after_sync();
    }
    // leave no TMA write in flight into this CTA's shared memory
    if (tid == 0) {
        if (pend_q >= 0 && !tc::mbar_wait(bar_q, pend_q & 1)) ok = false;
        if (pend_kv >= 0 && !tc::mbar_wait(bar_kv, pend_kv & 1)) ok = false;
    }
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, NCOLS);
}

// ---------------------------------------------------------------------------
// local part + merge, warp-specialised: one persistent CTA of 320 threads per
// SM walks the 128-query tiles of a group of (b, h) slices.
//   warp 0 (one lane)  TMA producer: the Q, K and V tiles of each tile into an
//                      NST-deep ring of stages ("full" / "empty" mbarriers);
//   warp 1 (one lane)  MMA issuer: S = Q K^T of tile i+1 is issued before
//                      O = P V of tile i, so that the tensor core works on
//                      one tile while the softmax runs on the other;
//   warps 2-5, 6-9     two softmax groups that take alternate tiles, one
//                      thread per query row: the masked softmax of S in fp32,
//                      P (bf16) written back over S in tensor memory and
//                      read from there by the P V MMA, then the merge with the
//                      remote partials and the output row.
// Tensor memory: 512 columns, 256 per group (S and P from column 0, O from
// column 256 - D).  Every wait is bounded; a role that gives up sets a shared
// abort flag that ends the others' waits, and the producer and the MMA issuer
// wait for their own copies and MMAs in flight before the CTA exits.
// ---------------------------------------------------------------------------
template <int D, int NK>
struct LocalWs {
    static constexpr int QB = 128 * D * 2, KB = NK * D * 2, STAGE = QB + 2 * KB;
    static constexpr int NST = (200 * 1024) / STAGE > 4 ? 4 : (200 * 1024) / STAGE;
    static constexpr int O_COL = 256 - D;
    static constexpr int BAR_OFF = NST * STAGE;
    // mbarriers: full[NST], empty[NST], s_full[2], p_full[2], o_full[2], t_free[2], drain; then TMEM base, abort
    static constexpr int NBAR = 2 * NST + 9;
    static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
    static constexpr bool supported = NST >= 2 && NK + D <= 256 && D % 64 == 0 && NK % 32 == 0;
};

template <int D, int BS, int NK, int RMAX>
__global__ void __launch_bounds__(320, 1) k_local_ws(const __grid_constant__ AttnMaps maps,
                                                     const int32_t *__restrict__ sel, const bf16 *__restrict__ part_o,
                                                     const float2 *__restrict__ part_ml, bf16 *__restrict__ O,
                                                     unsigned long long *__restrict__ counters, int S, int H, int R,
                                                     int L, float scale_log2, int bh0, int ng) {
    using Lay = LocalWs<D, NK>;
    static_assert(Lay::supported, "tile shape");
    constexpr int QB = Lay::QB, KB = Lay::KB, STAGE = Lay::STAGE, NST = Lay::NST;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *bars = (uint64_t *)(smem + Lay::BAR_OFF);
    uint64_t *full = bars, *empty = bars + NST, *s_full = bars + 2 * NST, *p_full = s_full + 2, *o_full = s_full + 4,
             *t_free = s_full + 6, *drain = s_full + 8;
    uint32_t *tmem_base = (uint32_t *)(bars + Lay::NBAR);
    volatile int *abort_flag = (volatile int *)(tmem_base + 1);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = (S + 127) / 128;
    const int total = ng * ntiles;
    const int G = gridDim.x;
    const int n = blockIdx.x < total ? (total - 1 - blockIdx.x) / G + 1 : 0;  // tiles of this CTA
    auto tile_of = [&](int i) { return blockIdx.x + i * G; };

    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int g = 0; g < 2; ++g) {
            tc::mbar_init(&s_full[g], 1);
            tc::mbar_init(&p_full[g], 4);
            tc::mbar_init(&o_full[g], 1);
            tc::mbar_init(&t_free[g], 4);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    bool ok = true;
    auto fail = [&]() {
        ok = false;
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int last_v[4] = {-1, -1, -1, -1};  // per stage: use count of its latest issue
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % NST, v = i / NST;
                if (v > 0 && !tc::mbar_wait_or_abort(&empty[s], (v - 1) & 1, abort_flag)) { fail(); break; }
                const int f = tile_of(i);
                const int bh = bh0 + f / ntiles, t0 = (f % ntiles) * 128;
                const int kstart = max(0, t0 / BS - L + 1) * BS;
                uint8_t *sQ = smem + s * STAGE, *sK = sQ + QB, *sV = sK + KB;
                tc::mbar_expect_tx(&full[s], QB + 2 * KB);
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    tc::tma_load_3d(sQ + a * (128 * 128), &maps.q, 64 * a, t0, bh, &full[s]);
                    tc::tma_load_3d(sK + a * (NK * 128), &maps.k, 64 * a, kstart, bh, &full[s]);
                    tc::tma_load_3d(sV + a * (NK * 128), &maps.v, 64 * a, kstart, bh, &full[s]);
                }
                last_v[s] = v;
            }
            // every copy issued has landed before the CTA may exit
            for (int s = 0; s < NST; ++s)
                if (last_v[s] >= 0 && !tc::mbar_wait(&full[s], last_v[s] & 1)) ok = false;
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t id1 = tc::idesc_bf16(128, NK), id2 = tc::idesc_bf16(128, D, true);
            auto mma1 = [&](int i) -> bool {
                const int s = i % NST, v = i / NST, g = i & 1, u = i >> 1;
                if (!tc::mbar_wait_or_abort(&full[s], v & 1, abort_flag)) return false;
                if (u > 0 && !tc::mbar_wait_or_abort(&t_free[g], (u - 1) & 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t aq = tc::smem_u32(smem + s * STAGE), bk = aq + QB;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_bf16(tmem + g * 256, tc::desc_sw128(aq + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                                 tc::desc_sw128(bk + (kk >> 2) * (NK * 128) + (kk & 3) * 32), id1, kk > 0);
                tc::commit(&s_full[g]);
                return true;
            };
            auto mma2 = [&](int i) -> bool {
                const int s = i % NST, g = i & 1, u = i >> 1;
                if (!tc::mbar_wait_or_abort(&p_full[g], u & 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t bv = tc::smem_u32(smem + s * STAGE) + QB + KB;
#pragma unroll
                for (int kk = 0; kk < NK / 16; ++kk)
                    tc::mma_bf16_ts(tmem + g * 256 + Lay::O_COL, tmem + g * 256 + 8 * kk,
                                    tc::desc_sw128_mn(bv + 2048 * kk, NK * 128), id2, kk > 0);
                tc::commit(&o_full[g]);
                tc::commit(&empty[s]);
                return true;
            };
            if (n > 0 && !mma1(0)) fail();
            for (int i = 0; i < n && ok; ++i) {
                if (i + 1 < n && !mma1(i + 1)) { fail(); break; }
                if (!mma2(i)) { fail(); break; }
            }
            // every MMA issued has completed before the CTA may exit
            tc::commit(drain);
            if (!tc::mbar_wait(drain, 0)) ok = false;
        }
    } else {
        // ---------------- softmax groups ----------------
        const int g = (warp - 2) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t tS = tmem + g * 256 + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tO = tS + Lay::O_COL;
        // remote partial rows held in registers from the tile's start (two of 64 or one of 128 values)
        constexpr int kPre = D == 64 ? (RMAX < 2 ? RMAX : 2) : (RMAX < 1 ? RMAX : 1);
        // this row's selections for the group's next tile, loaded one tile ahead
        int selv[RMAX];
        auto load_sel = [&](int i) {
            const int f = tile_of(i);
            const long long bh = bh0 + f / ntiles;
            const int t = (f % ntiles) * 128 + row;
#pragma unroll
            for (int r = 0; r < RMAX; ++r) selv[r] = (r < R && t < S) ? sel[((size_t)bh * S + t) * R + r] : -1;
        };
        if (g < n) load_sel(g);
        for (int i = g; i < n && ok; i += 2) {
            const int u = i >> 1;
            const int f = tile_of(i);
            const long long bh = bh0 + f / ntiles;
            const int b = (int)(bh / H), h = (int)(bh % H);
            const int t0 = (f % ntiles) * 128;
            const int kstart = max(0, t0 / BS - L + 1) * BS;
            const int t = t0 + row;
            const bool live = t < S;
            // this row's remote selections, their (max, sum) and partial rows, requested now
            int jr[RMAX];
            float2 ml[RMAX];
            uint4 pre[kPre > 0 ? kPre : 1][D / 8];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                jr[r] = -1;
                ml[r] = make_float2(0.f, 0.f);
                const int j = selv[r];
                if (!sel_valid(j, t, BS, L)) continue;
                const size_t pq = ((size_t)bh * S + t) * R + r;
                jr[r] = j;
                ml[r] = part_ml[pq];
                if (r < kPre) {
#pragma unroll
                    for (int q8 = 0; q8 < D / 8; ++q8)
                        pre[r < kPre ? r : 0][q8] = __ldg((const uint4 *)(part_o + pq * D) + q8);
                } else {
                    tc::prefetch_l2(part_o + pq * D);
                }
            }
            if (i + 2 < n) load_sel(i + 2);
            // (the decision to go on is warp-uniform: the TMEM accesses below are warp-collective)
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&s_full[g], u & 1, abort_flag))) { fail(); break; }
            tc::fence_after_sync();

            // masked softmax of row t over keys [lo(t), t]: columns [vlo, vhi]
            const int lo = max(0, t / BS - L + 1) * BS;
            const int vlo = lo - kstart, vhi = t - kstart;
            float v[32];
            float m = -INFINITY;
            // (tcgen05.ld / st are warp-collective: every lane issues them, whatever its row needs)
#pragma unroll 1
            for (int c0 = 0; c0 < NK; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tS + c0, v);
                if (c0 + 31 < vlo || c0 > vhi) continue;
                if (c0 >= vlo && c0 + 31 <= vhi) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) m = fmaxf(m, v[k]);
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (c0 + k >= vlo && c0 + k <= vhi) m = fmaxf(m, v[k]);
                }
            }
            const float m2 = (m == -INFINITY) ? 0.f : m * scale_log2;
            float l = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < NK; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tS + c0, v);
                uint32_t pk[16];
                if (c0 + 31 < vlo || c0 > vhi) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = 0u;
                } else {
                    const bool full_chunk = c0 >= vlo && c0 + 31 <= vhi;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float a = exp2f(fmaf(v[2 * k], scale_log2, -m2));
                        float bb = exp2f(fmaf(v[2 * k + 1], scale_log2, -m2));
                        if (!full_chunk) {
                            a = (c0 + 2 * k >= vlo && c0 + 2 * k <= vhi) ? a : 0.f;
                            bb = (c0 + 2 * k + 1 >= vlo && c0 + 2 * k + 1 <= vhi) ? bb : 0.f;
                        }
                        l += a + bb;
                        pk[k] = pack2(a, bb);
                    }
                }
                // P over the columns of S already read (column c0/2 .. c0/2 + 15 of this row)
                __syncwarp();
                tc::tmem_st16(tS + (c0 >> 1), pk);
            }
            __syncwarp();
            tc::tmem_st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&p_full[g]);

            // merge with the remote partials (max/sum rescaling)
            float mm = m2;
#pragma unroll
            for (int r = 0; r < RMAX; ++r)
                if (jr[r] >= 0) mm = fmaxf(mm, ml[r].x);
            const float wl = exp2f(m2 - mm);
            float den = l * wl;
            float wr[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                wr[r] = 0.f;
                if (jr[r] >= 0) {
                    wr[r] = ml[r].y * exp2f(ml[r].x - mm);
                    den += wr[r];
                }
            }
            const float inv = 1.f / den;
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&o_full[g], u & 1, abort_flag))) { fail(); break; }
            tc::fence_after_sync();
            bf16 *orow = O + (((size_t)b * S + t) * H + h) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tO + c0, v);
                if (live) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] *= wl;
#pragma unroll
                    for (int r = 0; r < RMAX; ++r) {
                        if (jr[r] < 0) continue;
                        const uint4 *src = (const uint4 *)(part_o + (((size_t)bh * S + t) * R + r) * D + c0);
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            uint4 u4;
                            if (kPre > 0 && r < kPre) u4 = pre[r < kPre ? r : 0][(c0 >> 3) + q8];
                            else u4 = __ldg(src + q8);
                            const __nv_bfloat162 *h2 = (const __nv_bfloat162 *)&u4;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 fv = __bfloat1622float2(h2[e]);
                                v[8 * q8 + 2 * e] = fmaf(wr[r], fv.x, v[8 * q8 + 2 * e]);
                                v[8 * q8 + 2 * e + 1] = fmaf(wr[r], fv.y, v[8 * q8 + 2 * e + 1]);
                            }
                        }
                    }
                    uint4 *dst = (uint4 *)(orow + c0);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        dst[q8] = make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv),
                                             pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                             pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv),
                                             pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&t_free[g]);
        }
    }
    if (!ok) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// The whole selected-set attention of a group of (b, h) slices in one
// persistent warp-specialised kernel (one 320-thread CTA per SM), so that a
// slice's remote partials are read back while they are still in L2 and no
// launch tail separates the two parts.  The work list runs in phases: phase k
// holds the remote items {block j, first pair, pair count} of slice k, then
// the 128-query local tiles of slice k-1.  The producer of each CTA takes the
// next item from a ticket counter, so items are taken in order by CTAs that
// are running.  The roles are those of k_remote_ws and k_local_ws:
//   warp 0             producer: a remote item's query rows by cp.async (every
//                      lane) and K_j, V_j by TMA, or a local tile's Q tile and
//                      K/V window by TMA (lane 0), into a ring of stages;
//   warp 1 (one lane)  MMA issuer: S = Q K^T of item i+1 before O = P V of
//                      item i (N = Bs keys for a remote item, NK for a tile);
//   warps 2-5, 6-9     softmax groups on alternate items: a remote item's
//                      softmax and partial, or a tile's masked softmax and its
//                      merge with the partials of its queries' remote blocks.
// A remote item's four warps each add 1 to the slice's done counter after
// their partial rows are stored (and fenced); a local tile of slice g first
// waits (bounded) until the counter reaches 4 x the slice's remote items.
// Every item taken before a waiting tile is held by a running CTA and is a
// remote item of an earlier or the same phase or a tile of an earlier slice,
// so the waits end.  When the tickets run out the producer writes an end
// record into the next two stages, one for each softmax group.
// ---------------------------------------------------------------------------
template <int D, int BS, int NK>
struct AttendWs {
    static constexpr int QB = 128 * D * 2, KVB = NK * D * 2;
    static constexpr int STAGE = QB + 2 * KVB + 1024;  // Q, K, V, then the item's record (pair ids, kind, slice)
    static constexpr int NST = (200 * 1024) / STAGE > 4 ? 4 : (200 * 1024) / STAGE;
    static constexpr int O_COL = 256 - D;
    static constexpr int PH_OFF = NST * STAGE;                                   // int [kMaxGroup + 2] phase starts
    static constexpr int NR_OFF = PH_OFF + (kMaxGroup + 2) * 4;                  // int [kMaxGroup] remote items
    static constexpr int BAR_OFF = (NR_OFF + kMaxGroup * 4 + 15) / 16 * 16;
    static constexpr int NBAR = 2 * NST + 9;
    static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
    static constexpr bool supported = NST >= 2 && NK + D <= 256 && BS <= NK && D % 64 == 0 && NK % 32 == 0 &&
                                      BS % 32 == 0 && STAGE % 1024 == 0 && BYTES <= 227 * 1024;
};

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint4 ld_cg16(const void *p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ float2 ld_cg_f2(const float2 *p) {
    float2 v;
    asm volatile("ld.global.cg.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}

template <int D, int BS, int NK, int RMAX>
__global__ void __launch_bounds__(320, 1) k_attend_ws(const __grid_constant__ AttnMaps lm, const __grid_constant__ AttnMaps rm,
                                                      const bf16 *__restrict__ Q, const int32_t *__restrict__ sel,
                                                      const int32_t *__restrict__ pairs, const int4 *__restrict__ work,
                                                      const int32_t *__restrict__ nwork, bf16 *part_o, float2 *part_ml,
                                                      int *done, int *ticket, bf16 *__restrict__ O,
                                                      unsigned long long *__restrict__ counters, int S, int H, int R,
                                                      int L, int wcap, float scale_log2, int bh0, int ng) {
    using Lay = AttendWs<D, BS, NK>;
    static_assert(Lay::supported, "tile shape");
    constexpr int QB = Lay::QB, KVB = Lay::KVB, STAGE = Lay::STAGE, NST = Lay::NST;
    constexpr int RKB = BS * D * 2;  // a remote block's K (or V) tile
    constexpr int CH = D * 2 / 16;
    extern __shared__ __align__(1024) uint8_t smem[];
    int *s_ph = (int *)(smem + Lay::PH_OFF);
    int *s_nr = (int *)(smem + Lay::NR_OFF);
    uint64_t *bars = (uint64_t *)(smem + Lay::BAR_OFF);
    uint64_t *full = bars, *empty = bars + NST, *s_full = bars + 2 * NST, *p_full = s_full + 2, *o_full = s_full + 4,
             *t_free = s_full + 6, *drain = s_full + 8;
    uint32_t *tmem_base = (uint32_t *)(bars + Lay::NBAR);
    volatile int *abort_flag = (volatile int *)(tmem_base + 1);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = (S + 127) / 128;
    auto stage_q = [&](int s) { return smem + s * STAGE; };
    auto stage_rec = [&](int s) { return (int *)(smem + s * STAGE + QB + 2 * KVB); };  // [128] ids, kind, slice, n|t0
    pdl_wait();  // the work items, pair ids, done counters and ticket are ready

    if (tid == 0) {
        int acc = 0;
        for (int k = 0; k <= ng; ++k) {
            s_ph[k] = acc;
            if (k < ng) { s_nr[k] = nwork[bh0 + k]; acc += s_nr[k]; }
            if (k >= 1) acc += ntiles;
        }
        s_ph[ng + 1] = acc;
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(&full[s], 32 + 1);  // every producer lane + the transaction
            tc::mbar_init(&empty[s], 1 + 4);  // the MMA issuer + the group's four warps
        }
        for (int g = 0; g < 2; ++g) {
            tc::mbar_init(&s_full[g], 1);
            tc::mbar_init(&p_full[g], 4);
            tc::mbar_init(&o_full[g], 1);
            tc::mbar_init(&t_free[g], 4);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const int total = s_ph[ng + 1];
    bool ok = true;
    auto fail = [&]() {
        ok = false;
        *abort_flag = 1;
    };
    // item f: (remote?, slice within the group, index within the slice's remote items or tiles)
    auto item_of = [&](int f, bool &remote, int &g, int &idx) {
        int lo = 0, hi = ng + 1;  // last phase k with s_ph[k] <= f
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_ph[mid] <= f) lo = mid;
            else hi = mid;
        }
        const int u = f - s_ph[lo];
        const int nr = lo < ng ? s_nr[lo] : 0;
        remote = u < nr;
        g = remote ? lo : lo - 1;
        idx = remote ? u : u - nr;
    };

    if (warp == 0) {
        // ---------------- producer (the whole warp) ----------------
        int last_v[NST];
#pragma unroll
        for (int s = 0; s < NST; ++s) last_v[s] = -1;
        int ends = 0;  // end records written (one per softmax group)
        for (int i = 0; ends < 2 && ok; ++i) {
            const int s = i % NST, v = i / NST;
            if (v > 0 && !__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&empty[s], (v - 1) & 1, abort_flag))) {
                fail();
                break;
            }
            int f = 0;
            if (lane == 0 && ends == 0) f = atomicAdd(ticket, 1);
            f = ends ? total : __shfl_sync(0xffffffffu, f, 0);
            uint8_t *sQ = stage_q(s), *sK = sQ + QB, *sV = sK + KVB;
            int *rec = stage_rec(s);
            if (f >= total) {
                // no item left: an end record for the softmax group of this slot
                if (lane == 0) rec[128] = 2;
                __syncwarp();
                tc::mbar_arrive(&full[s]);
                if (lane == 0) tc::mbar_arrive(&full[s]);
                last_v[s] = v;
                ++ends;
                continue;
            }
            bool remote;
            int g, idx;
            item_of(f, remote, g, idx);
            const int bh = bh0 + g;
            if (remote) {
                const int4 w = work[(size_t)bh * wcap + idx];
                const int j = w.x, p0 = w.y, cnt = w.z;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int row = lane + 32 * k;
                    const bool live = row < cnt;
                    const int pr = live ? pairs[(size_t)bh * S * R + p0 + row] : -1;
                    rec[row] = pr;
                    const bf16 *qrow = Q + ((size_t)bh * S + (live ? pr / R : 0)) * D;
#pragma unroll
                    for (int c = 0; c < CH; ++c) tc::cp_async16(sQ + tc::kmajor_chunk(row, c, D), qrow + 8 * c, live);
                }
                if (lane == 0) { rec[128] = 1; rec[129] = g; rec[130] = cnt; }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(&full[s]))
                             : "memory");
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_expect_tx(&full[s], 2 * RKB);
#pragma unroll
                    for (int a = 0; a < D / 64; ++a) {
                        tc::tma_load_3d(sK + a * (BS * 128), &rm.k, 64 * a, j * BS, bh, &full[s]);
                        tc::tma_load_3d(sV + a * (BS * 128), &rm.v, 64 * a, j * BS, bh, &full[s]);
                    }
                }
            } else {
                const int t0 = idx * 128;
                const int kstart = max(0, t0 / BS - L + 1) * BS;
                if (lane == 0) { rec[128] = 0; rec[129] = g; rec[130] = t0; }
                __syncwarp();
                tc::mbar_arrive(&full[s]);
                if (lane == 0) {
                    tc::mbar_expect_tx(&full[s], QB + 2 * KVB);
#pragma unroll
                    for (int a = 0; a < D / 64; ++a) {
                        tc::tma_load_3d(sQ + a * (128 * 128), &lm.q, 64 * a, t0, bh, &full[s]);
                        tc::tma_load_3d(sK + a * (NK * 128), &lm.k, 64 * a, kstart, bh, &full[s]);
                        tc::tma_load_3d(sV + a * (NK * 128), &lm.v, 64 * a, kstart, bh, &full[s]);
                    }
                }
            }
            last_v[s] = v;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0)
            for (int s = 0; s < NST; ++s)
                if (last_v[s] >= 0 && !tc::mbar_wait(&full[s], last_v[s] & 1)) ok = false;
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool kind_r[2] = {false, false};  // per group: is its current item remote
            // 1: issued; 0: an end record; -1: gave up
            auto mma1 = [&](int i) -> int {
                const int s = i % NST, v = i / NST, g = i & 1, u = i >> 1;
                if (!tc::mbar_wait_or_abort(&full[s], v & 1, abort_flag)) return -1;
                tc::fence_after_sync();
                const int kind = stage_rec(s)[128];
                if (kind == 2) return 0;
                if (u > 0 && !tc::mbar_wait_or_abort(&t_free[g], (u - 1) & 1, abort_flag)) return -1;
                tc::fence_smem_to_async();
                tc::fence_after_sync();
                const bool remote = kind != 0;
                kind_r[g] = remote;
                const uint32_t aq = tc::smem_u32(stage_q(s)), bk = aq + QB;
                if (remote) {
                    const uint32_t id1 = tc::idesc_bf16(128, BS);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        tc::mma_bf16(tmem + g * 256, tc::desc_kmajor(aq + 256 * kk, D),
                                     tc::desc_sw128(bk + (kk >> 2) * (BS * 128) + (kk & 3) * 32), id1, kk > 0);
                } else {
                    const uint32_t id1 = tc::idesc_bf16(128, NK);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        tc::mma_bf16(tmem + g * 256, tc::desc_sw128(aq + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
                                     tc::desc_sw128(bk + (kk >> 2) * (NK * 128) + (kk & 3) * 32), id1, kk > 0);
                }
                tc::commit(&s_full[g]);
                return 1;
            };
            auto mma2 = [&](int i) -> bool {
                const int s = i % NST, g = i & 1, u = i >> 1;
                if (!tc::mbar_wait_or_abort(&p_full[g], u & 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t bv = tc::smem_u32(stage_q(s)) + QB + KVB;
                const uint32_t id2 = tc::idesc_bf16(128, D, true);
                if (kind_r[g]) {
#pragma unroll
                    for (int kk = 0; kk < BS / 16; ++kk)
                        tc::mma_bf16_ts(tmem + g * 256 + Lay::O_COL, tmem + g * 256 + 8 * kk,
                                        tc::desc_sw128_mn(bv + 2048 * kk, BS * 128), id2, kk > 0);
                } else {
#pragma unroll
                    for (int kk = 0; kk < NK / 16; ++kk)
                        tc::mma_bf16_ts(tmem + g * 256 + Lay::O_COL, tmem + g * 256 + 8 * kk,
                                        tc::desc_sw128_mn(bv + 2048 * kk, NK * 128), id2, kk > 0);
                }
                tc::commit(&o_full[g]);
                tc::commit(&empty[s]);
                return true;
            };
            int r = mma1(0);
            if (r < 0) fail();
            for (int i = 0; r > 0 && ok; ++i) {
                const int r1 = mma1(i + 1);
                if (r1 < 0) { fail(); break; }
                if (!mma2(i)) { fail(); break; }
                r = r1;
            }
            tc::commit(drain);
            if (!tc::mbar_wait(drain, 0)) ok = false;
        }
    } else {
        // ---------------- softmax groups ----------------
        const int g = (warp - 2) >> 2, quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t tS = tmem + g * 256 + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tO = tS + Lay::O_COL;
        for (int i = g; ok; i += 2) {
            const int s = i % NST, v = i / NST, u = i >> 1;
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&full[s], v & 1, abort_flag))) { fail(); break; }
            const int *rec = stage_rec(s);
            if (rec[128] == 2) break;  // the end record of this group
            const bool remote = rec[128] != 0;
            const int sg = rec[129];
            const int pr = remote ? rec[row] : -1;
            const int t0 = remote ? 0 : rec[130];
            const long long bh = bh0 + sg;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[s]);
            float vv[32];
            if (remote) {
                if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&s_full[g], u & 1, abort_flag))) { fail(); break; }
                tc::fence_after_sync();
                float m = -INFINITY;
#pragma unroll
                for (int c0 = 0; c0 < BS; c0 += 32) {
                    __syncwarp();
                    tc::tmem_ld32(tS + c0, vv);
#pragma unroll
                    for (int k = 0; k < 32; ++k) m = fmaxf(m, vv[k]);
                }
                const float m2 = m * scale_log2;
                float l = 0.f;
#pragma unroll
                for (int c0 = 0; c0 < BS; c0 += 32) {
                    __syncwarp();
                    tc::tmem_ld32(tS + c0, vv);
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float a = exp2f(fmaf(vv[2 * k], scale_log2, -m2));
                        const float bb = exp2f(fmaf(vv[2 * k + 1], scale_log2, -m2));
                        l += a + bb;
                        pk[k] = pack2(a, bb);
                    }
                    __syncwarp();
                    tc::tmem_st16(tS + (c0 >> 1), pk);
                }
                __syncwarp();
                tc::tmem_st_wait();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&p_full[g]);
                const float inv = 1.f / l;
                if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&o_full[g], u & 1, abort_flag))) { fail(); break; }
                tc::fence_after_sync();
                const bool live = pr >= 0;
                const size_t slot = (size_t)bh * S * R + (live ? pr : 0);
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    __syncwarp();
                    tc::tmem_ld32(tO + c0, vv);
                    if (live) {
                        uint4 *dst = (uint4 *)(part_o + slot * D + c0);
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8)
                            dst[q8] = make_uint4(pack2(vv[8 * q8] * inv, vv[8 * q8 + 1] * inv),
                                                 pack2(vv[8 * q8 + 2] * inv, vv[8 * q8 + 3] * inv),
                                                 pack2(vv[8 * q8 + 4] * inv, vv[8 * q8 + 5] * inv),
                                                 pack2(vv[8 * q8 + 6] * inv, vv[8 * q8 + 7] * inv));
                    }
                }
                if (live) part_ml[slot] = make_float2(m2, l);
                __threadfence();   // this warp's partial rows are visible before its count
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    atomicAdd(&done[bh], 1);
                    tc::mbar_arrive(&t_free[g]);
                }
                continue;
            }
            // ---- a local tile: rows t0 .. t0 + 127 of slice sg ----
            const int b = (int)(bh / H), h = (int)(bh % H);
            const int kstart = max(0, t0 / BS - L + 1) * BS;
            const int t = t0 + row;
            const bool live = t < S;
            // this row's remote blocks; their partials once the slice's remote items are all done
            int jr[RMAX];
            float2 ml[RMAX];
            bool waited = true;
            {
                const int need = 4 * s_nr[sg];
                bool got = lane != 0;
                if (lane == 0)
                    for (uint32_t it = 0; it < (1u << 22) && !*abort_flag; ++it) {
                        if (ld_acquire(&done[bh]) >= need) { got = true; break; }
                        __nanosleep(64);
                    }
                waited = __all_sync(0xffffffffu, got);
            }
            if (!waited) { fail(); break; }
            (void)ld_acquire(&done[bh]);  // each lane's own acquire of the partials the count covers
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                jr[r] = -1;
                ml[r] = make_float2(0.f, 0.f);
                const int j = (r < R && live) ? sel[((size_t)bh * S + t) * R + r] : -1;
                if (!sel_valid(j, t, BS, L)) continue;
                jr[r] = j;
                ml[r] = ld_cg_f2(part_ml + ((size_t)bh * S + t) * R + r);
            }
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&s_full[g], u & 1, abort_flag))) { fail(); break; }
            tc::fence_after_sync();
            const int lo = max(0, t / BS - L + 1) * BS;
            const int vlo = lo - kstart, vhi = t - kstart;
            float m = -INFINITY;
#pragma unroll 1
            for (int c0 = 0; c0 < NK; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tS + c0, vv);
                if (c0 + 31 < vlo || c0 > vhi) continue;
                if (c0 >= vlo && c0 + 31 <= vhi) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) m = fmaxf(m, vv[k]);
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (c0 + k >= vlo && c0 + k <= vhi) m = fmaxf(m, vv[k]);
                }
            }
            const float m2 = (m == -INFINITY) ? 0.f : m * scale_log2;
            float l = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < NK; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tS + c0, vv);
                uint32_t pk[16];
                if (c0 + 31 < vlo || c0 > vhi) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = 0u;
                } else {
                    const bool full_chunk = c0 >= vlo && c0 + 31 <= vhi;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float a = exp2f(fmaf(vv[2 * k], scale_log2, -m2));
                        float bb = exp2f(fmaf(vv[2 * k + 1], scale_log2, -m2));
                        if (!full_chunk) {
                            a = (c0 + 2 * k >= vlo && c0 + 2 * k <= vhi) ? a : 0.f;
                            bb = (c0 + 2 * k + 1 >= vlo && c0 + 2 * k + 1 <= vhi) ? bb : 0.f;
                        }
                        l += a + bb;
                        pk[k] = pack2(a, bb);
                    }
                }
                __syncwarp();
                tc::tmem_st16(tS + (c0 >> 1), pk);
            }
            __syncwarp();
            tc::tmem_st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&p_full[g]);
            // merge with the remote partials (max/sum rescaling)
            float mm = m2;
#pragma unroll
            for (int r = 0; r < RMAX; ++r)
                if (jr[r] >= 0) mm = fmaxf(mm, ml[r].x);
            const float wl = exp2f(m2 - mm);
            float den = l * wl;
            float wr[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                wr[r] = 0.f;
                if (jr[r] >= 0) {
                    wr[r] = ml[r].y * exp2f(ml[r].x - mm);
                    den += wr[r];
                }
            }
            const float inv = 1.f / den;
            if (!__all_sync(0xffffffffu, tc::mbar_wait_or_abort(&o_full[g], u & 1, abort_flag))) { fail(); break; }
            tc::fence_after_sync();
            bf16 *orow = O + (((size_t)b * S + t) * H + h) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                __syncwarp();
                tc::tmem_ld32(tO + c0, vv);
                if (live) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) vv[k] *= wl;
#pragma unroll
                    for (int r = 0; r < RMAX; ++r) {
                        if (jr[r] < 0) continue;
                        const uint8_t *src = (const uint8_t *)(part_o + (((size_t)bh * S + t) * R + r) * D + c0);
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            const uint4 u4 = ld_cg16(src + 16 * q8);
                            const __nv_bfloat162 *h2 = (const __nv_bfloat162 *)&u4;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 fv = __bfloat1622float2(h2[e]);
                                vv[8 * q8 + 2 * e] = fmaf(wr[r], fv.x, vv[8 * q8 + 2 * e]);
                                vv[8 * q8 + 2 * e + 1] = fmaf(wr[r], fv.y, vv[8 * q8 + 2 * e + 1]);
                            }
                        }
                    }
                    uint4 *dst = (uint4 *)(orow + c0);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        dst[q8] = make_uint4(pack2(vv[8 * q8] * inv, vv[8 * q8 + 1] * inv),
                                             pack2(vv[8 * q8 + 2] * inv, vv[8 * q8 + 3] * inv),
                                             pack2(vv[8 * q8 + 4] * inv, vv[8 * q8 + 5] * inv),
                                             pack2(vv[8 * q8 + 6] * inv, vv[8 * q8 + 7] * inv));
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&t_free[g]);
        }
    }
    if (!ok) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
bool attend_tc_supported(const mono_config &c) {
    if (c.dtype != MONO_BF16 || (c.d != 64 && c.d != 128) || (c.Bs != 64 && c.Bs != 128)) return false;
    const int nk = 128 + (c.L - 1) * c.Bs;
    return nk <= 256;
}

// CTAs that are resident at once on the current device (SMs x CTAs per SM), for
// persistent kernels.  CTAs per SM = the tightest of the thread, register and
// shared-memory limits of an SM (2048 threads, 64K registers, 228 KB of
// shared memory with 1 KB reserved per CTA).
template <typename F>
static cudaError_t persistent_grid(F kernel, int threads, size_t smem, int *out) {
    int dev = 0, sms = 0;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
        return e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
    const int regs_per_warp = ((fa.numRegs * 32 + 255) / 256) * 256;
    const int by_threads = 2048 / threads;
    const int by_regs = 65536 / (regs_per_warp * (threads / 32));
    const int by_smem = (int)((228 * 1024) / (smem + fa.sharedSizeBytes + 1024));
    *out = sms * std::max(1, std::min(by_threads, std::min(by_regs, by_smem)));
    return cudaSuccess;
}

// [B*H, S, D] bf16 tensor, boxes of 64 columns x box_rows rows x 1 slice, 128-byte swizzle
static bool make_map_3d(CUtensorMap *map, const void *ptr, int D, int S, int BH, int box_rows) {
    auto enc = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// a kernel launched so that it may start while the kernel before it on the
// stream still runs (it waits for its predecessor itself: pdl_wait)
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, (KArgs)args...);
}

template <int D, int BS, int NK, int RMAX>
static cudaError_t launch_tc_shape(const Plan &p, const bf16 *Q, const bf16 *K, const bf16 *V, const int32_t *sel,
                                   bf16 *O, void *ws, cudaStream_t s, int parts) {
    const mono_config &c = p.cfg;
    unsigned long long *cnt_err = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.d));
    const int nbh = c.B * c.H * p.nb;
    cudaError_t e;
    AttnMaps lmaps, rmaps;
    if (!make_map_3d(&lmaps.q, Q, D, c.S, c.B * c.H, 128) || !make_map_3d(&lmaps.k, K, D, c.S, c.B * c.H, NK) ||
        !make_map_3d(&lmaps.v, V, D, c.S, c.B * c.H, NK) || !make_map_3d(&rmaps.q, Q, D, c.S, c.B * c.H, 128) ||
        !make_map_3d(&rmaps.k, K, D, c.S, c.B * c.H, BS) || !make_map_3d(&rmaps.v, V, D, c.S, c.B * c.H, BS))
        return cudaErrorInvalidValue;
    constexpr size_t rsmem = RemoteSmem<D, BS>::BYTES;
    // the warp-specialised remote kernel where its ring fits, else the two-stage one
    constexpr bool kRemoteWs = RemoteWs<D, BS>::supported && !MONO_REMOTE_TWO_STAGE;
    if (c.R > 0 && (parts & kAttendPairs)) {
        int32_t *pc = (int32_t *)ws_ptr(p, ws, kRegPairCount);
        int32_t *ps = (int32_t *)ws_ptr(p, ws, kRegPairStart);
        int32_t *pf = (int32_t *)ws_ptr(p, ws, kRegPairFill);
        int32_t *pairs = (int32_t *)ws_ptr(p, ws, kRegPairs);
        int4 *work = (int4 *)ws_ptr(p, ws, kRegWork);
        int32_t *nwork = (int32_t *)ws_ptr(p, ws, kRegNWork);
        int *done = (int *)ws_ptr(p, ws, kRegDone);
        const int nbhh = c.B * c.H;
        const int wcap = p.max_work;  // work items per (b, h)
        const int grp = std::min(kMaxGroup, nbhh);
        if ((e = cudaMemsetAsync(pc, 0, (size_t)nbh * 4, s)) != cudaSuccess) return e;
        dim3 gq((c.S + kQTile - 1) / kQTile, nbhh);
        const size_t hs = (size_t)p.nb * 4;
        if (2 * hs > 48 * 1024) {
            if ((e = cudaFuncSetAttribute(k_pair_count, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hs)) ||
                (e = cudaFuncSetAttribute(k_pair_fill, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * hs))))
                return e;
        }
        k_pair_count<<<gq, 256, hs, s>>>(sel, pc, c.S, c.R, p.nb, c.Bs, c.L, cnt_err);
        if ((e = launch_pdl(k_pair_scan, dim3(nbhh), dim3(1024), 0, s, (const int32_t *)pc, ps, pf, work, nwork, done,
                            done + nbhh, p.nb, wcap, grp)) != cudaSuccess)
            return e;
        if ((e = launch_pdl(k_pair_fill, gq, dim3(256), 2 * hs, s, sel, (const int32_t *)ps, pf, pairs, c.S, c.R, p.nb,
                            c.Bs, c.L)) != cudaSuccess)
            return e;
        count_launches(1);
        count_launches(2);
    }
    if (c.R > 0 && (parts & kAttendRemote)) {
        if constexpr (kRemoteWs) {
            if ((e = cudaFuncSetAttribute(k_remote_ws<D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)RemoteWs<D, BS>::BYTES)) != cudaSuccess)
                return e;
        } else if ((e = cudaFuncSetAttribute(k_remote_tc<D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)rsmem)) != cudaSuccess) {
            return e;
        }
    }
    // the local part: the warp-specialised kernel where its stages and tensor
    // memory fit, else the single-stage one
    constexpr bool ws_local = LocalWs<D, NK>::supported;
    const size_t smem = ws_local ? (size_t)LocalWs<D, NK>::BYTES : local_smem<D, NK>();
    auto kl = k_local_merge_tc<D, BS, NK, RMAX>;
    int local_ctas = 0;
    if constexpr (ws_local) {
        if ((e = cudaFuncSetAttribute(k_local_ws<D, BS, NK, RMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&local_ctas, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
    } else {
        if ((e = cudaFuncSetAttribute(kl, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
            return e;
        if ((e = persistent_grid(kl, 256, smem, &local_ctas)) != cudaSuccess) return e;
    }
    // Remote then local, over as many (b, h) slices per launch as the remote
    // kernel's per-group table holds (kMaxGroup).  One launch pair over all
    // slices measured faster than groups sized to keep their partials in L2
    // (attention at S = 32768, 16 heads: 275 us in one group, 327 us in four):
    // fewer launch tails, and the remote kernel balances more work items.
    int remote_ctas = 0;
    if (c.R > 0) {
        if constexpr (kRemoteWs) {
            int dev = 0;
            if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
                (e = cudaDeviceGetAttribute(&remote_ctas, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
                return e;
        } else if ((e = persistent_grid(k_remote_tc<D, BS>, 256, rsmem, &remote_ctas)) != cudaSuccess) {
            return e;
        }
    }
    const int nbhh = c.B * c.H;
    const int group = c.R > 0 ? std::min(kMaxGroup, nbhh) : nbhh;
    // all stages at once: the fused kernel per group of slices where it applies and is selected
    constexpr bool kFused = AttendWs<D, BS, NK>::supported && MONO_ATTEND_FUSED;
    if constexpr (kFused) {
        if (c.R > 0 && (parts & kAttendRemote) && (parts & kAttendLocal)) {
            constexpr size_t fsmem = AttendWs<D, BS, NK>::BYTES;
            auto kf = k_attend_ws<D, BS, NK, RMAX>;
            if ((e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem)) != cudaSuccess)
                return e;
            // [B*H] done counts, then one ticket per launch group: cleared by k_pair_scan
            int *done = (int *)ws_ptr(p, ws, kRegDone);
            int dev = 0, sms = 0;
            if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
                (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
                return e;
            for (int g0 = 0; g0 < nbhh; g0 += group) {
                const int ng = std::min(group, nbhh - g0);
                if ((e = launch_pdl(kf, dim3(sms), dim3(320), fsmem, s, lmaps, rmaps, Q, sel,
                                    (const int32_t *)ws_ptr(p, ws, kRegPairs), (const int4 *)ws_ptr(p, ws, kRegWork),
                                    (const int32_t *)ws_ptr(p, ws, kRegNWork), (bf16 *)ws_ptr(p, ws, kRegPartO),
                                    (float2 *)ws_ptr(p, ws, kRegPartML), done, done + nbhh + g0 / group, O, cnt_err,
                                    c.S, c.H, c.R, c.L, p.max_work, scale_log2, g0, ng)) != cudaSuccess)
                    return e;
                count_launches(1);
            }
            return cudaSuccess;
        }
    }
    // remote then local per group of slices; one stage at a time: over every group
    const bool both = (parts & kAttendRemote) && (parts & kAttendLocal);
    for (int pass = 0; pass < (both ? 1 : 2); ++pass)
    for (int g0 = 0; g0 < nbhh; g0 += group) {
        const int ng = std::min(group, nbhh - g0);
        const bool do_remote = (parts & kAttendRemote) && (both || pass == 0);
        const bool do_local = (parts & kAttendLocal) && (both || pass == 1);
        if (c.R > 0 && do_remote) {
            if constexpr (kRemoteWs)
                k_remote_ws<D, BS><<<remote_ctas, RemoteWs<D, BS>::THREADS, RemoteWs<D, BS>::BYTES, s>>>(
                    rmaps, Q, (const int32_t *)ws_ptr(p, ws, kRegPairs), (const int4 *)ws_ptr(p, ws, kRegWork),
                    (const int32_t *)ws_ptr(p, ws, kRegNWork), (bf16 *)ws_ptr(p, ws, kRegPartO),
                    (float2 *)ws_ptr(p, ws, kRegPartML), cnt_err, c.S, c.R, p.max_work, scale_log2, g0, ng);
            else
                k_remote_tc<D, BS><<<remote_ctas, 256, rsmem, s>>>(
                    rmaps, Q, (const int32_t *)ws_ptr(p, ws, kRegPairs), (const int4 *)ws_ptr(p, ws, kRegWork),
                    (const int32_t *)ws_ptr(p, ws, kRegNWork), (bf16 *)ws_ptr(p, ws, kRegPartO),
                    (float2 *)ws_ptr(p, ws, kRegPartML), cnt_err, c.S, c.R, p.max_work, scale_log2, g0, ng);
            count_launches(1);
        }
        if (!do_local) continue;
        if constexpr (ws_local) {
            const int tiles = ng * ((c.S + 127) / 128);
            k_local_ws<D, BS, NK, RMAX><<<std::min(local_ctas, tiles), 320, smem, s>>>(
                lmaps, sel, (const bf16 *)ws_ptr(p, ws, kRegPartO), (const float2 *)ws_ptr(p, ws, kRegPartML), O,
                cnt_err, c.S, c.H, c.R, c.L, scale_log2, g0, ng);
        } else {
            kl<<<local_ctas, 256, smem, s>>>(lmaps, sel, (const bf16 *)ws_ptr(p, ws, kRegPartO),
                                             (const float2 *)ws_ptr(p, ws, kRegPartML), O, cnt_err, c.S, c.H, c.R,
                                             c.L, scale_log2, g0, ng);
        }
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_attend_tc(const Plan &p, const void *Q, const void *K, const void *V, const int32_t *sel, void *O,
                             void *ws, cudaStream_t s, int parts) {
    const mono_config &c = p.cfg;
    const bf16 *q = (const bf16 *)Q, *k = (const bf16 *)K, *v = (const bf16 *)V;
    bf16 *o = (bf16 *)O;
    const int nk = 128 + (c.L - 1) * c.Bs;
    // NK = the local key range rounded up to a multiple of 32 (MMA N <= 256)
#define MONO_TC(DD, BB, NN)                                                                                     \
    do {                                                                                                        \
        if (c.R <= 2) return launch_tc_shape<DD, BB, NN, 2>(p, q, k, v, sel, o, ws, s, parts);                  \
        if (c.R <= 4) return launch_tc_shape<DD, BB, NN, 4>(p, q, k, v, sel, o, ws, s, parts);                  \
        return launch_tc_shape<DD, BB, NN, kMaxR>(p, q, k, v, sel, o, ws, s, parts);                            \
    } while (0)
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

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
// lets its successor's CTAs start at once (tc::grid_dep_launch), and each
// waits for its predecessor's results only before reading them
// (tc::grid_dep_wait; without a programmatic launch the wait returns at once).

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
// queries.  grid B*H, 1024 threads.
__global__ void __launch_bounds__(1024) k_pair_scan(const int32_t *__restrict__ cnt, int32_t *__restrict__ start,
                                                    int32_t *__restrict__ fill, int4 *__restrict__ work,
                                                    int32_t *__restrict__ nwork, int nb, int wcap) {
    __shared__ int s_w[32], s_c[32];
    __shared__ int carry_p, carry_c;
    tc::grid_dep_launch();
    const long long bh = blockIdx.x;
    if (threadIdx.x == 0) {
        carry_p = 0;
        carry_c = 0;
    }
    tc::grid_dep_wait();  // the counts are complete
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
    tc::grid_dep_launch();
    const long long bh = blockIdx.y;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s_h[j] = 0;
    tc::grid_dep_wait();  // the bucket starts and cleared cursors
    __syncthreads();
    const int t0 = blockIdx.x * kQTile, t1 = min(S, t0 + kQTile);
    // two passes over the tile's selections: count per block, then place each pair at its block's global
    // offset plus a shared cursor (no per-thread pair arrays, which would sit in local memory)
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x)
        for (int r = 0; r < R; ++r) {
            const int j = sel[((size_t)bh * S + t) * R + r];
            if (sel_valid(j, t, Bs, L)) atomicAdd(&s_h[j], 1);
        }
    __syncthreads();
    for (int j = threadIdx.x; j < nb; j += blockDim.x) {
        const int c = s_h[j];
        if (c) s_base[j] = start[bh * nb + j] + atomicAdd(&fill[bh * nb + j], c);
        s_h[j] = 0;
    }
    __syncthreads();
    int32_t *seg = pairs + (size_t)bh * S * R;
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x)
        for (int r = 0; r < R; ++r) {
            const int j = sel[((size_t)bh * S + t) * R + r];
            if (sel_valid(j, t, Bs, L)) seg[s_base[j] + atomicAdd(&s_h[j], 1)] = t * R + r;
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

// a and b as two bf16 terms each: hi = bf16(v), lo = bf16(v - hi) (16 significant bits together)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    hi = *(const uint32_t *)&h;
    lo = pack2(a - hf.x, b - hf.y);
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
// gathered query rows by cp.async, eight threads per 128-byte row segment, in
// the same 128-byte swizzled layout (a ring of the items' pair ids in shared
// memory tells each thread its rows).  Per item: S = Q_sel K_j^T and
// O = P V_j on tcgen05 (TMEM, 64 or 128 columns reused by every item),
// softmax in fp32, one partial per pair: the rows go through shared memory
// (swizzled) so that every store writes whole 128-byte lines.  As in the
// local kernel, warps q and q+4 share TMEM lane quarter q and split the
// columns.
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
    static constexpr int PR_OFF = PREF_OFF + ((kMaxGroup + 1) * 4 + 15) / 16 * 16;  // int [3][128] pair-id ring
    static constexpr int BAR_OFF = PR_OFF + 3 * 128 * 4;           // 3 mbarriers + TMEM base
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
    int(*s_pr)[128] = (int(*)[128])(smem + L::PR_OFF);  // pair ids of item k at s_pr[k % 3]
    uint64_t *bar_kv = (uint64_t *)(smem + L::BAR_OFF);  // [2]: K/V of each stage landed
    uint64_t *mbar = bar_kv + 2;                          // MMA completion
    uint32_t *tmem_base = (uint32_t *)(mbar + 1);
    tc::grid_dep_launch();  // the local kernel may start; it waits for the partials itself
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {  // uniform; TMA's 128-byte swizzle needs 1024-byte aligned tiles
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;

    tc::grid_dep_wait();  // the work items and pair ids (pair kernels) are complete
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
    // 16-byte chunk c of row r of a [128, D] bf16 tile in 64-column slabs of
    // 128-byte rows, chunks swizzled by (r mod 8): the layout of a TMA tile
    // with 128-byte swizzle
    auto sw_off = [](int r, int c) { return (uint32_t)((c >> 3) * (128 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4)); };
    auto issue = [&](int stage, const RemoteItem &it, const int *prs) {
        uint8_t *sQ = smem + stage * STAGE, *sK = sQ + QB, *sV = sK + KB;
        if (tid == 0) {
            tc::mbar_expect_tx(&bar_kv[stage], 2 * KB);
#pragma unroll
            for (int a = 0; a < D / 64; ++a) {
                tc::tma_load_3d(sK + a * (BS * 128), &maps.k, 64 * a, it.j * BS, (int)it.bh, &bar_kv[stage]);
                tc::tma_load_3d(sV + a * (BS * 128), &maps.v, 64 * a, it.j * BS, (int)it.bh, &bar_kv[stage]);
            }
        }
        constexpr int CPR = D / 8;  // chunks per row
#pragma unroll
        for (int k = 0; k < 128 * CPR / 256; ++k) {
            const int idx = tid + 256 * k, r = idx / CPR, c = idx % CPR;
            const bool live = r < it.n;
            const bf16 *src = live ? Q + ((size_t)it.bh * S + prs[r] / R) * D + 8 * c : Q;
            tc::cp_async16(sQ + sw_off(r, c), src, live);
        }
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
        int f1 = f + G;
        bool have1 = f1 < total;
        RemoteItem it1{};
        int pr1 = 0;
        if (have1) { it1 = descr(f1); pr1 = pair_of(it1); }
        if (half == 0) {
            s_pr[0][row] = pr0;
            s_pr[1][row] = pr1;
        }
        __syncthreads();
        issue(0, it0, s_pr[0]);
        pend[0] = 0;
        for (int k = 0; ok; ++k) {
            const int stage = k & 1;
            const uint32_t kv_parity = (k >> 1) & 1;  // completions of bar_kv[stage] so far, mod 2
            if (have1) {
                issue(stage ^ 1, it1, s_pr[(k + 1) % 3]);
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
                    tc::mma_bf16(tmem, tc::desc_sw128(aq + (kk >> 2) * (128 * 128) + (kk & 3) * 32),
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
                        const float a = tc::ex2_fast(fmaf(v[8 * q8 + 2 * u], scale_log2, -m2));
                        const float bb = tc::ex2_fast(fmaf(v[8 * q8 + 2 * u + 1], scale_log2, -m2));
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
            if (half == 0) s_pr[(k + 2) % 3][row] = pr2;
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
            const size_t base = (size_t)it0.bh * S * R;
            const float inv = 1.f / l;
            // this row's partial, bf16, into shared memory over P (free once the P V MMA has completed)
#pragma unroll
            for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
                tc::tmem_ld32(trow + c0, v);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    *(uint4 *)(sP + sw_off(row, (c0 >> 3) + q8)) =
                        make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv),
                                   pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                   pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv),
                                   pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
            }
            if (live && ok && half == 0) part_ml[base + pr0] = make_float2(m2, l);
            __syncthreads();
            // the rows out, eight threads per 128-byte line of a row
            if (ok) {
                constexpr int CPR = D / 8;
                const int *prs = s_pr[k % 3];
#pragma unroll
                for (int kq = 0; kq < 128 * CPR / 256; ++kq) {
                    const int idx = tid + 256 * kq, r = idx / CPR, c = idx % CPR;
                    if (r < it0.n)
                        *(uint4 *)(part_o + (base + prs[r]) * D + 8 * c) = *(const uint4 *)(sP + sw_off(r, c));
                }
            }
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
                    float a = tc::ex2_fast(fmaf(v[i], scale_log2, -m2));
                    float bb = tc::ex2_fast(fmaf(v[i + 1], scale_log2, -m2));
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
                                                     float *__restrict__ o32, float *__restrict__ lse_out,
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
        tc::grid_dep_wait();  // the remote partials (remote kernel) are complete
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
                    for (int q8 = 0; q8 < D / 8; q8 += 2)  // 32-byte loads (the rows are 128-byte aligned)
                        tc::ldg_v8(part_o + pq * D + 8 * q8, pre[r < kPre ? r : 0][q8], pre[r < kPre ? r : 0][q8 + 1]);
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
                        float a = tc::ex2_fast(fmaf(v[2 * k], scale_log2, -m2));
                        float bb = tc::ex2_fast(fmaf(v[2 * k + 1], scale_log2, -m2));
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
            if (lse_out && live) lse_out[(size_t)bh * S + t] = (mm + log2f(den)) * 0.69314718055994531f;  // ln 2
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
                    if (o32) {
                        float4 *d32 = (float4 *)(o32 + (((size_t)b * S + t) * H + h) * D + c0);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            d32[q4] = make_float4(v[4 * q4] * inv, v[4 * q4 + 1] * inv, v[4 * q4 + 2] * inv,
                                                  v[4 * q4 + 3] * inv);
                    }
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
// stream still runs (it waits for its predecessor itself: tc::grid_dep_wait)
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
                                   bf16 *O, void *ws, cudaStream_t s, int parts, float *o32, float *lse, bool *stats) {
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
    if (c.R > 0 && (parts & kAttendPairs)) {
        int32_t *pc = (int32_t *)ws_ptr(p, ws, kRegPairCount);
        int32_t *ps = (int32_t *)ws_ptr(p, ws, kRegPairStart);
        int32_t *pf = (int32_t *)ws_ptr(p, ws, kRegPairFill);
        int32_t *pairs = (int32_t *)ws_ptr(p, ws, kRegPairs);
        int4 *work = (int4 *)ws_ptr(p, ws, kRegWork);
        int32_t *nwork = (int32_t *)ws_ptr(p, ws, kRegNWork);
        const int nbhh = c.B * c.H;
        const int wcap = p.max_work;  // work items per (b, h)
        if ((e = cudaMemsetAsync(pc, 0, (size_t)nbh * 4, s)) != cudaSuccess) return e;
        dim3 gq((c.S + kQTile - 1) / kQTile, nbhh);
        const size_t hs = (size_t)p.nb * 4;
        if (2 * hs > 48 * 1024) {
            if ((e = cudaFuncSetAttribute(k_pair_count, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hs)) ||
                (e = cudaFuncSetAttribute(k_pair_fill, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * hs))))
                return e;
        }
        k_pair_count<<<gq, 256, hs, s>>>(sel, pc, c.S, c.R, p.nb, c.Bs, c.L, cnt_err);
        if ((e = launch_pdl(k_pair_scan, dim3(nbhh), dim3(1024), 0, s, (const int32_t *)pc, ps, pf, work, nwork, p.nb,
                            wcap)) != cudaSuccess)
            return e;
        if ((e = launch_pdl(k_pair_fill, gq, dim3(256), 2 * hs, s, sel, (const int32_t *)ps, pf, pairs, c.S, c.R, p.nb,
                            c.Bs, c.L)) != cudaSuccess)
            return e;
        count_launches(1);
        count_launches(2);
    }
    if (c.R > 0 && (parts & kAttendRemote)) {
        if ((e = cudaFuncSetAttribute(k_remote_tc<D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem)) !=
            cudaSuccess)
            return e;
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
    if (stats) *stats = ws_local && o32 && lse;
    if (!ws_local) o32 = lse = nullptr;
    // Remote then local, over as many (b, h) slices per launch as the remote
    // kernel's per-group table holds (kMaxGroup).  One launch pair over all
    // slices measured faster than groups sized to keep their partials in L2
    // (attention at S = 32768, 16 heads: 275 us in one group, 327 us in four):
    // fewer launch tails, and the remote kernel balances more work items.
    int remote_ctas = 0;
    if (c.R > 0 && (e = persistent_grid(k_remote_tc<D, BS>, 256, rsmem, &remote_ctas)) != cudaSuccess)
        return e;
    const int nbhh = c.B * c.H;
    const int group = c.R > 0 ? std::min(kMaxGroup, nbhh) : nbhh;
    // remote then local per group of slices; one stage at a time: over every group
    const bool both = (parts & kAttendRemote) && (parts & kAttendLocal);
    for (int pass = 0; pass < (both ? 1 : 2); ++pass)
    for (int g0 = 0; g0 < nbhh; g0 += group) {
        const int ng = std::min(group, nbhh - g0);
        const bool do_remote = (parts & kAttendRemote) && (both || pass == 0);
        const bool do_local = (parts & kAttendLocal) && (both || pass == 1);
        if (c.R > 0 && do_remote) {
            if ((e = launch_pdl(k_remote_tc<D, BS>, dim3(remote_ctas), dim3(256), rsmem, s, rmaps, Q,
                                (const int32_t *)ws_ptr(p, ws, kRegPairs), (const int4 *)ws_ptr(p, ws, kRegWork),
                                (const int32_t *)ws_ptr(p, ws, kRegNWork), (bf16 *)ws_ptr(p, ws, kRegPartO),
                                (float2 *)ws_ptr(p, ws, kRegPartML), cnt_err, c.S, c.R, p.max_work, scale_log2, g0,
                                ng)) != cudaSuccess)
                return e;
            count_launches(1);
        }
        if (!do_local) continue;
        if constexpr (ws_local) {
            const int tiles = ng * ((c.S + 127) / 128);
            if ((e = launch_pdl(k_local_ws<D, BS, NK, RMAX>, dim3(std::min(local_ctas, tiles)), dim3(320), smem, s,
                                lmaps, sel, (const bf16 *)ws_ptr(p, ws, kRegPartO),
                                (const float2 *)ws_ptr(p, ws, kRegPartML), O, o32, lse, cnt_err, c.S, c.H, c.R, c.L,
                                scale_log2, g0, ng)) != cudaSuccess)
                return e;
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

// ---------------------------------------------------------------------------
// backward, local keys, on the tensor cores: for each 128-query tile and its
// local key window (the forward local kernel's tile), with the forward's
// log-sum-exp and D = dO . O of each row given,
//   S  = Q K^T                      (tcgen05, fp32 in TMEM)
//   dP = dO V^T                     (dO as two bf16 terms hi + lo, both products accumulated)
//   P  = exp(S / sqrt(d) - lse),  dS = P (dP - D)   (fp32; causal window mask as in the forward)
//   dQ_local = dS K                 (dS as two bf16 terms from shared memory, K as the MN-major operand)
// dQ_local (fp32, without the 1/sqrt(d) factor) goes to dq_loc [B*H, S, d]; the
// SIMT dQ kernel adds the remote keys' part and applies the factor and RoPE.
// One persistent CTA of 256 threads per SM walks the tiles; TMEM lane quarter
// q is read by warps q and q + 4, each taking half of the columns.
// ---------------------------------------------------------------------------
struct BwdMaps {
    CUtensorMap q, k, v, dohi, dolo;
};

template <int D, int NK>
struct BwdLocalSmem {
    static constexpr int QB = 128 * D * 2, KB = NK * D * 2, PB = 128 * NK * 2;
    static constexpr int Q_OFF = 0, K_OFF = QB, V_OFF = QB + KB, DOH_OFF = QB + 2 * KB, DOL_OFF = 2 * QB + 2 * KB;
    static constexpr int DS_OFF = 3 * QB + 2 * KB, DSL_OFF = DS_OFF + PB;  // dS hi and lo terms
    static constexpr int BAR_OFF = DSL_OFF + PB;                          // 2 mbarriers + TMEM base
    static constexpr int BYTES = BAR_OFF + 32;
    static constexpr bool supported = 2 * NK + D <= 512 && NK % 32 == 0 && D % 64 == 0 && BYTES <= 227 * 1024;
};

template <int D, int BS, int NK>
__global__ void __launch_bounds__(256, 1) k_bwd_local_dq_tc(const __grid_constant__ BwdMaps maps,
                                                            const float *__restrict__ lse,
                                                            const float *__restrict__ dsum, float *__restrict__ dq_loc,
                                                            unsigned long long *__restrict__ counters, int S, int L,
                                                            float scale_log2, int nbh) {
    using Lay = BwdLocalSmem<D, NK>;
    static_assert(Lay::supported, "tile shape");
    constexpr int QB = Lay::QB, KB = Lay::KB, HALF = NK / 2, DH = D / 2;
    static_assert(HALF % 32 == 0 && DH % 32 == 0, "column halves of 32");
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *sQ = smem + Lay::Q_OFF, *sK = smem + Lay::K_OFF, *sV = smem + Lay::V_OFF;
    uint8_t *sDOH = smem + Lay::DOH_OFF, *sDOL = smem + Lay::DOL_OFF, *sDS = smem + Lay::DS_OFF;
    uint8_t *sDSL = smem + Lay::DSL_OFF;
    uint64_t *bar_ld = (uint64_t *)(smem + Lay::BAR_OFF), *mbar = bar_ld + 1;
    uint32_t *tmem_base = (uint32_t *)(bar_ld + 2);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int ntiles = (S + 127) / 128;
    const int total = nbh * ntiles;
    if (warp == 0) {
        tc::tmem_alloc(tmem_base, 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar_ld, 1);
        tc::mbar_init(mbar, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = trow, tP = trow + NK, tQ = trow + 2 * NK;  // S, dP and dQ columns of this lane quarter
    bool ok = true;
    int pend = -1;       // thread 0: the load of tile k issued and not yet seen complete
    uint32_t mph = 0;    // completions of mbar so far, mod 2
    int k = 0;
    for (int f = blockIdx.x; f < total && ok; f += gridDim.x, ++k) {
        const int bh = f / ntiles, t0 = (f % ntiles) * 128;
        const int kstart = max(0, t0 / BS - L + 1) * BS;
        const int nq = min(128, S - t0);
        const int t = t0 + row;
        const bool live = row < nq;
        if (tid == 0) {
            tc::mbar_expect_tx(bar_ld, 3 * QB + 2 * KB);
#pragma unroll
            for (int a = 0; a < D / 64; ++a) {
                tc::tma_load_3d(sQ + a * (128 * 128), &maps.q, 64 * a, t0, bh, bar_ld);
                tc::tma_load_3d(sDOH + a * (128 * 128), &maps.dohi, 64 * a, t0, bh, bar_ld);
                tc::tma_load_3d(sDOL + a * (128 * 128), &maps.dolo, 64 * a, t0, bh, bar_ld);
                tc::tma_load_3d(sK + a * (NK * 128), &maps.k, 64 * a, kstart, bh, bar_ld);
                tc::tma_load_3d(sV + a * (NK * 128), &maps.v, 64 * a, kstart, bh, bar_ld);
            }
            pend = k;
        }
        // this row's log-sum-exp (in the exp2 domain) and D
        const float lse2 = live ? lse[(size_t)bh * S + t] * 1.4426950408889634f : 0.f;
        const float Drow = live ? dsum[(size_t)bh * S + t] : 0.f;
        bool landed = true;
        if (tid == 0) {
            landed = tc::mbar_wait(bar_ld, (uint32_t)(k & 1));
            if (landed) pend = -1;
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(landed);
        tc::fence_after_sync();
        if (!ok) break;
        if (tid == 0) {
            const uint32_t id = tc::idesc_bf16(128, NK);
            const uint32_t aq = tc::smem_u32(sQ), ah = tc::smem_u32(sDOH), al = tc::smem_u32(sDOL);
            const uint32_t bk = tc::smem_u32(sK), bv = tc::smem_u32(sV);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32, bo = (kk >> 2) * (NK * 128) + (kk & 3) * 32;
                tc::mma_bf16(tmem, tc::desc_sw128(aq + ao), tc::desc_sw128(bk + bo), id, kk > 0);
                tc::mma_bf16(tmem + NK, tc::desc_sw128(ah + ao), tc::desc_sw128(bv + bo), id, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32, bo = (kk >> 2) * (NK * 128) + (kk & 3) * 32;
                tc::mma_bf16(tmem + NK, tc::desc_sw128(al + ao), tc::desc_sw128(bv + bo), id, 1u);
            }
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
        // dS over keys s in [lo(t), t]: columns [vlo, vhi]
        const int lo = max(0, t / BS - L + 1) * BS;
        const int vlo = lo - kstart, vhi = t - kstart;
#pragma unroll 1
        for (int c0 = half * HALF; c0 < half * HALF + HALF; c0 += 32) {
            float sv[32], pv[32];
            tc::tmem_ld32(tS + c0, sv);
            tc::tmem_ld32(tP + c0, pv);
            uint32_t hk[16], lk[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = 2 * u;
                const bool in0 = live && c0 + i >= vlo && c0 + i <= vhi;
                const bool in1 = live && c0 + i + 1 >= vlo && c0 + i + 1 <= vhi;
                const float p0 = in0 ? tc::ex2_fast(fmaf(sv[i], scale_log2, -lse2)) : 0.f;
                const float p1 = in1 ? tc::ex2_fast(fmaf(sv[i + 1], scale_log2, -lse2)) : 0.f;
                split2(p0 * (pv[i] - Drow), p1 * (pv[i + 1] - Drow), hk[u], lk[u]);
            }
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                const uint32_t off = tc::kmajor_chunk(row, (c0 >> 3) + q8, NK);
                *(uint4 *)(sDS + off) = make_uint4(hk[4 * q8], hk[4 * q8 + 1], hk[4 * q8 + 2], hk[4 * q8 + 3]);
                *(uint4 *)(sDSL + off) = make_uint4(lk[4 * q8], lk[4 * q8 + 1], lk[4 * q8 + 2], lk[4 * q8 + 3]);
            }
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) {
            const uint32_t id = tc::idesc_bf16(128, D, true);
            const uint32_t ad = tc::smem_u32(sDS), adl = tc::smem_u32(sDSL), bk = tc::smem_u32(sK);
#pragma unroll
            for (int kk = 0; kk < NK / 16; ++kk) {
                const uint64_t bd = tc::desc_sw128_mn(bk + 2048 * kk, NK * 128);
                tc::mma_bf16(tmem + 2 * NK, tc::desc_kmajor(ad + 256 * kk, NK), bd, id, kk > 0);
                tc::mma_bf16(tmem + 2 * NK, tc::desc_kmajor(adl + 256 * kk, NK), bd, id, 1u);
            }
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
#pragma unroll 1
        for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tQ + c0, v);
            if (live) {
                float4 *dst = (float4 *)(dq_loc + ((size_t)bh * S + t) * D + c0);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            }
        }
        tc::fence_before_sync();
        __syncthreads();  // shared memory and TMEM are free for the next tile
        tc::fence_after_sync();
    }
    // leave no TMA write in flight into this CTA's shared memory
    if (tid == 0 && pend >= 0 && !tc::mbar_wait(bar_ld, (uint32_t)(pend & 1))) ok = false;
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}


// ---------------------------------------------------------------------------
// backward, local queries of each key, on the tensor cores (key-major): for
// each tile of 128 keys [k0, k0 + 128) of one head, the NQ = 128 + (L-1) Bs
// queries [k0, k0 + NQ) whose local window holds some of them,
//   S^T  = K Q^T,  dP^T = V dO^T   (dO as two bf16 terms, both products accumulated)
//   P^T  = exp(S^T / sqrt(d) - lse_t),  dS^T = P^T (dP^T - D_t)   (fp32; the window mask of each query)
//   dV_local = P^T dO,  dK_local = dS^T Q   (P^T and dS^T as two bf16 terms each: the hi terms in a first
//                                            round, the lo terms through the same buffers in a second, which
//                                            drops only lo x lo; dO and Q MN-major)
// to dv_loc and dk_loc [B*H, S, d] (fp32, dK without the 1/sqrt(d) factor);
// the SIMT dK/dV kernel adds the selecting queries' part.  Same roles as
// k_bwd_local_dq_tc: one persistent CTA of 256 threads per SM, one MMA thread,
// TMEM lane quarter q read by warps q and q + 4.
// ---------------------------------------------------------------------------
template <int D, int NQ>
struct BwdKvSmem {
    static constexpr int KB = 128 * D * 2, QB = NQ * D * 2, PB = 128 * NQ * 2;
    static constexpr int K_OFF = 0, V_OFF = KB, Q_OFF = 2 * KB, DOH_OFF = 2 * KB + QB, DOL_OFF = 2 * KB + 2 * QB;
    static constexpr int P_OFF = 2 * KB + 3 * QB, DS_OFF = P_OFF + PB;
    static constexpr int LSE_OFF = DS_OFF + PB, DD_OFF = LSE_OFF + NQ * 4;  // per query: lse (exp2 domain), D
    static constexpr int BAR_OFF = DD_OFF + NQ * 4;                         // 2 mbarriers + TMEM base
    static constexpr int BYTES = BAR_OFF + 32;
    static constexpr bool supported =
        2 * NQ + 2 * D <= 512 && NQ % 32 == 0 && NQ <= 256 && D % 64 == 0 && BYTES <= 227 * 1024;
};

template <int D, int BS, int NQ>
__global__ void __launch_bounds__(256, 1) k_bwd_local_dkdv_tc(const __grid_constant__ BwdMaps maps,
                                                              const float *__restrict__ lse,
                                                              const float *__restrict__ dsum,
                                                              float *__restrict__ dk_loc, float *__restrict__ dv_loc,
                                                              unsigned long long *__restrict__ counters, int S, int L,
                                                              float scale_log2, int nbh) {
    using Lay = BwdKvSmem<D, NQ>;
    static_assert(Lay::supported, "tile shape");
    constexpr int KB = Lay::KB, QB = Lay::QB, HALF = NQ / 2, DH = D / 2;
    static_assert(HALF % 32 == 0 && DH % 32 == 0, "column halves of 32");
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *sK = smem + Lay::K_OFF, *sV = smem + Lay::V_OFF, *sQ = smem + Lay::Q_OFF;
    uint8_t *sDOH = smem + Lay::DOH_OFF, *sDOL = smem + Lay::DOL_OFF, *sP = smem + Lay::P_OFF, *sDS = smem + Lay::DS_OFF;
    float *s_lse = (float *)(smem + Lay::LSE_OFF), *s_D = (float *)(smem + Lay::DD_OFF);
    uint64_t *bar_ld = (uint64_t *)(smem + Lay::BAR_OFF), *mbar = bar_ld + 1;
    uint32_t *tmem_base = (uint32_t *)(bar_ld + 2);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int ntiles = (S + 127) / 128;
    const int total = nbh * ntiles;
    if (warp == 0) {
        tc::tmem_alloc(tmem_base, 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar_ld, 1);
        tc::mbar_init(mbar, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    // S^T, dP^T, dV and dK columns of this lane quarter
    const uint32_t tS = trow, tP = trow + NQ, tV = trow + 2 * NQ, tK = trow + 2 * NQ + D;
    bool ok = true;
    int pend = -1;     // thread 0: the load of tile k issued and not yet seen complete
    uint32_t mph = 0;  // completions of mbar so far, mod 2
    int k = 0;
    for (int f = blockIdx.x; f < total && ok; f += gridDim.x, ++k) {
        const int bh = f / ntiles, k0 = (f % ntiles) * 128;
        const int s = k0 + row;  // this thread's key
        const bool live = s < S;
        if (tid == 0) {
            tc::mbar_expect_tx(bar_ld, 2 * KB + 3 * QB);
#pragma unroll
            for (int a = 0; a < D / 64; ++a) {
                tc::tma_load_3d(sK + a * (128 * 128), &maps.k, 64 * a, k0, bh, bar_ld);
                tc::tma_load_3d(sV + a * (128 * 128), &maps.v, 64 * a, k0, bh, bar_ld);
                tc::tma_load_3d(sQ + a * (NQ * 128), &maps.q, 64 * a, k0, bh, bar_ld);
                tc::tma_load_3d(sDOH + a * (NQ * 128), &maps.dohi, 64 * a, k0, bh, bar_ld);
                tc::tma_load_3d(sDOL + a * (NQ * 128), &maps.dolo, 64 * a, k0, bh, bar_ld);
            }
            pend = k;
        }
        // the queries' log-sum-exp (exp2 domain) and D
        for (int c = tid; c < NQ; c += 256) {
            const int t = k0 + c;
            s_lse[c] = t < S ? lse[(size_t)bh * S + t] * 1.4426950408889634f : 0.f;
            s_D[c] = t < S ? dsum[(size_t)bh * S + t] : 0.f;
        }
        bool landed = true;
        if (tid == 0) {
            landed = tc::mbar_wait(bar_ld, (uint32_t)(k & 1));
            if (landed) pend = -1;
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(landed);
        tc::fence_after_sync();
        if (!ok) break;
        if (tid == 0) {
            const uint32_t id = tc::idesc_bf16(128, NQ);
            const uint32_t ak = tc::smem_u32(sK), av = tc::smem_u32(sV);
            const uint32_t bq = tc::smem_u32(sQ), bh_ = tc::smem_u32(sDOH), bl = tc::smem_u32(sDOL);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32, bo = (kk >> 2) * (NQ * 128) + (kk & 3) * 32;
                tc::mma_bf16(tmem, tc::desc_sw128(ak + ao), tc::desc_sw128(bq + bo), id, kk > 0);
                tc::mma_bf16(tmem + NQ, tc::desc_sw128(av + ao), tc::desc_sw128(bh_ + bo), id, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32, bo = (kk >> 2) * (NQ * 128) + (kk & 3) * 32;
                tc::mma_bf16(tmem + NQ, tc::desc_sw128(av + ao), tc::desc_sw128(bl + bo), id, 1u);
            }
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
        // query column c is t = k0 + c; key s is in its window when s <= t < (s / BS + L) BS
        const int vlo = row, vhi = min((s / BS + L) * BS, S) - 1 - k0;
        // the hi (lo_terms false) or lo terms of P^T to sP and of dS^T to sDS
        auto pass = [&](bool lo_terms) {
#pragma unroll 1
            for (int c0 = half * HALF; c0 < half * HALF + HALF; c0 += 32) {
                float sv[32], pv[32];
                tc::tmem_ld32(tS + c0, sv);
                tc::tmem_ld32(tP + c0, pv);
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = 2 * u;
                    const bool in0 = live && c0 + i >= vlo && c0 + i <= vhi;
                    const bool in1 = live && c0 + i + 1 >= vlo && c0 + i + 1 <= vhi;
                    const float p0 = in0 ? tc::ex2_fast(fmaf(sv[i], scale_log2, -s_lse[c0 + i])) : 0.f;
                    const float p1 = in1 ? tc::ex2_fast(fmaf(sv[i + 1], scale_log2, -s_lse[c0 + i + 1])) : 0.f;
                    uint32_t ph, pl, dh, dl;
                    split2(p0, p1, ph, pl);
                    split2(p0 * (pv[i] - s_D[c0 + i]), p1 * (pv[i + 1] - s_D[c0 + i + 1]), dh, dl);
                    pk[u] = lo_terms ? pl : ph;
                    dk[u] = lo_terms ? dl : dh;
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const uint32_t off = tc::kmajor_chunk(row, (c0 >> 3) + q8, NQ);
                    *(uint4 *)(sP + off) = make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
                    *(uint4 *)(sDS + off) = make_uint4(dk[4 * q8], dk[4 * q8 + 1], dk[4 * q8 + 2], dk[4 * q8 + 3]);
                }
            }
            tc::fence_smem_to_async();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
        };
        pass(false);
        if (tid == 0) {
            const uint32_t id = tc::idesc_bf16(128, D, true);
            const uint32_t ap = tc::smem_u32(sP), ad = tc::smem_u32(sDS);
            const uint32_t bq = tc::smem_u32(sQ), bh_ = tc::smem_u32(sDOH), bl = tc::smem_u32(sDOL);
#pragma unroll
            for (int kk = 0; kk < NQ / 16; ++kk) {
                const uint64_t pa = tc::desc_kmajor(ap + 256 * kk, NQ), da = tc::desc_kmajor(ad + 256 * kk, NQ);
                tc::mma_bf16(tmem + 2 * NQ, pa, tc::desc_sw128_mn(bh_ + 2048 * kk, NQ * 128), id, kk > 0);
                tc::mma_bf16(tmem + 2 * NQ, pa, tc::desc_sw128_mn(bl + 2048 * kk, NQ * 128), id, 1u);
                tc::mma_bf16(tmem + 2 * NQ + D, da, tc::desc_sw128_mn(bq + 2048 * kk, NQ * 128), id, kk > 0);
            }
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
        pass(true);  // sP and sDS are free: the products above have completed
        if (tid == 0) {
            const uint32_t id = tc::idesc_bf16(128, D, true);
            const uint32_t ap = tc::smem_u32(sP), ad = tc::smem_u32(sDS);
            const uint32_t bq = tc::smem_u32(sQ), bh_ = tc::smem_u32(sDOH);
#pragma unroll
            for (int kk = 0; kk < NQ / 16; ++kk) {
                tc::mma_bf16(tmem + 2 * NQ, tc::desc_kmajor(ap + 256 * kk, NQ),
                             tc::desc_sw128_mn(bh_ + 2048 * kk, NQ * 128), id, 1u);
                tc::mma_bf16(tmem + 2 * NQ + D, tc::desc_kmajor(ad + 256 * kk, NQ),
                             tc::desc_sw128_mn(bq + 2048 * kk, NQ * 128), id, 1u);
            }
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
#pragma unroll 1
        for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
            float v[32], g[32];
            tc::tmem_ld32(tV + c0, v);
            tc::tmem_ld32(tK + c0, g);
            if (live) {
                float4 *dv = (float4 *)(dv_loc + ((size_t)bh * S + s) * D + c0);
                float4 *dk = (float4 *)(dk_loc + ((size_t)bh * S + s) * D + c0);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    dv[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                    dk[q4] = make_float4(g[4 * q4], g[4 * q4 + 1], g[4 * q4 + 2], g[4 * q4 + 3]);
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();  // shared memory and TMEM are free for the next tile
        tc::fence_after_sync();
    }
    // leave no TMA write in flight into this CTA's shared memory
    if (tid == 0 && pend >= 0 && !tc::mbar_wait(bar_ld, (uint32_t)(pend & 1))) ok = false;
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}


// ---------------------------------------------------------------------------
// backward, the remote blocks on the tensor cores: one persistent CTA of 256
// threads per SM walks the (b, h, block j) of the selection lists; for each
// block, K_j and V_j arrive by TMA and its selecting queries are taken 128 at a
// time, their Q, dO hi and dO lo rows gathered by cp.async into the 128-byte
// swizzled layout (eight threads per row).  Per chunk of queries g:
//   S = Q_g K_j^T,  dP = dO_g V_j^T           (TMEM columns [0, 64), [64, 128))
//   P = exp(S / sqrt(d) - lse),  dS = P (dP - D)   (every key of a selected block is visible)
//   dQ_g = dS K_j        -> one fp32 row per (query, slot) in dq_pair, summed in slot order later
//   dV_j += P^T dO_g,  dK_j += dS^T Q_g      (TMEM, over all chunks of the block)
// P and dS are stored once, row-major by query as two bf16 terms each; the
// row-major tile is the K-major A operand of dQ and the MN-major A operand
// (M = the block's 64 keys, padded to 128 rows whose results are not read) of
// dV and dK.  dV_j and dK_j (without the 1/sqrt(d) factor) are then added to the
// rows of dv_loc and dk_loc that the local kernel wrote: only this CTA writes
// block j's rows.
// ---------------------------------------------------------------------------
template <int D>
struct BwdRemoteSmem {
    // NS stages of the gathered rows and of K/V: two at d = 64 (the next chunk's rows and the next block's K/V
    // load while a chunk is computed), one at d = 128 (shared memory)
    static constexpr int NS = D == 64 ? 2 : 1;
    static constexpr int KB = 64 * D * 2, QB = 128 * D * 2, PB = 128 * 64 * 2;
    // K, V per stage; P hi, P lo, dS hi, dS lo; then Q, dO hi, dO lo per stage.  Each P/dS tile is followed by at
    // least 16 KB of other tiles, which the padding half of its MN-major operand reads
    static constexpr int K_OFF = 0, V_OFF = NS * KB, PH_OFF = 2 * NS * KB, PL_OFF = PH_OFF + PB;
    static constexpr int DH_OFF = PL_OFF + PB, DL_OFF = DH_OFF + PB, Q_OFF = DL_OFF + PB;
    static constexpr int GH_OFF = Q_OFF + NS * QB, GL_OFF = GH_OFF + NS * QB;
    static constexpr int BAR_OFF = GL_OFF + NS * QB;  // NS K/V mbarriers, the MMA mbarrier, TMEM base
    static constexpr int WIN_OFF = BAR_OFF + 64;      // int [2][256]: list sizes and starts of a window of blocks
    static constexpr int BYTES = WIN_OFF + 2 * 256 * 4;
    static constexpr int TCOLS = 128 + 3 * D;
    static constexpr bool supported = TCOLS <= 512 && BYTES <= 227 * 1024 && QB >= PB;
};

__device__ __forceinline__ uint32_t sw128(int r, int c) {  // 16-byte chunk c of row r, 128-row slabs of 64 columns
    return (uint32_t)((c >> 3) * (128 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// one chunk of the remote work: up to 128 selecting queries [g0, g0 + 128) of the CTA's k-th block (list entry
// f = blockIdx.x + k gridDim.x, n queries from list position st); k < 0: none
struct BwdChunk {
    int k, g0, n, st;
};

template <int D>
__global__ void __launch_bounds__(256, 1) k_bwd_remote_tc(const __grid_constant__ BwdMaps maps, const bf16 *__restrict__ Q,
                                                          const bf16 *__restrict__ dohi, const bf16 *__restrict__ dolo,
                                                          const float *__restrict__ lse, const float *__restrict__ dsum,
                                                          const int32_t *__restrict__ cnt,
                                                          const int32_t *__restrict__ start,
                                                          const int32_t *__restrict__ list, float *__restrict__ dq_pair,
                                                          float *__restrict__ dk_loc, float *__restrict__ dv_loc,
                                                          unsigned long long *__restrict__ counters, int S, int R,
                                                          int nb, float scale_log2, int nbh) {
    constexpr int BS = 64;
    using Lay = BwdRemoteSmem<D>;
    static_assert(Lay::supported, "tile shape");
    constexpr int NS = Lay::NS, KB = Lay::KB, QB = Lay::QB, DH = D / 2;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *sPH = smem + Lay::PH_OFF, *sPL = smem + Lay::PL_OFF, *sDH = smem + Lay::DH_OFF, *sDL = smem + Lay::DL_OFF;
    uint64_t *bar_kv = (uint64_t *)(smem + Lay::BAR_OFF), *mbar = bar_kv + NS;
    uint32_t *tmem_base = (uint32_t *)(mbar + 1);
    if (timed_out(counters)) return;
    if (tc::smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) record_error(counters, kDevErrSmemAlign);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    if (warp == 0) {
        tc::tmem_alloc(tmem_base, 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) tc::mbar_init(&bar_kv[i], 1);
        tc::mbar_init(mbar, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    // S, dP, dQ, dV and dK columns of this lane quarter
    const uint32_t tS = trow, tP = trow + 64, tQ = trow + 128, tV = trow + 128 + D, tK = trow + 128 + 2 * D;
    const uint32_t idS = tc::idesc_bf16(128, BS), idQ = tc::idesc_bf16(128, D, true),
                   idKV = tc::idesc_bf16(128, D, true, true);
    const int total = nbh * nb;

    // This CTA's chunks in order: its blocks f = blockIdx.x + k gridDim.x with a nonempty list, 128 queries at a
    // time.  The list sizes and starts of 256 of its blocks at a time sit in shared memory, so that finding the
    // next chunk waits on no global load; the next chunk's list entries are requested at the top of a chunk, its
    // rows gathered once the first products are issued, its log-sum-exp and D read there too.
    int *s_bn = (int *)(smem + Lay::WIN_OFF), *s_bs = s_bn + 256;
    const int G = gridDim.x;
    int kw = -256;  // first k of the window
    auto find_block = [&](int k) {  // the first of this CTA's blocks k' >= k with a nonempty list (uniform)
        for (;; ++k) {
            if ((long long)blockIdx.x + (long long)k * G >= total) return BwdChunk{-1, 0, 0, 0};
            if (k >= kw + 256) {
                __syncthreads();  // every thread is done with the old window
                const long long f = (long long)blockIdx.x + (long long)(k + tid) * G;
                s_bn[tid] = f < total ? cnt[f] : 0;
                s_bs[tid] = f < total ? start[f] : 0;
                __syncthreads();
                kw = k;
            }
            const int n = s_bn[k - kw];
            if (n > 0) return BwdChunk{k, 0, n, s_bs[k - kw]};
        }
    };
    auto next_of = [&](const BwdChunk &c) {
        if (c.g0 + 128 < c.n) return BwdChunk{c.k, c.g0 + 128, c.n, c.st};
        return find_block(c.k + 1);
    };
    auto f_of = [&](const BwdChunk &c) { return blockIdx.x + c.k * G; };
    constexpr int CPR = D / 8, KQ = 128 * CPR / 256;  // 16-byte segments per row; rows per thread in a gather
    // the list entries of chunk c this thread gathers (rows tid / CPR + (256 / CPR) kq) and its softmax row's
    auto req_idx = [&](const BwdChunk &c, int (&ri)[KQ], int &rt) {
        const int f = f_of(c), bh = f / nb, ng = min(128, c.n - c.g0);
        const int32_t *lst = list + (size_t)bh * S * R + c.st + c.g0;
#pragma unroll
        for (int kq = 0; kq < KQ; ++kq) {
            const int r = tid / CPR + (256 / CPR) * kq;
            ri[kq] = r < ng ? lst[r] / R : -1;
        }
        rt = row < ng ? lst[row] : -1;  // the pair t * R + r
    };
    // stage `st` of the gathered rows of chunk c (zeros past its end) from the requested entries
    auto gather = [&](const BwdChunk &c, int st, const int (&ri)[KQ]) {
        const int bh = f_of(c) / nb;
        uint8_t *sQ = smem + Lay::Q_OFF + st * QB, *sGH = smem + Lay::GH_OFF + st * QB, *sGL = smem + Lay::GL_OFF + st * QB;
        const int cc = tid % CPR;
#pragma unroll
        for (int kq = 0; kq < KQ; ++kq) {
            const int r = tid / CPR + (256 / CPR) * kq;
            const bool live = ri[kq] >= 0;
            const size_t off = live ? ((size_t)bh * S + ri[kq]) * D + 8 * cc : 0;
            tc::cp_async16(sQ + sw128(r, cc), Q + off, live);
            tc::cp_async16(sGH + sw128(r, cc), dohi + off, live);
            tc::cp_async16(sGL + sw128(r, cc), dolo + off, live);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    int pend[NS];  // thread 0: per K/V stage, the parity of a load issued and not yet seen complete, or -1
#pragma unroll
    for (int i = 0; i < NS; ++i) pend[i] = -1;
    auto load_kv = [&](const BwdChunk &c, int kb) {  // K_j, V_j of chunk c's block into K/V stage kb % NS
        if (tid != 0) return;
        const int f = f_of(c), ks = kb % NS, bh = f / nb, j = f % nb;
        uint8_t *sK = smem + Lay::K_OFF + ks * KB, *sV = smem + Lay::V_OFF + ks * KB;
        tc::mbar_expect_tx(&bar_kv[ks], 2 * KB);
#pragma unroll
        for (int a = 0; a < D / 64; ++a) {
            tc::tma_load_3d(sK + a * (BS * 128), &maps.k, 64 * a, j * BS, bh, &bar_kv[ks]);
            tc::tma_load_3d(sV + a * (BS * 128), &maps.v, 64 * a, j * BS, bh, &bar_kv[ks]);
        }
        pend[ks] = (kb / NS) & 1;
    };
    // this thread's softmax row of a chunk: pair, log-sum-exp of its query (exp2 domain), D
    auto row_stats = [&](const BwdChunk &c, int rt, int &t, float &l2, float &dd) {
        const size_t base = (size_t)(f_of(c) / nb) * S;
        t = rt >= 0 ? rt : 0;
        l2 = rt >= 0 ? lse[base + rt / R] * 1.4426950408889634f : 0.f;
        dd = rt >= 0 ? dsum[base + rt / R] : 0.f;
    };

    bool ok = true;
    uint32_t mph = 0;  // completions of mbar so far, mod 2
    BwdChunk c = find_block(0);
    int kb = 0, ck = 0;  // blocks and chunks begun
    int t_c = 0;
    float lse_c = 0.f, D_c = 0.f;
    if (c.k >= 0) {
        int ri[KQ], rt;
        req_idx(c, ri, rt);
        load_kv(c, 0);
        gather(c, 0, ri);
        row_stats(c, rt, t_c, lse_c, D_c);
    }
    while (c.k >= 0 && ok) {
        const int f = f_of(c), bh = f / nb, j = f % nb;
        const int ng = min(128, c.n - c.g0);
        const int st = ck % NS, ks = kb % NS;
        const bool live = row < ng;
        const int t = t_c;
        const float lse2 = lse_c, Drow = D_c;
        const BwdChunk nx = next_of(c);
        const bool nx_new_block = nx.k != c.k;
        int ri_nx[KQ], rt_nx = -1;
        if (nx.k >= 0) {
            req_idx(nx, ri_nx, rt_nx);  // used below (two stages) or after this chunk (one)
            if (NS == 2 && nx_new_block) load_kv(nx, kb + 1);
        }
        tc::cp_async_wait_all();  // this chunk's rows (the only copies in flight)
        bool landed = true;
        if (tid == 0 && c.g0 == 0) {
            landed = tc::mbar_wait(&bar_kv[ks], (uint32_t)((kb / NS) & 1));
            if (landed) pend[ks] = -1;
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        ok = __syncthreads_and(landed);
        tc::fence_after_sync();
        if (!ok) break;
        const uint8_t *sK = smem + Lay::K_OFF + ks * KB, *sV = smem + Lay::V_OFF + ks * KB;
        const uint8_t *sQ = smem + Lay::Q_OFF + st * QB, *sGH = smem + Lay::GH_OFF + st * QB,
                      *sGL = smem + Lay::GL_OFF + st * QB;
        if (tid == 0) {
            const uint32_t aq = tc::smem_u32(sQ), ah = tc::smem_u32(sGH), al = tc::smem_u32(sGL);
            const uint32_t bk = tc::smem_u32(sK), bv = tc::smem_u32(sV);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32, bo = (kk >> 2) * (BS * 128) + (kk & 3) * 32;
                tc::mma_bf16(tmem, tc::desc_sw128(aq + ao), tc::desc_sw128(bk + bo), idS, kk > 0);
                tc::mma_bf16(tmem + 64, tc::desc_sw128(ah + ao), tc::desc_sw128(bv + bo), idS, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32, bo = (kk >> 2) * (BS * 128) + (kk & 3) * 32;
                tc::mma_bf16(tmem + 64, tc::desc_sw128(al + ao), tc::desc_sw128(bv + bo), idS, 1u);
            }
            tc::commit(mbar);
        }
        if (NS == 2 && nx.k >= 0) {  // the next chunk's rows load while this one is computed
            gather(nx, (ck + 1) % NS, ri_nx);
            row_stats(nx, rt_nx, t_c, lse_c, D_c);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
        // P and dS of this row over the block's 64 keys (this warp's 32 of them), hi and lo terms
        {
            const int c0 = half * 32;
            float sv[32], pv[32];
            tc::tmem_ld32(tS + c0, sv);
            tc::tmem_ld32(tP + c0, pv);
            uint32_t ph[16], pl[16], dh[16], dl[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float p0 = live ? tc::ex2_fast(fmaf(sv[2 * u], scale_log2, -lse2)) : 0.f;
                const float p1 = live ? tc::ex2_fast(fmaf(sv[2 * u + 1], scale_log2, -lse2)) : 0.f;
                split2(p0, p1, ph[u], pl[u]);
                split2(p0 * (pv[2 * u] - Drow), p1 * (pv[2 * u + 1] - Drow), dh[u], dl[u]);
            }
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                const uint32_t off = sw128(row, (c0 >> 3) + q8);
                *(uint4 *)(sPH + off) = make_uint4(ph[4 * q8], ph[4 * q8 + 1], ph[4 * q8 + 2], ph[4 * q8 + 3]);
                *(uint4 *)(sPL + off) = make_uint4(pl[4 * q8], pl[4 * q8 + 1], pl[4 * q8 + 2], pl[4 * q8 + 3]);
                *(uint4 *)(sDH + off) = make_uint4(dh[4 * q8], dh[4 * q8 + 1], dh[4 * q8 + 2], dh[4 * q8 + 3]);
                *(uint4 *)(sDL + off) = make_uint4(dl[4 * q8], dl[4 * q8 + 1], dl[4 * q8 + 2], dl[4 * q8 + 3]);
            }
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) {
            const uint32_t bk = tc::smem_u32(sK), bq = tc::smem_u32(sQ), gh = tc::smem_u32(sGH),
                           gl = tc::smem_u32(sGL);
            const uint32_t a_ph = tc::smem_u32(sPH), a_pl = tc::smem_u32(sPL), a_dh = tc::smem_u32(sDH),
                           a_dl = tc::smem_u32(sDL);
            // dQ_g = dS K_j: A = dS (K-major over the 64 keys), B = K_j (MN-major)
#pragma unroll
            for (int kk = 0; kk < BS / 16; ++kk) {
                const uint64_t bd = tc::desc_sw128_mn(bk + 2048 * kk, BS * 128);
                tc::mma_bf16(tmem + 128, tc::desc_sw128(a_dh + 32 * kk), bd, idQ, kk > 0);
                tc::mma_bf16(tmem + 128, tc::desc_sw128(a_dl + 32 * kk), bd, idQ, 1u);
            }
            // dV_j += P^T dO_g and dK_j += dS^T Q_g: A = P, dS read MN-major (M = keys; the second 64-key
            // half of the 128-row operand points at another tile and its rows are not read), K = the chunk's
            // queries, B = dO, Q (MN-major)
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk) {
                const bool acc = c.g0 > 0 || kk > 0;
                const uint64_t bgh = tc::desc_sw128_mn(gh + 2048 * kk, 128 * 128);
                const uint64_t bgl = tc::desc_sw128_mn(gl + 2048 * kk, 128 * 128);
                const uint64_t bqd = tc::desc_sw128_mn(bq + 2048 * kk, 128 * 128);
                const uint64_t aph = tc::desc_sw128_mn(a_ph + 2048 * kk, Lay::PB);
                const uint64_t apl = tc::desc_sw128_mn(a_pl + 2048 * kk, Lay::PB);
                const uint64_t adh = tc::desc_sw128_mn(a_dh + 2048 * kk, Lay::PB);
                const uint64_t adl = tc::desc_sw128_mn(a_dl + 2048 * kk, Lay::PB);
                tc::mma_bf16(tmem + 128 + D, aph, bgh, idKV, acc);
                tc::mma_bf16(tmem + 128 + D, aph, bgl, idKV, 1u);
                tc::mma_bf16(tmem + 128 + D, apl, bgh, idKV, 1u);
                tc::mma_bf16(tmem + 128 + 2 * D, adh, bqd, idKV, acc);
                tc::mma_bf16(tmem + 128 + 2 * D, adl, bqd, idKV, 1u);
            }
            tc::commit(mbar);
        }
        ok = __syncthreads_and(tc::mbar_wait(mbar, mph));
        mph ^= 1u;
        tc::fence_after_sync();
        if (!ok) break;
        // this row's dQ part, to its (query, slot) row (t holds the pair)
#pragma unroll 1
        for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tQ + c0, v);
            if (live) {
                float4 *dst = (float4 *)(dq_pair + ((size_t)bh * S * R + t) * D + c0);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            }
        }
        if (nx_new_block) {
            // dV_j and dK_j: TMEM rows 0..63 (lane quarters 0 and 1; quarters 2 and 3 hold the padding rows), added
            // to the local parts of the block's keys (only this CTA writes them)
            if (quarter < 2) {
                const size_t key = (size_t)bh * S + j * BS + row;
#pragma unroll 1
                for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
                    float v[32], g[32];
                    tc::tmem_ld32(tV + c0, v);
                    tc::tmem_ld32(tK + c0, g);
                    float4 *dv = (float4 *)(dv_loc + key * D + c0);
                    float4 *dk = (float4 *)(dk_loc + key * D + c0);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 a = dv[q4], b = dk[q4];
                        dv[q4] = make_float4(a.x + v[4 * q4], a.y + v[4 * q4 + 1], a.z + v[4 * q4 + 2],
                                             a.w + v[4 * q4 + 3]);
                        dk[q4] = make_float4(b.x + g[4 * q4], b.y + g[4 * q4 + 1], b.z + g[4 * q4 + 2],
                                             b.w + g[4 * q4 + 3]);
                    }
                }
            }
            ++kb;
        }
        tc::fence_before_sync();
        __syncthreads();  // this chunk's shared memory and TMEM columns are free
        tc::fence_after_sync();
        if (NS == 1 && nx.k >= 0) {  // one stage: the next chunk loads only now
            if (nx_new_block) load_kv(nx, kb);
            gather(nx, 0, ri_nx);
            row_stats(nx, rt_nx, t_c, lse_c, D_c);
        }
        c = nx;
        ++ck;
    }
    // leave no copy in flight into this CTA's shared memory
    tc::cp_async_wait_all();
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < NS; ++i)
            if (pend[i] >= 0 && !tc::mbar_wait(&bar_kv[i], (uint32_t)pend[i])) ok = false;
    }
    if (!ok && tid == 0) record_error(counters, kDevErrTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

template <int D, int BS, int NK>
static cudaError_t launch_bwd_local_dq_shape(const Plan &p, const void *Q, const void *K, const void *V,
                                             const void *dohi, const void *dolo, const float *lse, const float *dsum,
                                             float *dq_loc, unsigned long long *counters, cudaStream_t s) {
    const mono_config &c = p.cfg;
    using Lay = BwdLocalSmem<D, NK>;
    BwdMaps maps;
    const int BH = c.B * c.H;
    if (!make_map_3d(&maps.q, Q, D, c.S, BH, 128) || !make_map_3d(&maps.k, K, D, c.S, BH, NK) ||
        !make_map_3d(&maps.v, V, D, c.S, BH, NK) || !make_map_3d(&maps.dohi, dohi, D, c.S, BH, 128) ||
        !make_map_3d(&maps.dolo, dolo, D, c.S, BH, 128))
        return cudaErrorInvalidValue;
    auto kern = k_bwd_local_dq_tc<D, BS, NK>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES)) != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int tiles = BH * ((c.S + 127) / 128);
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.d));
    kern<<<std::min(tiles, sms), 256, Lay::BYTES, s>>>(maps, lse, dsum, dq_loc, counters, c.S, c.L, scale_log2, BH);
    count_launches(1);
    return cudaGetLastError();
}

template <int D, int BS, int NQ>
static cudaError_t launch_bwd_local_dkdv_shape(const Plan &p, const void *Q, const void *K, const void *V,
                                               const void *dohi, const void *dolo, const float *lse,
                                               const float *dsum, float *dk_loc, float *dv_loc,
                                               unsigned long long *counters, cudaStream_t s) {
    const mono_config &c = p.cfg;
    using Lay = BwdKvSmem<D, NQ>;
    BwdMaps maps;
    const int BH = c.B * c.H;
    if (!make_map_3d(&maps.k, K, D, c.S, BH, 128) || !make_map_3d(&maps.v, V, D, c.S, BH, 128) ||
        !make_map_3d(&maps.q, Q, D, c.S, BH, NQ) || !make_map_3d(&maps.dohi, dohi, D, c.S, BH, NQ) ||
        !make_map_3d(&maps.dolo, dolo, D, c.S, BH, NQ))
        return cudaErrorInvalidValue;
    auto kern = k_bwd_local_dkdv_tc<D, BS, NQ>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES)) != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int tiles = BH * ((c.S + 127) / 128);
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.d));
    kern<<<std::min(tiles, sms), 256, Lay::BYTES, s>>>(maps, lse, dsum, dk_loc, dv_loc, counters, c.S, c.L,
                                                       scale_log2, BH);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_bwd_local_dkdv_tc(const Plan &p, const void *Q, const void *K, const void *V, const void *dohi,
                                     const void *dolo, const float *lse, const float *dsum, float *dk_loc,
                                     float *dv_loc, unsigned long long *counters, cudaStream_t s) {
    const mono_config &c = p.cfg;
    if (!bwd_local_dq_tc_supported(c)) return cudaErrorInvalidValue;
    const int nq = 128 + (c.L - 1) * c.Bs;
    if (c.d == 64 && nq <= 128)
        return launch_bwd_local_dkdv_shape<64, 64, 128>(p, Q, K, V, dohi, dolo, lse, dsum, dk_loc, dv_loc, counters, s);
    if (c.d == 64)
        return launch_bwd_local_dkdv_shape<64, 64, 192>(p, Q, K, V, dohi, dolo, lse, dsum, dk_loc, dv_loc, counters, s);
    return launch_bwd_local_dkdv_shape<128, 64, 128>(p, Q, K, V, dohi, dolo, lse, dsum, dk_loc, dv_loc, counters, s);
}

template <int D>
static cudaError_t launch_bwd_remote_shape(const Plan &p, const void *Q, const void *K, const void *V,
                                           const void *dohi, const void *dolo, const float *lse, const float *dsum,
                                           const int32_t *cnt, const int32_t *start, const int32_t *list,
                                           float *dq_pair, float *dk_loc, float *dv_loc, unsigned long long *counters,
                                           cudaStream_t s) {
    const mono_config &c = p.cfg;
    using Lay = BwdRemoteSmem<D>;
    BwdMaps maps;
    const int BH = c.B * c.H;
    if (!make_map_3d(&maps.k, K, D, c.S, BH, 64) || !make_map_3d(&maps.v, V, D, c.S, BH, 64))
        return cudaErrorInvalidValue;
    maps.q = maps.k;  // unused
    maps.dohi = maps.k;
    maps.dolo = maps.k;
    auto kern = k_bwd_remote_tc<D>;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES)) != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.d));
    const int total = BH * p.nb;
    kern<<<std::min(total, sms), 256, Lay::BYTES, s>>>(maps, (const bf16 *)Q, (const bf16 *)dohi, (const bf16 *)dolo,
                                                       lse, dsum, cnt, start, list, dq_pair, dk_loc, dv_loc, counters,
                                                       c.S, c.R, p.nb, scale_log2, BH);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_bwd_remote_tc(const Plan &p, const void *Q, const void *K, const void *V, const void *dohi,
                                 const void *dolo, const float *lse, const float *dsum, const int32_t *cnt,
                                 const int32_t *start, const int32_t *list, float *dq_pair, float *dk_loc,
                                 float *dv_loc, unsigned long long *counters, cudaStream_t s) {
    const mono_config &c = p.cfg;
    if (!bwd_local_dq_tc_supported(c)) return cudaErrorInvalidValue;
    if (c.d == 64)
        return launch_bwd_remote_shape<64>(p, Q, K, V, dohi, dolo, lse, dsum, cnt, start, list, dq_pair, dk_loc,
                                           dv_loc, counters, s);
    return launch_bwd_remote_shape<128>(p, Q, K, V, dohi, dolo, lse, dsum, cnt, start, list, dq_pair, dk_loc, dv_loc,
                                        counters, s);
}

bool bwd_local_dq_tc_supported(const mono_config &c) {
    if (c.dtype != MONO_BF16 || c.Bs != 64 || c.L < 1) return false;
    const int nk = 128 + (c.L - 1) * c.Bs;
    return (c.d == 64 && nk <= 192) || (c.d == 128 && nk <= 128);
}

cudaError_t launch_bwd_local_dq_tc(const Plan &p, const void *Q, const void *K, const void *V, const void *dohi,
                                  const void *dolo, const float *lse, const float *dsum, float *dq_loc,
                                  unsigned long long *counters, cudaStream_t s) {
    const mono_config &c = p.cfg;
    if (!bwd_local_dq_tc_supported(c)) return cudaErrorInvalidValue;
    const int nk = 128 + (c.L - 1) * c.Bs;
    if (c.d == 64 && nk <= 128)
        return launch_bwd_local_dq_shape<64, 64, 128>(p, Q, K, V, dohi, dolo, lse, dsum, dq_loc, counters, s);
    if (c.d == 64)
        return launch_bwd_local_dq_shape<64, 64, 192>(p, Q, K, V, dohi, dolo, lse, dsum, dq_loc, counters, s);
    return launch_bwd_local_dq_shape<128, 64, 128>(p, Q, K, V, dohi, dolo, lse, dsum, dq_loc, counters, s);
}

cudaError_t launch_attend_tc(const Plan &p, const void *Q, const void *K, const void *V, const int32_t *sel, void *O,
                             void *ws, cudaStream_t s, int parts, float *o32, float *lse, bool *stats) {
    if (stats) *stats = false;
    const mono_config &c = p.cfg;
    const bf16 *q = (const bf16 *)Q, *k = (const bf16 *)K, *v = (const bf16 *)V;
    bf16 *o = (bf16 *)O;
    const int nk = 128 + (c.L - 1) * c.Bs;
    // NK = the local key range rounded up to a multiple of 32 (MMA N <= 256)
#define MONO_TC(DD, BB, NN)                                                                                     \
    do {                                                                                                        \
        if (c.R <= 2) return launch_tc_shape<DD, BB, NN, 2>(p, q, k, v, sel, o, ws, s, parts, o32, lse, stats);                  \
        if (c.R <= 4) return launch_tc_shape<DD, BB, NN, 4>(p, q, k, v, sel, o, ws, s, parts, o32, lse, stats);                  \
        return launch_tc_shape<DD, BB, NN, kMaxR>(p, q, k, v, sel, o, ws, s, parts, o32, lse, stats);                            \
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

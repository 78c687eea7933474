// route.cu -- learned product-hash routing: block summary + codebook assign,
// bounded causal posting lists, and the per-query probe / union / causal
// filter / E cap / rerank.
//
// Source: aitechinspire.com Monodratic article, "Snapshot: key facts from the
// report" (after RoPE, source blocks are assigned to bounded causal posting
// lists; each query probes product addresses, reranks the returned
// candidates and selects a fixed number of remote blocks); "Monodratic 将稀疏
// 注意力转化为检索决策" (remio.ai): a product address combines the decisions of
// several code components, lists have a strict capacity, and no source block
// may become visible to an earlier query.
//
// Every floating-point value that decides an integer is computed in fp32 in a
// fixed order: sums in ascending index order, dot products as a chain of fused
// multiply-adds from +0 in ascending element order, grid scores summed in
// ascending subspace order.  Ties go to the lowest code, address or block id.
// The explicit __fadd_rn / __fmaf_rn / __fdiv_rn intrinsics keep the compiler
// from contracting or reordering that arithmetic.
#include "internal.cuh"
#include "tc.cuh"

namespace mono {

// Programmatic dependent launch between the posting lists and the probe: the
// lists kernel lets the probe's CTAs start at once (they load their queries
// and score the codebooks meanwhile), and the probe waits for the lists to be
// complete and visible only before it reads them.  Without a programmatic
// launch the wait returns at once.

// ---------------------------------------------------------------------------
// (A2, A3) block summary kbar = mean of the Bs post-RoPE keys, and the product
// address: per subspace m the code with the largest <kbar_m, cw[h,m,c]>.
// grid (nb, H, B), 128 threads.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) k_summary_assign(const T *__restrict__ K, const float *__restrict__ cb,
                                                        float *__restrict__ kbar, int32_t *__restrict__ addr, int S,
                                                        int d, int Bs, int M, int C, int H) {
    __shared__ float kb[kMaxD];
    __shared__ float sc[kMaxM * kMaxC];
    const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nb = S / Bs;
    const size_t bh = (size_t)b * H + h;
    const T *Kb = K + (bh * S + (size_t)j * Bs) * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        float acc = 0.0f;
        for (int t = 0; t < Bs; ++t) acc = __fadd_rn(acc, to_f(Kb[(size_t)t * d + i]));
        float v = __fdiv_rn(acc, (float)Bs);
        kb[i] = v;
        kbar[(bh * nb + j) * d + i] = v;
    }
    __syncthreads();
    const int dm = d / M;
    for (int mc = threadIdx.x; mc < M * C; mc += blockDim.x) {
        const int m = mc / C;
        const float *w = cb + ((size_t)h * M * C + mc) * dm;
        const float *kv = kb + m * dm;
        float acc = 0.0f;
        for (int i = 0; i < dm; ++i) acc = __fmaf_rn(kv[i], w[i], acc);
        sc[mc] = acc;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        long long a = 0;
        for (int m = 0; m < M; ++m) {
            float best = sc[m * C];
            int bc = 0;
            for (int c = 1; c < C; ++c)
                if (sc[m * C + c] > best) { best = sc[m * C + c]; bc = c; }
            a = a * C + bc;
        }
        addr[bh * nb + j] = (int32_t)a;
    }
}

// ---------------------------------------------------------------------------
// (A2, A3) the same summaries with one warp per block: each lane owns D/32
// adjacent columns and walks the block's rows in ascending t, reading its
// columns of a row as one 32- or 64-bit word straight from global memory (a
// row per warp load; 16 registers of rows per batch, the next batch in
// flight while one is summed).  A CTA takes 4 x bpw
// consecutive blocks of one (b, h), each warp bpw of them; the grid is sized
// to about one wave of 6 CTAs per SM.  The head's codebook sits in shared
// memory, transposed so that lane mc reads codeword mc without bank conflicts.
// grid (ceil(nb / (4 bpw)), H, B), 128 threads.
// ---------------------------------------------------------------------------
inline size_t summary_smem(int M, int C, int Bs, int D, int es) {
    (void)Bs;
    (void)es;
    return ((size_t)M * C * (D / M) + 4 * (size_t)D + 4 * (size_t)M * C) * 4;
}

template <typename T, int PER>
struct RowWord;  // this lane's PER columns of one row
template <>
struct RowWord<__nv_bfloat16, 2> {
    using W = uint32_t;
    static __device__ __forceinline__ void cvt(W w, float (&v)[2]) {
        const float2 f = __bfloat1622float2(*(const __nv_bfloat162 *)&w);
        v[0] = f.x; v[1] = f.y;
    }
};
template <>
struct RowWord<__nv_bfloat16, 4> {
    using W = uint2;
    static __device__ __forceinline__ void cvt(W w, float (&v)[4]) {
        const float2 f0 = __bfloat1622float2(*(const __nv_bfloat162 *)&w.x);
        const float2 f1 = __bfloat1622float2(*(const __nv_bfloat162 *)&w.y);
        v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
    }
};
template <>
struct RowWord<float, 2> {
    using W = float2;
    static __device__ __forceinline__ void cvt(W w, float (&v)[2]) { v[0] = w.x; v[1] = w.y; }
};
template <>
struct RowWord<float, 4> {
    using W = float4;
    static __device__ __forceinline__ void cvt(W w, float (&v)[4]) { v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w; }
};

template <typename T, int D>
__global__ void __launch_bounds__(128, 6) k_summary_assign_w(const T *__restrict__ K, const float *__restrict__ cb,
                                                          float *__restrict__ kbar, int32_t *__restrict__ addr, int S,
                                                          int Bs, int M, int C, int H, int bpw) {
    constexpr int PER = D / 32;  // columns per lane
    static_assert(PER == 2 || PER == 4, "D = 64 or 128");
    tc::grid_dep_launch();  // the lists kernel may start; it waits for the addresses itself
    using RW = RowWord<T, PER>;
    using W = typename RW::W;
    constexpr int U = 16 / ((int)sizeof(W) / 4);  // rows per batch: 16 registers of words
    extern __shared__ __align__(16) float sm[];
    const int MC = M * C, dm = D / M;
    float *s_cbT = sm;                              // [dm][M*C]: element i of codeword mc at i * MC + mc
    float *s_kb = s_cbT + MC * dm;                  // [4][D]
    float *s_sc = s_kb + 4 * D;                     // [4][M*C]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int nb = S / Bs;
    const size_t bh = (size_t)b * H + h;
    const int j0 = (blockIdx.x * 4 + warp) * bpw;
    const int nq = max(0, min(bpw, nb - j0));  // this warp's blocks
    const int nbt = Bs / U;                     // whole batches per block; Bs % U rows follow them
    const int total = nq * nbt;
    auto row_ptr = [&](int q) { return (const W *)(K + (bh * S + (size_t)(j0 + q) * Bs) * D) + lane; };
    auto load = [&](int k, W (&buf)[U]) {
        const W *rq = row_ptr(k / nbt) + (size_t)(k % nbt) * U * 32;
#pragma unroll
        for (int u = 0; u < U; ++u) buf[u] = __ldg(rq + (size_t)u * 32);
    };
    W b0[U], b1[U];
    if (total > 0) load(0, b0);  // the first rows are in flight while the codebook is staged
    // the head's codebook (C*D floats, [M][C][dm]), transposed, with independent 16-byte loads
    {
        const float4 *src = (const float4 *)(cb + (size_t)h * C * D);
        for (int i4 = threadIdx.x; i4 < C * D / 4; i4 += blockDim.x) {
            const float4 f = __ldg(src + i4);
            const int mc = (4 * i4) / dm, i = (4 * i4) % dm;  // dm is a multiple of 4
            s_cbT[(i + 0) * MC + mc] = f.x;
            s_cbT[(i + 1) * MC + mc] = f.y;
            s_cbT[(i + 2) * MC + mc] = f.z;
            s_cbT[(i + 3) * MC + mc] = f.w;
        }
    }
    __syncthreads();
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
    // block q after its whole batches: the tail rows, kbar, scores and address; acc is reset for the next block
    auto finish = [&](int q) {
        const int j = j0 + q;
        const W *rq = row_ptr(q);
        for (int t = nbt * U; t < Bs; ++t) {
            float v[PER];
            RW::cvt(__ldg(rq + (size_t)t * 32), v);
#pragma unroll
            for (int e = 0; e < PER; ++e) acc[e] = __fadd_rn(acc[e], v[e]);
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const float v = __fdiv_rn(acc[e], (float)Bs);
            s_kb[warp * D + lane * PER + e] = v;
            kbar[(bh * nb + j) * D + lane * PER + e] = v;
        }
        __syncwarp();
        for (int mc = lane; mc < MC; mc += 32) {
            const int m = mc / C;
            const float *kv = s_kb + warp * D + m * dm;
            float a = 0.0f;
            for (int i = 0; i < dm; ++i) a = __fmaf_rn(kv[i], s_cbT[i * MC + mc], a);
            s_sc[warp * MC + mc] = a;
        }
        __syncwarp();
        // one lane per subspace: the first maximum wins (ascending c); lane 0 combines
        int bc = 0;
        if (lane < M) {
            const float *sc = s_sc + warp * MC + lane * C;
            float best = sc[0];
            for (int c = 1; c < C; ++c)
                if (sc[c] > best) { best = sc[c]; bc = c; }
        }
        long long ad = 0;
        for (int m = 0; m < M; ++m) ad = ad * C + __shfl_sync(0xffffffffu, bc, m);
        if (lane == 0) addr[bh * nb + j] = (int32_t)ad;
        __syncwarp();
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
    };
    auto consume = [&](int k, const W (&buf)[U]) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float v[PER];
            RW::cvt(buf[u], v);
#pragma unroll
            for (int e = 0; e < PER; ++e) acc[e] = __fadd_rn(acc[e], v[e]);
        }
        if (k % nbt == nbt - 1) finish(k / nbt);
    };
    if (nbt == 0)  // blocks shorter than one batch
        for (int q = 0; q < nq; ++q) finish(q);
    // batches in two register buffers: batch k+1 is in flight while batch k is summed
    for (int k = 0; k < total; k += 2) {
        if (k + 1 < total) load(k + 1, b1);
        consume(k, b0);
        if (k + 1 < total) {
            if (k + 2 < total) load(k + 2, b0);
            consume(k + 1, b1);
        }
    }
}

// ---------------------------------------------------------------------------
// (A4) posting lists by counting, for address spaces that fit in shared
// memory (C^M <= kDenseA).  One warp walks the blocks in ascending id, 32 at a
// time: __match_any_sync groups equal addresses, so each block's rank among
// the earlier blocks of its address is the running count plus its position
// in the group.  A scan of the counts over the addresses then gives each
// block its slot in the (address, id) order.  Deterministic, no atomics.
// grid (H, B), 1024 threads.
// ---------------------------------------------------------------------------
constexpr int kDenseA = 4096;

__global__ void __launch_bounds__(1024) k_posting_dense(const int32_t *__restrict__ addr, int32_t *__restrict__ ids,
                                                        int32_t *__restrict__ saddr, int32_t *__restrict__ rank,
                                                        int32_t *__restrict__ overflow, int nb, int cap, int H, int A,
                                                        unsigned long long *__restrict__ stats) {
    tc::grid_dep_launch();
    tc::grid_dep_wait();  // the addresses (summaries kernel) are complete
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < kCntStats) stats[threadIdx.x] = 0ull;  // the probe's
    __shared__ int s_cnt[kDenseA];
    __shared__ int s_part[32];
    __shared__ int s_ov[32];
    extern __shared__ int32_t s_dyn[];
    int32_t *s_addr = s_dyn;          // [nb]
    int32_t *s_rank = s_dyn + nb;     // [nb]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bh = (size_t)blockIdx.y * H + blockIdx.x;
    for (int a = tid; a < A; a += blockDim.x) s_cnt[a] = 0;
    for (int j = tid; j < nb; j += blockDim.x) s_addr[j] = addr[bh * nb + j];
    __syncthreads();
    if (warp == 0) {
        for (int j0 = 0; j0 < nb; j0 += 32) {
            const int j = j0 + lane;
            const bool in = j < nb;
            const int a = in ? s_addr[j] : -1 - lane;       // distinct dummies never match a real address
            const unsigned peers = __match_any_sync(0xffffffffu, a);
            const int base = in ? s_cnt[a] : 0;
            const int pos = __popc(peers & ((1u << lane) - 1));
            __syncwarp();
            if (in) {
                s_rank[j] = base + pos;
                if (pos == 0) s_cnt[a] = base + __popc(peers);
            }
            __syncwarp();
        }
    }
    __syncthreads();
    // exclusive scan of s_cnt over the A addresses (each thread a contiguous run)
    const int per = (A + blockDim.x - 1) / blockDim.x;
    const int a0 = tid * per;
    int run = 0;
    for (int a = a0; a < min(A, a0 + per); ++a) run += s_cnt[a];
    int x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_part[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (int)(blockDim.x >> 5) ? s_part[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_part[lane] = w;
    }
    __syncthreads();
    int off = (warp ? s_part[warp - 1] : 0) + x - run;
    for (int a = a0; a < min(A, a0 + per); ++a) {
        const int c = s_cnt[a];
        s_cnt[a] = off;   // now the start of address a
        off += c;
    }
    __syncthreads();
    int dropped = 0;
    for (int j = tid; j < nb; j += blockDim.x) {
        const int a = s_addr[j], r = s_rank[j];
        const int pos = s_cnt[a] + r;
        ids[bh * nb + pos] = j;
        saddr[bh * nb + pos] = a;
        rank[bh * nb + pos] = r;
        dropped += r >= cap;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dropped += __shfl_xor_sync(0xffffffffu, dropped, o);
    if (lane == 0) s_ov[warp] = dropped;
    __syncthreads();
    if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_ov[w];
        overflow[bh] = tot;
    }
}

// ---------------------------------------------------------------------------
// (A4) posting lists in canonical form: ids sorted by (address, id), the
// address of each entry and its rank among the blocks of that address.  The
// lists keep the earliest `cap` blocks of each address (rank < cap); the
// others are dropped and counted.  Each block's slot is found by counting the
// blocks that sort before it, so the result is deterministic.
// grid (H, B), 1024 threads, dynamic smem nb ints.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_posting_build(const int32_t *__restrict__ addr, int32_t *__restrict__ ids,
                                                        int32_t *__restrict__ saddr, int32_t *__restrict__ rank,
                                                        int32_t *__restrict__ overflow, int nb, int cap, int H,
                                                        unsigned long long *__restrict__ stats) {
    tc::grid_dep_launch();
    tc::grid_dep_wait();  // the addresses (summaries kernel) are complete
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < kCntStats) stats[threadIdx.x] = 0ull;  // the probe's
    extern __shared__ int32_t s_addr[];
    __shared__ int s_ov[32];
    const size_t bh = (size_t)blockIdx.y * H + blockIdx.x;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s_addr[j] = addr[bh * nb + j];
    __syncthreads();
    int dropped = 0;
    for (int j = threadIdx.x; j < nb; j += blockDim.x) {
        const int a = s_addr[j];
        int less = 0, before = 0;
        for (int k = 0; k < nb; ++k) {
            const int ak = s_addr[k];
            less += ak < a;
            before += (ak == a) & (k < j);
        }
        const int pos = less + before;
        ids[bh * nb + pos] = j;
        saddr[bh * nb + pos] = a;
        rank[bh * nb + pos] = before;
        dropped += before >= cap;
    }
    for (int o = 16; o > 0; o >>= 1) dropped += __shfl_xor_sync(0xffffffffu, dropped, o);
    if ((threadIdx.x & 31) == 0) s_ov[threadIdx.x >> 5] = dropped;
    __syncthreads();
    if (threadIdx.x == 0) {
        int tot = 0;
        for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) tot += s_ov[w];
        overflow[bh] = tot;
    }
}

// ---------------------------------------------------------------------------
// (A4, redirect-on-overflow) the lists of one (b, h) when a block whose own
// list is full goes to the first list with room among the next addresses in
// mixed-radix order (a+1, a+2, ... mod C^M), and is dropped (and counted) only
// when every list is full.  The placement depends on the order of the blocks,
// so one warp places them in ascending order: a count per address and a
// bitmap of the full lists in shared memory; the search for a list with room
// scans the bitmap 32 words (1024 addresses) per step.  Then every thread
// takes part in the canonical export by comparison counting over the list
// addresses, the dropped blocks last under the address C^M.
// grid (H, B), 1024 threads; dynamic smem: bitmap [ceil(A/32)] u32, list
// addresses [nb] int32, counts [A] u16 (A <= kRedirectMaxA).
// ---------------------------------------------------------------------------
inline size_t redirect_smem(long long A, int nb) {
    return (size_t)((A + 31) / 32) * 4 + (size_t)nb * 4 + (size_t)A * 2;
}

// first address in [p0, p1) whose list is not full, or -1 (all lanes of warp 0)
__device__ __forceinline__ int first_free(const uint32_t *s_full, int p0, int p1, int lane) {
    if (p0 >= p1) return -1;
    const int wl = p0 >> 5, wh = (p1 - 1) >> 5;
    for (int w0 = wl; w0 <= wh; w0 += 32) {
        const int w = w0 + lane;
        uint32_t freeb = 0;
        if (w <= wh) {
            freeb = ~s_full[w];
            if (w == wl) freeb &= ~0u << (p0 & 31);
            if (w == wh && (p1 & 31) != 0) freeb &= (1u << (p1 & 31)) - 1u;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, freeb != 0);
        if (bal) {
            const int src = __ffs(bal) - 1;
            const uint32_t fb = __shfl_sync(0xffffffffu, freeb, src);
            return ((w0 + src) << 5) + __ffs(fb) - 1;
        }
    }
    return -1;
}

__global__ void __launch_bounds__(1024) k_posting_redirect(const int32_t *__restrict__ addr, int32_t *__restrict__ ids,
                                                           int32_t *__restrict__ saddr, int32_t *__restrict__ rank,
                                                           int32_t *__restrict__ overflow, int nb, int cap, int H,
                                                           int A, unsigned long long *__restrict__ stats) {
    tc::grid_dep_launch();
    tc::grid_dep_wait();  // the addresses (summaries kernel) are complete
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < kCntStats) stats[threadIdx.x] = 0ull;  // the probe's
    extern __shared__ uint32_t s_red[];
    const int nw = (A + 31) / 32;
    uint32_t *s_full = s_red;                          // [nw]: bit set = list full (and every bit past A)
    int32_t *s_key = (int32_t *)(s_full + nw);         // [nb]: own address, then list address (A = dropped)
    uint16_t *s_cnt = (uint16_t *)(s_key + nb);        // [A]
    __shared__ int s_ov;
    const int tid = threadIdx.x, lane = tid & 31;
    const size_t bh = (size_t)blockIdx.y * H + blockIdx.x;
    const int ecap = min(cap, nb + 1);                 // a list can never hold more than nb blocks
    for (int i = tid; i < nw; i += blockDim.x)
        s_full[i] = (i == nw - 1 && (A & 31)) ? ~((1u << (A & 31)) - 1u) : 0u;
    for (int i = tid; i < A; i += blockDim.x) s_cnt[i] = 0;
    for (int j = tid; j < nb; j += blockDim.x) s_key[j] = addr[bh * nb + j];
    __syncthreads();
    if (tid < 32) {
        int ov = 0;
        for (int j = 0; j < nb; ++j) {
            const int a = s_key[j];
            int dst = -1;
            if ((unsigned)a < (unsigned)A) {
                if (s_cnt[a] < ecap) dst = a;
                else {
                    dst = first_free(s_full, a + 1, A, lane);
                    if (dst < 0) dst = first_free(s_full, 0, a, lane);
                }
            }
            __syncwarp();
            if (lane == 0) {
                if (dst >= 0) {
                    const int n = s_cnt[dst] + 1;
                    s_cnt[dst] = (uint16_t)n;
                    if (n >= ecap) s_full[dst >> 5] |= 1u << (dst & 31);
                    s_key[j] = dst;
                } else {
                    s_key[j] = A;
                }
            }
            ov += dst < 0;
            __syncwarp();
        }
        if (lane == 0) s_ov = ov;
    }
    __syncthreads();
    for (int j = tid; j < nb; j += blockDim.x) {
        const int a = s_key[j];
        int less = 0, before = 0;
        for (int k = 0; k < nb; ++k) {
            const int ak = s_key[k];
            less += ak < a;
            before += (ak == a) & (k < j);
        }
        const int pos = less + before;
        ids[bh * nb + pos] = j;
        saddr[bh * nb + pos] = a;
        rank[bh * nb + pos] = before;
    }
    if (tid == 0) overflow[bh] = s_ov;
}

// ---------------------------------------------------------------------------
// (A5-A7) per-query probe, union, causal filter, E cap and rerank.
//
// Probe: the top-T addresses of the product grid under (g desc, address asc),
// g = s_0[c_0] + s_1[c_1] + ... in fp32.  The grid is not enumerated: the
// prefixes of the address (codes of subspaces 0..m, most significant first)
// are pruned one stage at a time.  The pruning is exact:
//  * fp32 addition is monotone, so g is non-decreasing in every prefix score.
//  * delta = (M+1) ulp(2G), with G >= every |partial sum|, exceeds what the at
//    most M-1 later roundings can absorb.  So a prefix u "dominates" a prefix
//    p when v_u > v_p + delta (then g(u,s) > g(p,s) for every suffix s), or
//    when v_u >= v_p and u < p (then g(u,s) >= g(p,s) and the address of (u,s)
//    is lower).  Either way (u,s) ranks before (p,s).
//  * A prefix with T dominators has no completion in the top T, and is
//    dropped.  The stage keeps U, its own top T under (value desc, index asc),
//    which never have T dominators.  It also keeps every prefix within delta
//    of U's last value that is not dominated by all of U.
//  * The final stage ranks the completions of the survivors exactly.
// Exact ties (e.g. a zero query) collapse to the T lowest prefixes.  If a
// stage would still keep more than kPrefMax prefixes, the query falls back
// to scoring the whole grid.
// ---------------------------------------------------------------------------
constexpr int kPrefMax = 64;

struct TopT {
    float v[kMaxT];
    int a[kMaxT];
    int n, T;
    __device__ void init(int T_) {
        T = T_;
        n = 0;
    }
    // order: (value desc, index asc)
    __device__ static bool before(float v1, int a1, float v2, int a2) { return v1 > v2 || (v1 == v2 && a1 < a2); }
    __device__ void push(float val, int ad) {
        if (n == T && !before(val, ad, v[T - 1], a[T - 1])) return;
        int pos = n < T ? n : T - 1;
        while (pos > 0 && before(val, ad, v[pos - 1], a[pos - 1])) {
            v[pos] = v[pos - 1];
            a[pos] = a[pos - 1];
            --pos;
        }
        v[pos] = val;
        a[pos] = ad;
        if (n < T) ++n;
    }
    // the entry is one of this top set
    __device__ bool holds(float val, int ad) const {
        return n < T || !before(v[T - 1], a[T - 1], val, ad);
    }
    // every kept entry dominates (val, ad) in the sense above
    __device__ bool all_dominate(float val, int ad, float delta) const {
        if (n < T) return false;
        const float hi = val + delta;
        for (int k = 0; k < n; ++k)
            if (!(v[k] > hi || (v[k] >= val && a[k] < ad))) return false;
        return true;
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(128) k_probe_rerank(const T *__restrict__ Q, const float *__restrict__ kbar,
                                                      const float *__restrict__ cb, const int32_t *__restrict__ post_ids,
                                                      const int32_t *__restrict__ post_addr,
                                                      const int32_t *__restrict__ forced, int32_t *__restrict__ sel,
                                                      unsigned long long *__restrict__ counters,
                                                      int32_t *__restrict__ walk_log, int S, int H, int Bs,
                                                      int L, int R, int E, int M, int C, int Tp, int cap) {
    tc::grid_dep_wait();  // the posting lists are complete
    tc::grid_dep_launch();
    extern __shared__ float smem[];
    const int nb = S / Bs;
    float *s_cb = smem;                                     // [M*C*dm] = C*D floats
    int32_t *s_addr = (int32_t *)(s_cb + C * D);            // [nb]
    int32_t *s_ids = s_addr + nb;                           // [nb]
    const int h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * H + h;
    for (int i = threadIdx.x; i < C * D; i += blockDim.x) s_cb[i] = cb[(size_t)h * C * D + i];
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        s_addr[i] = post_addr[bh * nb + i];
        s_ids[i] = post_ids[bh * nb + i];
    }
    __syncthreads();

    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    int n_sel = 0, lt_r = 0, ign = 0;
    if (t < S) {
        float q[D];
        const T *qp = Q + (bh * S + t) * D;
#pragma unroll
        for (int i = 0; i < D; ++i) q[i] = to_f(qp[i]);
        const int dm = D / M;

        // subspace scores s[m][c]
        float s[kMaxM * kMaxC];
        float G = 0.f;
        for (int m = 0; m < M; ++m) {
            float mx = 0.f;
            for (int c = 0; c < C; ++c) {
                const float *w = s_cb + (m * C + c) * dm;
                float acc = 0.0f;
                for (int i = 0; i < dm; ++i) acc = __fmaf_rn(q[m * dm + i], w[i], acc);
                s[m * C + c] = acc;
                mx = fmaxf(mx, fabsf(acc));
            }
            G += mx;
        }
        int e2;
        frexpf(2.f * G + 1e-30f, &e2);                       // 2G < 2^e2
        const float delta = (float)(M + 1) * ldexpf(1.f, e2 - 24);

        // staged exact top-T over the product grid
        float pv[kPrefMax];
        int pi[kPrefMax];
        int np = 0;
        bool fallback = false;
        TopT top;
        for (int m = 0; m < M && !fallback; ++m) {
            // entries of this stage: (prefix value, prefix index)
            const int ne = m == 0 ? C : np * C;
            top.init(Tp);
            for (int e = 0; e < ne; ++e) {
                const int p = e / C, c = e % C;
                const float v = m == 0 ? s[c] : __fadd_rn(pv[p], s[m * C + c]);
                top.push(v, m == 0 ? c : pi[p] * C + c);
            }
            if (m == M - 1) break;  // final stage: `top` is the exact answer
            const float thr = top.n < Tp ? -INFINITY : top.v[Tp - 1] - delta;
            float nv[kPrefMax];
            int ni[kPrefMax];
            int nn = 0;
            for (int e = 0; e < ne && !fallback; ++e) {
                const int p = e / C, c = e % C;
                const float v = m == 0 ? s[c] : __fadd_rn(pv[p], s[m * C + c]);
                const int idx = m == 0 ? c : pi[p] * C + c;
                if (!(v >= thr)) continue;
                if (!top.holds(v, idx) && top.all_dominate(v, idx, delta)) continue;
                if (nn == kPrefMax) { fallback = true; break; }
                nv[nn] = v;
                ni[nn] = idx;
                ++nn;
            }
            for (int p = 0; p < nn; ++p) {
                pv[p] = nv[p];
                pi[p] = ni[p];
            }
            np = nn;
        }
        if (fallback) {
            log_walk(counters, walk_log, (long long)bh * S + t);
            top.init(Tp);
            long long A = 1;
            for (int m = 0; m < M; ++m) A *= C;
            for (long long a = 0; a < A; ++a) {
                long long rem = a;
                int code[kMaxM];
                for (int m = M - 1; m >= 0; --m) {
                    code[m] = (int)(rem % C);
                    rem /= C;
                }
                float g = s[code[0]];
                for (int m = 1; m < M; ++m) g = __fadd_rn(g, s[m * C + code[m]]);
                top.push(g, (int)a);
            }
        }

        // union of the probed lists in probe-rank order, causal filter, E cap
        const int bq = t / Bs;
        const int lim = bq - L;
        int cand[kMaxE];
        int nc = 0;
        for (int r = 0; r < top.n && nc < E; ++r) {
            const int a = top.a[r];
            int lo = 0, hi = nb;  // lower bound of a in s_addr
            while (lo < hi) {
                int mid = (lo + hi) >> 1;
                if (s_addr[mid] < a) lo = mid + 1;
                else hi = mid;
            }
            for (int k = lo; k < nb && s_addr[k] == a && k - lo < cap && nc < E; ++k) {
                const int j = s_ids[k];
                if (j > lim) break;  // ids ascend within an address
                cand[nc++] = j;
            }
        }

        // rerank by <q, kbar_j>, keep the top R (score desc, id asc)
        float rv[kMaxR];
        int ra[kMaxR];
        int nr = 0;
        for (int k = 0; k < nc && R > 0; ++k) {
            const int j = cand[k];
            const float4 *kr = (const float4 *)(kbar + (bh * nb + j) * D);
            // eight runs of D/8 elements as fma chains, added as a balanced tree
            float run[8];
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                float acc = 0.0f;
#pragma unroll
                for (int i4 = l * (D / 32); i4 < (l + 1) * (D / 32); ++i4) {
                    const float4 v = __ldg(kr + i4);
                    acc = __fmaf_rn(q[4 * i4 + 0], v.x, acc);
                    acc = __fmaf_rn(q[4 * i4 + 1], v.y, acc);
                    acc = __fmaf_rn(q[4 * i4 + 2], v.z, acc);
                    acc = __fmaf_rn(q[4 * i4 + 3], v.w, acc);
                }
                run[l] = acc;
            }
            const float acc = __fadd_rn(__fadd_rn(__fadd_rn(run[0], run[1]), __fadd_rn(run[2], run[3])),
                                        __fadd_rn(__fadd_rn(run[4], run[5]), __fadd_rn(run[6], run[7])));
            if (nr == R && !(acc > rv[R - 1] || (acc == rv[R - 1] && j < ra[R - 1]))) continue;
            int pos = nr < R ? nr : R - 1;
            while (pos > 0 && (acc > rv[pos - 1] || (acc == rv[pos - 1] && j < ra[pos - 1]))) {
                rv[pos] = rv[pos - 1];
                ra[pos] = ra[pos - 1];
                --pos;
            }
            rv[pos] = acc;
            ra[pos] = j;
            if (nr < R) ++nr;
        }
        // forced block: appended, or replaces the lowest-ranked selection
        if (forced && R > 0) {
            const int f = forced[bh * S + t];
            if (f >= 0) {
                if (f <= lim) {
                    bool present = false;
                    for (int k = 0; k < nr; ++k) present |= ra[k] == f;
                    if (!present) {
                        if (nr < R) ra[nr++] = f;
                        else ra[R - 1] = f;
                    }
                } else {
                    ign = 1;
                }
            }
        }
        // ascending ids, -1 padding
        for (int x = 1; x < nr; ++x)
            for (int y = x; y > 0 && ra[y - 1] > ra[y]; --y) {
                int tmp = ra[y];
                ra[y] = ra[y - 1];
                ra[y - 1] = tmp;
            }
        int32_t *out = sel + (bh * S + t) * R;
        for (int k = 0; k < R; ++k) out[k] = k < nr ? ra[k] : -1;
        n_sel = nr;
        lt_r = nr < R;
    }
    // statistics
    for (int o = 16; o > 0; o >>= 1) {
        n_sel += __shfl_xor_sync(0xffffffffu, n_sel, o);
        lt_r += __shfl_xor_sync(0xffffffffu, lt_r, o);
        ign += __shfl_xor_sync(0xffffffffu, ign, o);
    }
    if ((threadIdx.x & 31) == 0) {
        if (lt_r) atomicAdd(&counters[kCntQueriesLtR], (unsigned long long)lt_r);
        if (n_sel) atomicAdd(&counters[kCntRemoteSel], (unsigned long long)n_sel);
        if (ign) atomicAdd(&counters[kCntForcedIgnored], (unsigned long long)ign);
    }
}

// ---------------------------------------------------------------------------
// (A5-A7) the same computation for M = 2 with every size fixed at compile
// time, so all per-query state stays in registers.  The subspace-0 scores
// also go to shared memory (one column per thread) so that the final stage can
// walk the surviving codes by index.  Same pruning rule and arithmetic order
// as k_probe_rerank.
// ---------------------------------------------------------------------------
template <int T_>
struct RegTop {  // top-T_ by (value desc, index asc); fully unrolled
    float v[T_];
    int a[T_];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int k = 0; k < T_; ++k) { v[k] = -INFINITY; a[k] = 0x7fffffff; }
    }
    __device__ __forceinline__ static bool before(float v1, int a1, float v2, int a2) {
        return v1 > v2 || (v1 == v2 && a1 < a2);
    }
    __device__ __forceinline__ void push(float val, int ad) {
        if (!before(val, ad, v[T_ - 1], a[T_ - 1])) return;
        v[T_ - 1] = val;
        a[T_ - 1] = ad;
#pragma unroll
        for (int k = T_ - 1; k > 0; --k) {
            if (before(v[k], a[k], v[k - 1], a[k - 1])) {
                float tv = v[k]; v[k] = v[k - 1]; v[k - 1] = tv;
                int ta = a[k]; a[k] = a[k - 1]; a[k - 1] = ta;
            }
        }
    }
};

// Bit mask of the codes of one subspace that are not dominated by T0 others:
// U = the top T0 by (score desc, code asc), found by T0 passes of an
// ascending argmax (the first maximum wins a tie), plus every code within
// delta of U's last score that some member of U does not dominate.
template <int C, int T0>
__device__ __forceinline__ unsigned survivors(const float (&s)[C], float delta) {
    if constexpr (T0 >= C) {
        return C == 32 ? 0xffffffffu : ((1u << C) - 1);
    } else {
        float uv[T0];
        int ui[T0];
        unsigned taken = 0;
#pragma unroll
        for (int k = 0; k < T0; ++k) {
            float best = -INFINITY;
            int bi = 0;
            bool any = false;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const bool free = !((taken >> c) & 1u);
                const bool better = free && (!any || s[c] > best);
                best = better ? s[c] : best;
                bi = better ? c : bi;
                any = any || free;
            }
            uv[k] = best;
            ui[k] = bi;
            taken |= 1u << bi;
        }
        const float thr = uv[T0 - 1] - delta;
        unsigned keep = taken;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (((taken >> c) & 1u) || !(s[c] >= thr)) continue;
            const float hi = s[c] + delta;
            bool dom = true;
#pragma unroll
            for (int k = 0; k < T0; ++k) dom = dom && (uv[k] > hi || (uv[k] >= s[c] && ui[k] < c));
            if (!dom) keep |= 1u << c;
        }
        return keep;
    }
}

// The top T0 codes of one subspace by (score desc, code asc), in that order:
// T0 passes of a tree argmax over the codes not yet taken, in which the right
// operand wins only when strictly greater, so that the lowest code wins a tie.
// Taken codes are masked with -inf; the scores are finite for finite inputs.
template <int C, int T0>
__device__ __forceinline__ void top_codes(const float (&s)[C], float (&uv)[T0], int (&ui)[T0]) {
    static_assert((C & (C - 1)) == 0 && C >= 2 && C <= 32, "C a power of two");
    unsigned taken = 0;  // codes already ranked read as -inf (no copy of the scores: fewer registers)
#pragma unroll
    for (int k = 0; k < T0; ++k) {
        float tv[C / 2];
        int ti[C / 2];
#pragma unroll
        for (int p = 0; p < C / 2; ++p) {
            const float a = (taken >> (2 * p)) & 1u ? -INFINITY : s[2 * p];
            const float b = (taken >> (2 * p + 1)) & 1u ? -INFINITY : s[2 * p + 1];
            const bool r = b > a;
            tv[p] = r ? b : a;
            ti[p] = r ? 2 * p + 1 : 2 * p;
        }
#pragma unroll
        for (int n = C / 4; n >= 1; n >>= 1) {
#pragma unroll
            for (int p = 0; p < n; ++p) {
                const bool r = tv[2 * p + 1] > tv[2 * p];
                tv[p] = r ? tv[2 * p + 1] : tv[2 * p];
                ti[p] = r ? ti[2 * p + 1] : ti[2 * p];
            }
        }
        uv[k] = tv[0];
        ui[k] = ti[0];
        taken |= 1u << ti[0];
    }
}

// Codes outside U = {ui} within delta of U's last score: candidates for the
// near-tie rule below (a bit mask; almost always empty).
template <int C, int T0>
__device__ __forceinline__ unsigned near_codes(const float (&s)[C], const float (&uv)[T0], unsigned taken, float delta) {
    const float thr = uv[T0 - 1] - delta;
    unsigned m = 0;
#pragma unroll
    for (int c = 0; c < C; ++c) m |= (s[c] >= thr ? 1u : 0u) << c;
    return m & ~taken;
}

// Of the near codes, those that some member of U does not dominate (the
// pruning rule: u dominates p if s_u > s_p + delta, or s_u >= s_p and u < p).
template <int C, int T0>
__device__ __forceinline__ unsigned undominated(unsigned near, const float (&s)[C], const float (&uv)[T0],
                                                const int (&ui)[T0], float delta) {
    unsigned keep = 0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        if (!((near >> c) & 1u)) continue;
        const float sc = s[c], hi = sc + delta;
        bool dom = true;
#pragma unroll
        for (int k = 0; k < T0; ++k) dom = dom && (uv[k] > hi || (uv[k] >= sc && ui[k] < c));
        if (!dom) keep |= 1u << c;
    }
    return keep;
}

// eight consecutive elements of a query row in shared memory, as fp32
template <typename T>
__device__ __forceinline__ void q8(const T *qm, float (&qv)[8]) {
    if constexpr (sizeof(T) == 2) {
        const uint4 u = *(const uint4 *)qm;
        const __nv_bfloat162 *h2 = (const __nv_bfloat162 *)&u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            qv[2 * e] = f.x;
            qv[2 * e + 1] = f.y;
        }
    } else {
        const float4 a = ((const float4 *)qm)[0], b = ((const float4 *)qm)[1];
        qv[0] = a.x; qv[1] = a.y; qv[2] = a.z; qv[3] = a.w;
        qv[4] = b.x; qv[5] = b.y; qv[6] = b.z; qv[7] = b.w;
    }
}

using tc::f2_t;
using tc::f2_dup;
using tc::f2_split;
using tc::f2_fma;

// Scores of one subspace for NQ queries: s[q][c] = q_m . codeword_{m,c}, one
// fma chain per (query, code) in ascending element order from +0.  The
// subspace's codebook is stored transposed in shared memory (element i of
// codes 0..C-1 contiguous), so one 16-byte read gives element i of four codes
// as two pairs, and one paired fma advances the chains of codes c and c+1 of
// a query together; the NQ queries share the codebook reads.  q is read from
// the query tile in shared memory eight elements at a time.  The chains run
// interleaved, which changes nothing in any one of them.
template <typename T, int DM, int C, int NQ>
__device__ __forceinline__ void sub_scores_x2(const T *const (&qm)[NQ], const float *cbT, float (&s)[NQ][C]) {
    static_assert(C % 4 == 0, "codes in groups of four");
    f2_t acc[NQ][C / 2];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int p = 0; p < C / 2; ++p) acc[q][p] = 0ull;  // (+0, +0)
#pragma unroll
    for (int i8 = 0; i8 < DM / 8; ++i8) {
        float qv[NQ][8];
#pragma unroll
        for (int q = 0; q < NQ; ++q) q8<T>(qm[q] + 8 * i8, qv[q]);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const ulonglong2 *row = (const ulonglong2 *)(cbT + (8 * i8 + e) * C);
            f2_t w[C / 2];
#pragma unroll
            for (int c4 = 0; c4 < C / 4; ++c4) {
                const ulonglong2 v = row[c4];
                w[2 * c4] = v.x;
                w[2 * c4 + 1] = v.y;
            }
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const f2_t qq = f2_dup(qv[q][e]);
#pragma unroll
                for (int p = 0; p < C / 2; ++p) acc[q][p] = f2_fma(qq, w[p], acc[q][p]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int p = 0; p < C / 2; ++p) f2_split(acc[q][p], s[q][2 * p], s[q][2 * p + 1]);
}

// Row pitch (bytes) of the query tile in shared memory: the row plus 16 bytes,
// so that the 16-byte reads of one warp (one row per lane) hit every bank once
// per eight lanes.
template <typename T, int D>
constexpr int probe_q_pitch() {
    return D * (int)sizeof(T) + 16;
}
// queries per thread (one: a thread's scores and probe state fit in 80 registers, so six CTAs of 128 threads
// share an SM and their warps hide each other's latency; two queries per thread at 128 registers, which share
// every codebook read, measured 12 % slower), threads per CTA and the CTAs per SM the register budget is sized for
template <int C>
constexpr int probe_nq() {
    return 1;
}
template <int C>
constexpr int probe_threads() {
    return 128;
}
template <int C>
constexpr int probe_min_ctas() {
    return C <= 16 ? 6 : 3;
}
// shared memory of the probe's candidates: ids (int16), counts, rerank scores
template <int E>
constexpr size_t cand_smem(int nq) {
    return ((size_t)nq * E * 2 + 15) / 16 * 16 + (size_t)nq * 4 + (size_t)nq * E * 4;
}
static_assert(kMaxNb <= 32768, "block ids fit int16");

template <typename T, int D, int C, int E>
constexpr size_t probe_m2_smem(int nb) {
    return (size_t)C * D * 4 + (size_t)C * C * 8 + (size_t)probe_threads<C>() * probe_nq<C>() * probe_q_pitch<T, D>() +
           cand_smem<E>(probe_threads<C>() * probe_nq<C>()) + (size_t)nb * 8;
}

// Top R of the candidates' rerank scores acc (score desc, id asc), the forced
// block, sel in ascending order with -1 padding.  Returns the number of remote
// blocks selected and adds 1 to *ign when a forced id was not eligible.
template <int E, int R>
__device__ __forceinline__ int select_top_r(const float (&acc)[E], const int (&cid)[E], int nc,
                                            const int32_t *forced, int32_t *out, int t, size_t bh, int S, int Bs,
                                            int L, int *ign) {
    const int lim = t / Bs - L;
    RegTop<R> rk;
    rk.init();
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e < nc) rk.push(acc[e], cid[e]);
    int ra[R];
    int nr = nc < R ? nc : R;
#pragma unroll
    for (int k = 0; k < R; ++k) ra[k] = rk.a[k];
    if (forced) {
        const int f = forced[bh * S + t];
        if (f >= 0) {
            if (f <= lim) {
                bool present = false;
#pragma unroll
                for (int k = 0; k < R; ++k) present |= (k < nr) && ra[k] == f;
                if (!present) {
                    const int slot = nr < R ? nr : R - 1;
#pragma unroll
                    for (int k = 0; k < R; ++k)
                        if (k == slot) ra[k] = f;
                    if (nr < R) ++nr;
                }
            } else {
                *ign += 1;
            }
        }
    }
    // ascending ids, -1 padding
#pragma unroll
    for (int k = 0; k < R; ++k)
        if (k >= nr) ra[k] = 0x7fffffff;
#pragma unroll
    for (int x = 0; x < R; ++x)
#pragma unroll
        for (int y = 0; y + 1 < R - x; ++y)
            if (ra[y] > ra[y + 1]) { int tmp = ra[y]; ra[y] = ra[y + 1]; ra[y + 1] = tmp; }
#pragma unroll
    for (int k = 0; k < R; ++k) out[k] = k < nr ? ra[k] : -1;
    return nr;
}

// The rerank scores of the query-heads a warp probed (its threads' rows
// qi = tid + NT q, q < NQ, of the CTA's tile; each one's candidates in
// s_cid[qi][E], their number in s_nc[qi]) into s_score[qi][E], eight lanes
// per query-head: lane l of a group holds run l (elements [l D/8, (l+1) D/8))
// of q and reads the same run of each candidate's kbar row, so a group reads
// whole rows.  Its fma chain is the run's value, and three butterfly additions
// form the tree ((c0 + c1) + (c2 + c3)) + ((c4 + c5) + (c6 + c7)) in every
// lane of the group (fp32 addition is commutative, so both partners get the
// same bits).  Four query-heads per round, two rounds' loads in flight.
template <typename T, int D, int E, int NQ, int NT>
__device__ __forceinline__ void rerank_scores(const uint8_t *s_q, int qpitch, const int16_t *s_cid,
                                              const int32_t *s_nc, const float *kb, float *s_score) {
    constexpr int RUN = D / 8, RPI = 2;
    static_assert(RUN % 8 == 0 && (8 * NQ) % RPI == 0, "runs of whole 8-element chunks");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, grp = lane >> 3, run = lane & 7;
#pragma unroll 1
    for (int r0 = 0; r0 < 8 * NQ; r0 += RPI) {
        int qi[RPI], nc[RPI];
        float qv[RPI][RUN], acc[RPI][E];
#pragma unroll
        for (int h = 0; h < RPI; ++h) {
            const int wq = 4 * (r0 + h) + grp;
            qi[h] = 32 * warp + (wq & 31) + NT * (wq >> 5);
            nc[h] = s_nc[qi[h]];
#pragma unroll
            for (int i8 = 0; i8 < RUN / 8; ++i8) {
                float v8[8];
                q8<T>((const T *)(s_q + qi[h] * qpitch) + run * RUN + 8 * i8, v8);
#pragma unroll
                for (int i = 0; i < 8; ++i) qv[h][8 * i8 + i] = v8[i];
            }
        }
#pragma unroll
        for (int h = 0; h < RPI; ++h)
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float a = 0.0f;
                if (e < nc[h]) {
                    const float *row = kb + (size_t)s_cid[qi[h] * E + e] * D + run * RUN;
#pragma unroll
                    for (int i8 = 0; i8 < RUN / 8; ++i8) {
                        float kv[8];
                        tc::ldg_v8(row + 8 * i8, kv);
#pragma unroll
                        for (int i = 0; i < 8; ++i) a = __fmaf_rn(qv[h][8 * i8 + i], kv[i], a);
                    }
                }
                acc[h][e] = a;
            }
#pragma unroll
        for (int h = 0; h < RPI; ++h)
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float a = acc[h][e];
                a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 1));
                a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 2));
                a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 4));
                acc[h][e] = a;
            }
        if (run == 0) {
#pragma unroll
            for (int h = 0; h < RPI; ++h)
#pragma unroll
                for (int e = 0; e < E; ++e) s_score[qi[h] * E + e] = acc[h][e];
        }
    }
}

// The rerank q . kbar_j of the (at most E) candidates cid[0 .. nc) of
// query-head t by one thread, in the order of rerank_scores: the eight runs
// of D/8 elements each as an fma chain from +0 (the candidates' chains
// advancing together), the run values added as ((c0 + c1) + (c2 + c3)) +
// ((c4 + c5) + (c6 + c7)); then select_top_r.
template <typename T, int D, int E, int R>
__device__ __forceinline__ int rerank_thread(const T *qp, const float *kb, const int (&cid)[E], int nc,
                                             const int32_t *forced, int32_t *out, int t, size_t bh, int S, int Bs,
                                             int L, int *ign) {
    static_assert(D % 64 == 0, "runs of whole 8-element chunks");
    constexpr int CPR = D / 64;  // 8-element chunks per run
    float acc[E], half0[E], pair1[E];
    // runs 2p and 2p + 1 per step: their loads in flight together
#pragma unroll 1
    for (int p = 0; p < 4; ++p) {
        float c[2][E];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int e = 0; e < E; ++e) c[h][e] = 0.0f;
#pragma unroll
            for (int k = 0; k < CPR; ++k) {
                const int i8 = (2 * p + h) * CPR + k;
                float qv[8];
                q8<T>(qp + 8 * i8, qv);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    if (e < nc) {
                        float kv[8];  // one 32-byte load (the rows are 32-byte aligned)
                        tc::ldg_v8(kb + (size_t)cid[e] * D + 8 * i8, kv);
                        float a = c[h][e];
#pragma unroll
                        for (int i = 0; i < 8; ++i) a = __fmaf_rn(qv[i], kv[i], a);
                        c[h][e] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float pr = __fadd_rn(c[0][e], c[1][e]);  // c_2p + c_2p+1
            if (p == 0 || p == 2) pair1[e] = pr;
            else if (p == 1) half0[e] = __fadd_rn(pair1[e], pr);
            else acc[e] = __fadd_rn(half0[e], __fadd_rn(pair1[e], pr));  // p == 3: the score
        }
    }
    return select_top_r<E, R>(acc, cid, nc, forced, out, t, bh, S, Bs, L, ign);
}

// The top-R selection of this thread's query-heads (rows tid + NT q) from
// their candidates and rerank scores in shared memory; adds to the counts.
template <int E, int R, int NQ, int NT>
__device__ __forceinline__ void select_rows(const int16_t *s_cid, const int32_t *s_nc, const float *s_score,
                                            const int32_t *forced, int32_t *sel, int t_lo, size_t bh, int S, int Bs,
                                            int L, int &n_sel, int &lt_r, int &ign) {
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int qi = threadIdx.x + NT * q, t = t_lo + qi;
        if (t >= S) continue;
        int cid[E];
        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            cid[e] = s_cid[qi * E + e];
            acc[e] = s_score[qi * E + e];
        }
        const int nr = select_top_r<E, R>(acc, cid, s_nc[qi], forced, sel + (bh * S + t) * R, t, bh, S, Bs, L, &ign);
        n_sel += nr;
        lt_r += nr < R;
    }
}

// The probe, union, causal filter and E cap of one query-head t from its
// subspace scores (see k_probe_m2): the candidates in cid[0 .. nc), nc returned.
template <int C, int TP, int E>
__device__ __forceinline__ int probe_m2(const float (&s0)[C], const float (&s1)[C], const int2 *s_rng,
                                        const int32_t *s_ids, int (&cid)[E], int t, size_t bh, int S, int Bs, int L,
                                        int cap, unsigned long long *counters, int32_t *walk_log) {
    constexpr int A = C * C;
    float mx0 = 0.f, mx1 = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        mx0 = fmaxf(mx0, fabsf(s0[c]));
        mx1 = fmaxf(mx1, fabsf(s1[c]));
    }
    const bool finite = mx0 + mx1 <= 1.0e38f;
    int e2;
    frexpf(2.f * (mx0 + mx1) + 1e-30f, &e2);
    const float delta = 3.0f * ldexpf(1.f, e2 - 24);   // (M+1) ulp(2G)

    // Each subspace keeps U, its top T0 codes, and the near codes that some
    // member of U does not dominate (the pruning rule above): for subspace 0
    // as address prefixes, for subspace 1 as suffixes of any surviving prefix
    // (for a fixed prefix the completions rank by s1 with ties to the lower
    // code, which is the same rule).  The final top T lies in cand0 x cand1.
    constexpr int T0 = TP < C ? TP : C;
    constexpr unsigned kAll = C == 32 ? 0xffffffffu : ((1u << C) - 1);
    float uv0[T0], uv1[T0];
    int ui0[T0], ui1[T0];
    top_codes<C, T0>(s0, uv0, ui0);
    top_codes<C, T0>(s1, uv1, ui1);
    unsigned tk0 = 0, tk1 = 0;
#pragma unroll
    for (int k = 0; k < T0; ++k) { tk0 |= 1u << ui0[k]; tk1 |= 1u << ui1[k]; }
    const unsigned nr0 = near_codes<C, T0>(s0, uv0, tk0, delta), nr1 = near_codes<C, T0>(s1, uv1, tk1, delta);
    unsigned cand0 = tk0, cand1 = tk1;
    if (!finite) {
        cand0 = kAll;
        cand1 = kAll;
    } else if (nr0 | nr1) {
        cand0 |= undominated<C, T0>(nr0, s0, uv0, ui0, delta);
        cand1 |= undominated<C, T0>(nr1, s1, uv1, ui1, delta);
    }
    RegTop<TP> top;
    top.init();
    bool done = false;
    if (cand0 == tk0 && cand1 == tk1) {
        // U0 and U1 are sorted by score and fl(a + b) is monotone in a and
        // b, so pair (i, j) of the ranks is preceded by the (i+1)(j+1)-1
        // pairs (i' <= i, j' <= j) with scores at least as high: only pairs
        // with (i+1)(j+1) <= T can be in the top T, unless an excluded pair
        // reaches the T-th score (ties), which sends the query to the
        // general walk below.
        float vout = -INFINITY;
#pragma unroll
        for (int i = 0; i < T0; ++i)
#pragma unroll
            for (int j = 0; j < T0; ++j) {
                const float v = __fadd_rn(uv0[i], uv1[j]);
                if ((i + 1) * (j + 1) <= TP) top.push(v, ui0[i] * C + ui1[j]);
                else vout = fmaxf(vout, v);
            }
        done = vout < top.v[TP - 1];
    }
    if (!done) {
        // general walk over cand0 x cand1 (rare: near ties), on copies of the
        // scores that can be indexed by code
        log_walk(counters, walk_log, (long long)bh * S + t);
        float l0[C], l1[C];
#pragma unroll
        for (int c = 0; c < C; ++c) { l0[c] = s0[c]; l1[c] = s1[c]; }
        top.init();
        for (unsigned m0 = cand0; m0; m0 &= m0 - 1) {
            const int c0 = __ffs(m0) - 1;
            const float v0 = l0[c0];
            for (unsigned m1 = cand1; m1; m1 &= m1 - 1) {
                const int c1 = __ffs(m1) - 1;
                top.push(__fadd_rn(v0, l1[c1]), c0 * C + c1);
            }
        }
    }

    // union of the probed lists in probe order, causal filter, E cap
    const int bq = t / Bs;
    const int lim = bq - L;
#pragma unroll
    for (int e = 0; e < E; ++e) cid[e] = 0;
    int nc = 0;
    int2 rg[TP];  // every probed list's range, looked up at once
#pragma unroll
    for (int r = 0; r < TP; ++r) {
        const int a = top.a[r];
        rg[r] = (unsigned)a < (unsigned)A ? s_rng[a] : make_int2(0, 0);
    }
#pragma unroll
    for (int r = 0; r < TP; ++r) {
        const int kend = min(rg[r].y, rg[r].x + cap);
        for (int k = rg[r].x; k < kend && nc < E; ++k) {
            const int j = s_ids[k];
            if (j > lim) break;
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (e == nc) cid[e] = j;
            ++nc;
        }
    }
    return nc;
}

// M = 2 with every size fixed at compile time, so all per-query state stays
// in registers.  A CTA takes NT x NQ consecutive queries of one (b, h); its
// thread tid the queries tid, tid + NT, ...  Everything the CTA reads more
// than once goes to shared memory in one batch: the query rows, the head's
// codebooks (transposed for the paired chains) and the (b, h) posting arrays.
// Same pruning rule and arithmetic order as k_probe_rerank.
template <typename T, int D, int C, int TP, int E, int R>
__global__ void __launch_bounds__(probe_threads<C>(), probe_min_ctas<C>()) k_probe_m2(const T *__restrict__ Q, const float *__restrict__ kbar,
                                                     const float *__restrict__ cb, const int32_t *__restrict__ post_ids,
                                                     const int32_t *__restrict__ post_addr,
                                                     const int32_t *__restrict__ forced, int32_t *__restrict__ sel,
                                                     unsigned long long *__restrict__ counters,
                                                     int32_t *__restrict__ walk_log, int S, int H, int Bs,
                                                     int L, int cap) {
    constexpr int DM = D / 2, A = C * C, QP = probe_q_pitch<T, D>(), NQ = probe_nq<C>(), NT = probe_threads<C>();
    constexpr int QT = NT * NQ;
    static_assert(C <= 32 && TP <= C * C && R >= 1 && E >= 1 && QP % 16 == 0 && DM % 8 == 0, "shape");
    extern __shared__ __align__(16) float smem[];
    tc::grid_dep_launch();  // the attention's first kernel may start; it waits for sel itself
    const int nb = S / Bs;
    float *s_cbT = smem;                                 // [2][DM][C]: element i of codeword (m, c) at (m DM + i) C + c
    int2 *s_rng = (int2 *)(s_cbT + C * D);               // [A] positions [first, end) of each address's entries
    uint8_t *s_q = (uint8_t *)(s_rng + A);               // [QT] query rows, pitch QP
    int16_t *s_cid = (int16_t *)(s_q + QT * QP);         // [QT][E] candidates of each query-head
    int32_t *s_nc = (int32_t *)(s_q + QT * QP + (QT * E * 2 + 15) / 16 * 16);  // [QT] their number
    float *s_score = (float *)(s_nc + QT);               // [QT][E] their rerank scores
    int32_t *s_addr = (int32_t *)(s_score + QT * E);     // [nb]
    int32_t *s_ids = s_addr + nb;                        // [nb]
    // CTAs in dispatch order take the query tiles latest first, every (b, h) of a tile in turn: later queries have
    // more causal candidates to rerank, so the launch ends on its lightest tiles
    const int nbh = gridDim.y * gridDim.z;
    const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const int h = (lin % nbh) % gridDim.y, b = (lin % nbh) / gridDim.y;
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x;
    const int t_lo = (gridDim.x - 1 - lin / nbh) * QT;
    {
        constexpr int CH = D * (int)sizeof(T) / 16;  // 16-byte chunks per query row
        const uint8_t *src = (const uint8_t *)(Q + (bh * S + t_lo) * D);
        for (int i = tid; i < QT * CH; i += blockDim.x) {
            const int r = i / CH, c = i % CH;
            const bool ok = t_lo + r < S;
            tc::cp_async16(s_q + r * QP + 16 * c, ok ? (const void *)(src + (size_t)r * (D * sizeof(T)) + 16 * c) : Q, ok);
        }
    }
    // the head's codebooks ([2][C][DM] floats), transposed, with independent 16-byte loads
    {
        const float4 *src = (const float4 *)(cb + (size_t)h * C * D);
        for (int i4 = tid; i4 < C * D / 4; i4 += blockDim.x) {
            const float4 f = __ldg(src + i4);
            const int mc = (4 * i4) / DM, i = (4 * i4) % DM;  // DM is a multiple of 4
            float *dst = s_cbT + ((mc / C) * DM + i) * C + mc % C;
            dst[0] = f.x;
            dst[C] = f.y;
            dst[2 * C] = f.z;
            dst[3 * C] = f.w;
        }
    }
    for (int i = tid; i < A; i += blockDim.x) s_rng[i] = make_int2(0, 0);
    tc::cp_async_wait_all();
    __syncthreads();

    // subspace scores of this thread's queries (rows past S are zeros and are not routed)
    float s0[NQ][C], s1[NQ][C];
    {
        const T *qm0[NQ], *qm1[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            qm0[q] = (const T *)(s_q + (tid + NT * q) * QP);
            qm1[q] = qm0[q] + DM;
        }
        sub_scores_x2<T, DM, C, NQ>(qm0, s_cbT, s0);
        sub_scores_x2<T, DM, C, NQ>(qm1, s_cbT + DM * C, s1);
    }

    // the posting lists: complete once the lists kernel is (programmatic launch)
    tc::grid_dep_wait();
    if ((nb & 3) == 0) {  // 16-byte aligned rows of the posting arrays
        for (int i = tid; i < nb / 4; i += blockDim.x) {
            tc::cp_async16(s_addr + 4 * i, post_addr + bh * nb + 4 * i, true);
            tc::cp_async16(s_ids + 4 * i, post_ids + bh * nb + 4 * i, true);
        }
    } else {
        for (int i = tid; i < nb; i += blockDim.x) {
            s_addr[i] = post_addr[bh * nb + i];
            s_ids[i] = post_ids[bh * nb + i];
        }
    }
    tc::cp_async_wait_all();
    __syncthreads();
    // the posting arrays are sorted by address: each address's entries start
    // where the address differs from the previous entry's and end where it
    // differs from the next one's
    for (int i = tid; i < nb; i += blockDim.x) {
        const int a = s_addr[i];
        if ((unsigned)a >= (unsigned)A) continue;
        if (i == 0 || s_addr[i - 1] != a) s_rng[a].x = i;
        if (i == nb - 1 || s_addr[i + 1] != a) s_rng[a].y = i + 1;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int qi = tid + NT * q, t = t_lo + qi;
        int cid[E] = {};
        const int nc = t < S ? probe_m2<C, TP, E>(s0[q], s1[q], s_rng, s_ids, cid, t, bh, S, Bs, L, cap, counters,
                                                  walk_log)
                             : 0;
#pragma unroll
        for (int e = 0; e < E; ++e) s_cid[qi * E + e] = (int16_t)cid[e];
        s_nc[qi] = nc;
    }
    __syncwarp();
    rerank_scores<T, D, E, NQ, NT>(s_q, QP, s_cid, s_nc, kbar + bh * nb * D, s_score);
    __syncwarp();
    int n_sel = 0, lt_r = 0, ign = 0;
    select_rows<E, R, NQ, NT>(s_cid, s_nc, s_score, forced, sel, t_lo, bh, S, Bs, L, n_sel, lt_r, ign);
    for (int o = 16; o > 0; o >>= 1) {
        n_sel += __shfl_xor_sync(0xffffffffu, n_sel, o);
        lt_r += __shfl_xor_sync(0xffffffffu, lt_r, o);
        ign += __shfl_xor_sync(0xffffffffu, ign, o);
    }
    if ((threadIdx.x & 31) == 0) {
        if (lt_r) atomicAdd(&counters[kCntQueriesLtR], (unsigned long long)lt_r);
        if (n_sel) atomicAdd(&counters[kCntRemoteSel], (unsigned long long)n_sel);
        if (ign) atomicAdd(&counters[kCntForcedIgnored], (unsigned long long)ign);
    }
}

// ---------------------------------------------------------------------------
// (A5-A7) the probe for M >= 2 subspaces as a best-first walk of the product
// grid, every size fixed at compile time.  Same result, arithmetic order and
// rerank as k_probe_rerank.
//
// Each subspace's codes are ranked by (score desc, code asc) lazily: the next
// rank is an argmax over the codes not yet ranked, taken only when the walk
// first reaches it.  A tuple of ranks r = (r_0, .., r_{M-1}) scores
// g(r) = fl(..fl(v_0[r_0] + v_1[r_1]) .. + v_{M-1}[r_{M-1}]), which does not
// increase when any r_m grows (fp32 addition is monotone in each operand).
// The tuples form a tree in which the parent of r lowers its last nonzero
// rank by one.  The frontier, kept sorted in registers, gives up its first
// tuple under the probe order (g desc, address asc) T times; the first T pops
// are the probes provided that no tuple precedes its parent in that order.
// Only the first T frontier entries are kept: one that ranks below T others
// can never be popped.  A child with a lower g follows
// its parent; one with an equal g follows it when the raised rank's code is
// higher, which a tie of the two scores guarantees (ranks order tied codes
// ascending).  An equal g from unequal scores (the smaller one absorbed by
// rounding) needs the two scores within delta = (M+1) ulp(2G) of each other.
// So the walk falls back to scoring the whole grid when
//  * a child it pushes precedes its parent, or
//  * after T pops the frontier's best g equals the T-th probe's (the tie
//    runs past the probes, through tuples not yet visited) and some two
//    neighbouring ranks of a subspace differ by more than 0 and at most delta;
//  * or a score is not finite.
// Exact ties (a zero query, duplicated codewords) thus stay on the walk.
// ---------------------------------------------------------------------------
template <int C>
constexpr int rank_bits() {
    return C <= 2 ? 1 : C <= 4 ? 2 : C <= 8 ? 3 : C <= 16 ? 4 : 5;
}
template <typename T, int D, int M, int C>
constexpr size_t probe_bf_smem(int nb) {
    return (size_t)C * D * 4 + (size_t)128 * probe_q_pitch<T, D>() + (size_t)nb * 8 + 4 * (M * C + kMaxT) * 4;
}

template <typename T, int D, int M, int C, int TP, int E, int R>
__global__ void __launch_bounds__(128) k_probe_bf(const T *__restrict__ Q, const float *__restrict__ kbar,
                                                  const float *__restrict__ cb, const int32_t *__restrict__ post_ids,
                                                  const int32_t *__restrict__ post_addr,
                                                  const int32_t *__restrict__ forced, int32_t *__restrict__ sel,
                                                  unsigned long long *__restrict__ counters,
                                                  int32_t *__restrict__ walk_log, int S, int H, int Bs, int L,
                                                  int cap) {
    constexpr int DM = D / M, QP = probe_q_pitch<T, D>(), RB = rank_bits<C>();
    constexpr unsigned RMASK = (1u << RB) - 1u;
    static_assert(M >= 2 && M * RB <= 16 && C <= 16 && C % 4 == 0 && DM % 8 == 0 && TP >= 1 && R >= 1, "shape");
    static_assert(M * rank_bits<C>() <= 16 && (C == 16 ? M <= 4 : true), "ranks and address in 16 bits each");
    extern __shared__ __align__(16) float smem[];
    tc::grid_dep_launch();
    const int nb = S / Bs;
    float *s_cbT = smem;                                 // [M][DM][C]: element i of codeword (m, c) at (m DM + i) C + c
    uint8_t *s_q = (uint8_t *)(s_cbT + C * D);           // [128] query rows, pitch QP
    int32_t *s_addr = (int32_t *)(s_q + 128 * QP);       // [nb]
    int32_t *s_ids = s_addr + nb;                        // [nb]
    float *s_wsc = (float *)(s_ids + nb);                // [4][M*C] scores of the query a warp walks
    int *s_wtop = (int *)(s_wsc + 4 * M * C);            // [4][TP] its probes
    const int h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * H + h;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t_lo = blockIdx.x * 128;
    {
        constexpr int CH = D * (int)sizeof(T) / 16;
        const uint8_t *src = (const uint8_t *)(Q + (bh * S + t_lo) * D);
        for (int i = tid; i < 128 * CH; i += blockDim.x) {
            const int r = i / CH, c = i % CH;
            const bool ok = t_lo + r < S;
            tc::cp_async16(s_q + r * QP + 16 * c, ok ? (const void *)(src + (size_t)r * (D * sizeof(T)) + 16 * c) : Q, ok);
        }
    }
    {
        const float4 *src = (const float4 *)(cb + (size_t)h * C * D);
        for (int i4 = tid; i4 < C * D / 4; i4 += blockDim.x) {
            const float4 f = __ldg(src + i4);
            const int mc = (4 * i4) / DM, i = (4 * i4) % DM;
            float *dst = s_cbT + ((mc / C) * DM + i) * C + mc % C;
            dst[0] = f.x;
            dst[C] = f.y;
            dst[2 * C] = f.z;
            dst[3 * C] = f.w;
        }
    }
    tc::cp_async_wait_all();
    __syncthreads();

    const int t = t_lo + tid;
    const T *qrow = (const T *)(s_q + tid * QP);
    float s[M][C];
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const T *qm[1] = {qrow + m * DM};
        float sm[1][C];
        sub_scores_x2<T, DM, C, 1>(qm, s_cbT + m * DM * C, sm);
#pragma unroll
        for (int c = 0; c < C; ++c) s[m][c] = sm[0][c];
    }

    tc::grid_dep_wait();
    for (int i = tid; i < nb; i += blockDim.x) {
        s_addr[i] = post_addr[bh * nb + i];
        s_ids[i] = post_ids[bh * nb + i];
    }
    __syncthreads();

    int n_sel = 0, lt_r = 0, ign = 0;
    int top_a[TP];
    bool walk = false, finite = true;
    if (t < S) {
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int c = 0; c < C; ++c) finite = finite && fabsf(s[m][c]) <= 3.0e38f;

        // lazily ranked codes of each subspace
        float ov[M][C];
        uint8_t oc[M][C];
        unsigned taken[M];
        int ne[M];
        auto extract = [&](int m) {
#pragma unroll
            for (int mm = 0; mm < M; ++mm) {
                if (mm != m) continue;
                float best = -INFINITY;
                int bc = -1;
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    const bool better = !((taken[mm] >> c) & 1u) && (bc < 0 || s[mm][c] > best);
                    best = better ? s[mm][c] : best;
                    bc = better ? c : bc;
                }
                taken[mm] |= 1u << bc;
                ov[mm][ne[mm]] = best;
                oc[mm][ne[mm]] = (uint8_t)bc;
                ++ne[mm];
            }
        };
        auto gscore = [&](unsigned r) {
            float g = ov[0][r & RMASK];
#pragma unroll
            for (int m = 1; m < M; ++m) g = __fadd_rn(g, ov[m][(r >> (RB * m)) & RMASK]);
            return g;
        };
        auto address = [&](unsigned r) {
            int a = 0;
#pragma unroll
            for (int m = 0; m < M; ++m) a = a * C + oc[m][(r >> (RB * m)) & RMASK];
            return a;
        };

        walk = !finite;
        if (finite) {
            float G = 0.f;
#pragma unroll
            for (int m = 0; m < M; ++m) {
                float mx = 0.f;
#pragma unroll
                for (int c = 0; c < C; ++c) mx = fmaxf(mx, fabsf(s[m][c]));
                G += mx;
            }
            int e2;
            frexpf(2.f * G + 1e-30f, &e2);
            const float delta = (float)(M + 1) * ldexpf(1.f, e2 - 24);
#pragma unroll
            for (int m = 0; m < M; ++m) {
                taken[m] = 0u;
                ne[m] = 0;
                extract(m);
            }
            // the frontier in registers, sorted in the probe order (entry x precedes y when g_x > g_y, or
            // g_x == g_y and a_x < a_y), keyed by (a << 16) | r; only TP entries are kept: one that ranks below TP
            // others can never be among the TP pops
            float fg[TP];
            unsigned fk[TP];
            auto first = [](float g1, unsigned k1, float g2, unsigned k2) {
                return g1 > g2 || (g1 == g2 && (k1 >> 16) < (k2 >> 16));
            };
#pragma unroll
            for (int i = 0; i < TP; ++i) {
                fg[i] = -INFINITY;
                fk[i] = 0xffffffffu;
            }
            fg[0] = gscore(0u);
            fk[0] = ((unsigned)address(0u) << 16);
            float gT = 0.f;
            for (int np = 0; np < TP && !walk; ++np) {
                const float g = fg[0];
                const unsigned key = fk[0];
                const unsigned r = key & 0xffffu;
                const int a = (int)(key >> 16);
                top_a[np] = a;
                gT = g;
#pragma unroll
                for (int i = 0; i + 1 < TP; ++i) {
                    fg[i] = fg[i + 1];
                    fk[i] = fk[i + 1];
                }
                fg[TP - 1] = -INFINITY;
                fk[TP - 1] = 0xffffffffu;
                // children: raise one rank at or after the last nonzero one
                const int k0 = r == 0u ? 0 : (31 - __clz((int)r)) / RB;
#pragma unroll
                for (int k = 0; k < M; ++k) {
                    if (k < k0) continue;
                    const int rk = (int)((r >> (RB * k)) & RMASK);
                    if (rk + 1 >= C) continue;
                    if (ne[k] == rk + 1) extract(k);
                    const unsigned cr = r + (1u << (RB * k));
                    const float cv = gscore(cr);
                    const int ca = address(cr);
                    if (cv == g && ca < a) walk = true;  // the child would precede its parent
                    const unsigned ck = ((unsigned)ca << 16) | cr;
                    // insert: entries from the first one the child precedes move down by one
#pragma unroll
                    for (int i = TP - 1; i >= 0; --i) {
                        const bool here = first(cv, ck, fg[i], fk[i]);
                        const bool above = i > 0 && first(cv, ck, fg[i > 0 ? i - 1 : 0], fk[i > 0 ? i - 1 : 0]);
                        if (here) {
                            fg[i] = above ? fg[i > 0 ? i - 1 : 0] : cv;
                            fk[i] = above ? fk[i > 0 ? i - 1 : 0] : ck;
                        }
                    }
                }
            }
            if (!walk && fg[0] == gT) {  // (an empty slot holds -inf; every score is finite here)
                // the tie at the T-th probe runs on into unvisited tuples: exact only without absorbed scores
#pragma unroll
                for (int m = 0; m < M; ++m)
                    while (ne[m] < C) extract(m);
#pragma unroll
                for (int m = 0; m < M; ++m)
                    for (int k = 0; k + 1 < C; ++k) {
                        const float gap = ov[m][k] - ov[m][k + 1];
                        if (gap > 0.f && gap <= delta) walk = true;
                    }
            }
        }
        if (walk && !finite) {
            // every address of the grid, in address order (non-finite scores: the sequential order of pushes
            // decides, as in the general kernel)
            log_walk(counters, walk_log, (long long)bh * S + t);
            float sl[M * C];  // indexable copy of the scores
#pragma unroll
            for (int m = 0; m < M; ++m)
#pragma unroll
                for (int c = 0; c < C; ++c) sl[m * C + c] = s[m][c];
            TopT top;
            top.init(TP);
            int A = 1;
#pragma unroll
            for (int m = 0; m < M; ++m) A *= C;
            for (int a = 0; a < A; ++a) {
                int rem = a, code[M];
#pragma unroll
                for (int m = M - 1; m >= 0; --m) {
                    code[m] = rem % C;
                    rem /= C;
                }
                float g = sl[code[0]];
#pragma unroll
                for (int m = 1; m < M; ++m) g = __fadd_rn(g, sl[m * C + code[m]]);
                top.push(g, a);
            }
#pragma unroll
            for (int k = 0; k < TP; ++k) top_a[k] = top.a[k];
        }

    }
    // queries whose best-first walk could not certify its probes (finite scores): the whole grid, scored by the
    // warp together (lane l takes the addresses l, l + 32, ...; each keeps its own top TP; TP rounds of a warp
    // argmax merge them).  For finite scores the probe order is a strict total order, so this equals the
    // sequential walk.
    {
        unsigned wm = __ballot_sync(0xffffffffu, t < S && walk && finite);
        float *wsc = s_wsc + warp * M * C;
        int *wtop = s_wtop + warp * TP;
        while (wm) {
            const int src = __ffs(wm) - 1;
            wm &= wm - 1;
            if (lane == src) {
                log_walk(counters, walk_log, (long long)bh * S + t);
#pragma unroll
                for (int m = 0; m < M; ++m)
#pragma unroll
                    for (int c = 0; c < C; ++c) wsc[m * C + c] = s[m][c];
            }
            __syncwarp();
            TopT top;
            top.init(TP);
            int A = 1;
#pragma unroll
            for (int m = 0; m < M; ++m) A *= C;
            for (int a = lane; a < A; a += 32) {
                int rem = a, code[M];
#pragma unroll
                for (int m = M - 1; m >= 0; --m) {
                    code[m] = rem % C;
                    rem /= C;
                }
                float g = wsc[code[0]];
#pragma unroll
                for (int m = 1; m < M; ++m) g = __fadd_rn(g, wsc[m * C + code[m]]);
                top.push(g, a);
            }
            int ptr = 0;
            for (int r = 0; r < TP; ++r) {
                float bv = ptr < top.n ? top.v[ptr] : -INFINITY;
                int ba = ptr < top.n ? top.a[ptr] : 0x7fffffff;
                int bl = lane;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov2 = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oa = __shfl_xor_sync(0xffffffffu, ba, o);
                    const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
                    if (TopT::before(ov2, oa, bv, ba)) { bv = ov2; ba = oa; bl = ol; }
                }
                if (lane == 0) wtop[r] = ba;
                if (lane == bl) ++ptr;
            }
            __syncwarp();
            if (lane == src) {
#pragma unroll
                for (int k = 0; k < TP; ++k) top_a[k] = wtop[k];
            }
            __syncwarp();
        }
    }
    if (t < S) {
        // union of the probed lists in probe order, causal filter, E cap
        const int lim = t / Bs - L;
        int cid[E];
#pragma unroll
        for (int e = 0; e < E; ++e) cid[e] = 0;
        int nc = 0;
        for (int r = 0; r < TP && nc < E; ++r) {
            const int a = top_a[r];
            int lo = 0, hi = nb;  // first entry of address a
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (s_addr[mid] < a) lo = mid + 1;
                else hi = mid;
            }
            for (int k = lo; k < nb && s_addr[k] == a && k - lo < cap && nc < E; ++k) {
                const int j = s_ids[k];
                if (j > lim) break;
#pragma unroll
                for (int e = 0; e < E; ++e)
                    if (e == nc) cid[e] = j;
                ++nc;
            }
        }
        const int nr = rerank_thread<T, D, E, R>(qrow, kbar + bh * nb * D, cid, nc, forced, sel + (bh * S + t) * R, t,
                                                 bh, S, Bs, L, &ign);
        n_sel = nr;
        lt_r = nr < R;
    }
    for (int o = 16; o > 0; o >>= 1) {
        n_sel += __shfl_xor_sync(0xffffffffu, n_sel, o);
        lt_r += __shfl_xor_sync(0xffffffffu, lt_r, o);
        ign += __shfl_xor_sync(0xffffffffu, ign, o);
    }
    if ((threadIdx.x & 31) == 0) {
        if (lt_r) atomicAdd(&counters[kCntQueriesLtR], (unsigned long long)lt_r);
        if (n_sel) atomicAdd(&counters[kCntRemoteSel], (unsigned long long)n_sel);
        if (ign) atomicAdd(&counters[kCntForcedIgnored], (unsigned long long)ign);
    }
}

cudaError_t launch_summaries(const Plan &p, const void *K, const float *cb, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    float *kbar = (float *)ws_ptr(p, ws, kRegKbar);
    int32_t *addr = (int32_t *)ws_ptr(p, ws, kRegAddr);
    unsigned long long *cnt = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    cudaError_t e = cudaMemsetAsync(cnt, 0, kCntN * 8, s);
    if (e != cudaSuccess) return e;
    // blocks per warp: about one wave of 6 CTAs (24 warps) per SM over all blocks; a codebook too large for
    // shared memory takes the plain kernel (one CTA per block)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long blocks = (long long)c.B * c.H * p.nb;
    const int bpw = (int)std::min<long long>(16, std::max<long long>(1, (blocks + 24ll * sms - 1) / (24ll * sms)));
    const size_t smem = summary_smem(c.M, c.C, c.Bs, c.d, (int)p.es);
    if (smem > 160 * 1024) {
        dim3 g0(p.nb, c.H, c.B);
        if (c.dtype == MONO_BF16)
            k_summary_assign<__nv_bfloat16><<<g0, 128, 0, s>>>((const __nv_bfloat16 *)K, cb, kbar, addr, c.S, c.d,
                                                               c.Bs, c.M, c.C, c.H);
        else
            k_summary_assign<float><<<g0, 128, 0, s>>>((const float *)K, cb, kbar, addr, c.S, c.d, c.Bs, c.M, c.C, c.H);
        count_launches(1);
        return cudaGetLastError();
    }
    dim3 g1((p.nb + 4 * bpw - 1) / (4 * bpw), c.H, c.B);
#define MONO_SUMW(TT, DD)                                                                                         \
    do {                                                                                                          \
        auto kern = k_summary_assign_w<TT, DD>;                                                                   \
        if (smem > 48 * 1024 &&                                                                                   \
            (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) \
            return e;                                                                                             \
        kern<<<g1, 128, smem, s>>>((const TT *)K, cb, kbar, addr, c.S, c.Bs, c.M, c.C, c.H, bpw);               \
    } while (0)
    if (c.dtype == MONO_BF16) {
        if (c.d == 64) MONO_SUMW(__nv_bfloat16, 64);
        else MONO_SUMW(__nv_bfloat16, 128);
    } else {
        if (c.d == 64) MONO_SUMW(float, 64);
        else MONO_SUMW(float, 128);
    }
#undef MONO_SUMW
    count_launches(1);
    return cudaGetLastError();
}

// a kernel launched so that it may start while the kernel before it on the
// stream still runs (it waits for that kernel itself: griddepcontrol.wait)
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_k(void (*kern)(KArgs...), dim3 grid, int block, size_t smem, cudaStream_t s,
                                Args... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = dim3(block);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, (KArgs)args...);
}

cudaError_t launch_lists(const Plan &p, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    // the kernel clears the statistics the probe fills (so that the probe can follow it directly), and is
    // launched programmatically after the summaries: it may start while they run and waits for them itself
    unsigned long long *stats = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    dim3 g2(c.H, c.B);
    const int32_t *addr = (const int32_t *)ws_ptr(p, ws, kRegAddr);
    int32_t *ids = (int32_t *)ws_ptr(p, ws, kRegPostIds), *saddr = (int32_t *)ws_ptr(p, ws, kRegPostAddr);
    int32_t *rank = (int32_t *)ws_ptr(p, ws, kRegPostRank), *ov = (int32_t *)ws_ptr(p, ws, kRegOverflow);
    // dynamic shared memory beyond the default 48 KB (with the kernels' static arrays) needs the opt-in
    // attribute: up to 8192 blocks take 64 KB of addresses and ranks in the dense kernel
    cudaError_t e = cudaSuccess;
    if (c.flags & MONO_FLAG_REDIRECT) {
        const size_t dyn = redirect_smem(p.A, p.nb);
        if (dyn + 64 > 48 * 1024 &&
            (e = cudaFuncSetAttribute(k_posting_redirect, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn)) !=
                cudaSuccess)
            return e;
        e = launch_pdl_k(k_posting_redirect, g2, 1024, dyn, s, addr, ids, saddr, rank, ov, p.nb, c.cap, c.H,
                         (int)p.A, stats);
    } else if (p.A <= kDenseA) {
        const size_t dyn = (size_t)p.nb * 8;
        if (dyn + sizeof(int) * (kDenseA + 64) > 48 * 1024 &&
            (e = cudaFuncSetAttribute(k_posting_dense, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn)) !=
                cudaSuccess)
            return e;
        e = launch_pdl_k(k_posting_dense, g2, 1024, dyn, s, addr, ids, saddr, rank, ov, p.nb, c.cap, c.H, (int)p.A,
                         stats);
    } else {
        const size_t dyn = (size_t)p.nb * sizeof(int32_t);
        if (dyn + sizeof(int) * 32 > 48 * 1024 &&
            (e = cudaFuncSetAttribute(k_posting_build, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn)) !=
                cudaSuccess)
            return e;
        e = launch_pdl_k(k_posting_build, g2, 1024, dyn, s, addr, ids, saddr, rank, ov, p.nb, c.cap, c.H, stats);
    }
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

// a probe kernel, launched so that it may start while the lists kernel before
// it on the stream still runs (it waits for the lists itself: tc::grid_dep_wait)
template <typename... KArgs, typename... Args>
static cudaError_t launch_after_lists(void (*kern)(KArgs...), dim3 grid, int threads, size_t smem, cudaStream_t s,
                                      Args... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = dim3(threads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, (KArgs)args...);
}

cudaError_t launch_queries(const Plan &p, const void *Q, const float *cb, const int32_t *forced, int32_t *sel,
                           void *ws, cudaStream_t s, bool reset_stats) {
    const mono_config &c = p.cfg;
    unsigned long long *cnt = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    int32_t *walk_log = (int32_t *)ws_ptr(p, ws, kRegWalkLog);
    cudaError_t e = cudaSuccess;
    if (reset_stats && (e = cudaMemsetAsync(cnt, 0, kCntStats * 8, s)) != cudaSuccess)  // the error word is kept
        return e;
    if (c.R == 0) return cudaSuccess;  // nothing to select: sel has no entries
    const float *kbar = (const float *)ws_ptr(p, ws, kRegKbar);
    const int32_t *ids = (const int32_t *)ws_ptr(p, ws, kRegPostIds);
    const int32_t *saddr = (const int32_t *)ws_ptr(p, ws, kRegPostAddr);
    dim3 g3((c.S + 127) / 128, c.H, c.B);
    const bool bf = c.dtype == MONO_BF16;
    // compile-time shapes of the configured workloads; any other shape takes the general kernel
#define MONO_M2(TT, DD, CC, TPP, EE, RR)                                                                          \
    if (c.M == 2 && c.d == DD && c.C == CC && c.T == TPP && c.E == EE && c.R == RR) {                           \
        const size_t sm2 = probe_m2_smem<TT, DD, CC, EE>(p.nb);                                                 \
        auto kern = k_probe_m2<TT, DD, CC, TPP, EE, RR>;                                                        \
        if (sm2 > 48 * 1024 &&                                                                                   \
            (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2)) != cudaSuccess) \
            return e;                                                                                            \
        const dim3 gm2((c.S + probe_threads<CC>() * probe_nq<CC>() - 1) / (probe_threads<CC>() * probe_nq<CC>()), c.H, \
                       c.B);                  \
        if ((e = launch_after_lists(kern, gm2, probe_threads<CC>(), sm2, s, (const TT *)Q, kbar, cb, ids, saddr, forced, sel, cnt,        \
                                    walk_log, c.S, c.H, c.Bs, c.L, c.cap)) != cudaSuccess)                          \
            return e;                                                                                            \
        count_launches(1);                                                                                       \
        return cudaGetLastError();                                                                               \
    }
    if (bf) {
        MONO_M2(__nv_bfloat16, 64, 16, 4, 5, 2)
        MONO_M2(__nv_bfloat16, 128, 32, 8, 8, 4)
    } else {
        MONO_M2(float, 64, 16, 4, 5, 2)
        MONO_M2(float, 64, 8, 4, 5, 2)
    }
#undef MONO_M2
#define MONO_BF(TT, DD, MM, CC, TPP, EE, RR)                                                                      \
    if (c.M == MM && c.d == DD && c.C == CC && c.T == TPP && c.E == EE && c.R == RR) {                          \
        const size_t smb = probe_bf_smem<TT, DD, MM, CC>(p.nb);                                                  \
        auto kern = k_probe_bf<TT, DD, MM, CC, TPP, EE, RR>;                                                     \
        if (smb > 48 * 1024 &&                                                                                   \
            (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smb)) != cudaSuccess) \
            return e;                                                                                            \
        if ((e = launch_after_lists(kern, g3, 128, smb, s, (const TT *)Q, kbar, cb, ids, saddr, forced, sel, cnt,         \
                                    walk_log, c.S, c.H, c.Bs, c.L, c.cap)) != cudaSuccess)                          \
            return e;                                                                                            \
        count_launches(1);                                                                                       \
        return cudaGetLastError();                                                                               \
    }
    if (bf) {
        MONO_BF(__nv_bfloat16, 128, 4, 16, 16, 8, 4)
        MONO_BF(__nv_bfloat16, 64, 4, 16, 16, 5, 2)
        MONO_BF(__nv_bfloat16, 64, 4, 4, 8, 8, 4)
    } else {
        MONO_BF(float, 64, 4, 4, 8, 8, 4)
    }
#undef MONO_BF
    const size_t smem = (size_t)c.C * c.d * 4 + (size_t)p.nb * 8;
#define MONO_LAUNCH_PR(TT, DD)                                                                                     \
    do {                                                                                                           \
        auto kern = k_probe_rerank<TT, DD>;                                                                        \
        if (smem > 48 * 1024) {                                                                                    \
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                \
            if (e != cudaSuccess) return e;                                                                        \
        }                                                                                                          \
        if ((e = launch_after_lists(kern, g3, 128, smem, s, (const TT *)Q, kbar, cb, ids, saddr, forced, sel, cnt,        \
                                    walk_log, c.S, c.H, c.Bs, c.L, c.R, c.E, c.M, c.C, c.T, c.cap)) != cudaSuccess)  \
            return e;                                                                                              \
    } while (0)
    if (bf && c.d == 64) MONO_LAUNCH_PR(__nv_bfloat16, 64);
    else if (bf) MONO_LAUNCH_PR(__nv_bfloat16, 128);
    else if (c.d == 64) MONO_LAUNCH_PR(float, 64);
    else MONO_LAUNCH_PR(float, 128);
#undef MONO_LAUNCH_PR
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mono

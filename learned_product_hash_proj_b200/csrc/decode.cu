// decode.cu -- one new token per sequence against caller-owned caches.
//
// Every stage of the mixer is causal, so decode step t computes row t of the
// batch forward on the first t+1 tokens ("Monodratic Routes Sparse Attention
// with Learned Product Hashes", Key Points: bounded causal posting lists; the
// remio.ai article, section on retrieval decisions: lists keep the earliest
// blocks of each address up to their capacity).  What is incremental:
//   * the key and value of position t are appended to the cache;
//   * when t completes block j, its summary kbar_j (mean of its post-RoPE
//     keys), its product address and its append to that address's posting
//     list (kept while the list holds fewer than cap blocks, else counted as
//     overflow).  A list is a chain head -> next -> ... in ascending block id;
//   * the query is routed against the lists: top-T product addresses by the
//     summed subspace scores, union of their lists in probe order, causal
//     filter j <= t/Bs - L, E cap, rerank by q.kbar, top R;
//   * exact softmax over the tokens of the selected blocks plus the local
//     tokens [max(0, t/Bs - L + 1) * Bs, t].
// Routing decisions use the fp32 order of the batch kernels: dot products as
// fma chains in ascending element order from +0, block sums in ascending t,
// grid scores summed in ascending subspace order, ties to the lowest code,
// address and block id.  For one query the exact top T is found by scoring
// every one of the C^M addresses (C^M <= 4096).
#include <cuda_runtime.h>

#include <math.h>

#include <initializer_list>

#include "internal.cuh"
#include "mono.h"
#include "tc.cuh"

#include <cooperative_groups.h>
namespace cg = cooperative_groups;

namespace mono {
namespace {

constexpr int kDecMaxA = 4096;

struct DecLayout {
    size_t off[MONO_DEC_NREGIONS];
    size_t bytes[MONO_DEC_NREGIONS];
    size_t total;
};

DecLayout dec_layout(const Plan &p) {
    const mono_config &c = p.cfg;
    const size_t B = c.B, H = c.H, S = c.S, d = c.d, nb = p.nb, A = (size_t)p.A, es = p.es;
    const size_t R = c.R > 0 ? c.R : 1;
    DecLayout L{};
    size_t sz[MONO_DEC_NREGIONS] = {};
    sz[MONO_DEC_K] = B * H * S * d * es;
    sz[MONO_DEC_V] = B * H * S * d * es;
    sz[MONO_DEC_KBAR] = B * H * nb * d * 4;
    sz[MONO_DEC_ADDR] = B * H * nb * 4;
    sz[MONO_DEC_COUNT] = B * H * A * 4;
    sz[MONO_DEC_HEAD] = B * H * A * 4;
    sz[MONO_DEC_TAIL] = B * H * A * 4;
    sz[MONO_DEC_NEXT] = B * H * nb * 4;
    sz[MONO_DEC_OVERFLOW] = B * H * 4;
    sz[MONO_DEC_Q] = B * H * d * es;
    sz[MONO_DEC_SEL] = B * H * R * 4;
    sz[MONO_DEC_O] = B * H * d * es;
    size_t o = 0;
    for (int r = 0; r < MONO_DEC_NREGIONS; ++r) {
        L.off[r] = o;
        L.bytes[r] = sz[r];
        o += (sz[r] + 255) / 256 * 256;
    }
    L.total = o;
    return L;
}

struct DecPtrs {
    void *K, *V, *Q, *O;
    float *kbar;
    int32_t *addr, *count, *head, *tail, *next, *overflow, *sel;
};

DecPtrs dec_ptrs(const DecLayout &L, void *cache) {
    char *c = (char *)cache;
    DecPtrs P;
    P.K = c + L.off[MONO_DEC_K];
    P.V = c + L.off[MONO_DEC_V];
    P.Q = c + L.off[MONO_DEC_Q];
    P.O = c + L.off[MONO_DEC_O];
    P.kbar = (float *)(c + L.off[MONO_DEC_KBAR]);
    P.addr = (int32_t *)(c + L.off[MONO_DEC_ADDR]);
    P.count = (int32_t *)(c + L.off[MONO_DEC_COUNT]);
    P.head = (int32_t *)(c + L.off[MONO_DEC_HEAD]);
    P.tail = (int32_t *)(c + L.off[MONO_DEC_TAIL]);
    P.next = (int32_t *)(c + L.off[MONO_DEC_NEXT]);
    P.overflow = (int32_t *)(c + L.off[MONO_DEC_OVERFLOW]);
    P.sel = (int32_t *)(c + L.off[MONO_DEC_SEL]);
    return P;
}

// dot product of two rows of n elements, lanes taking 16-byte chunks (n * sizeof(T)
// a multiple of 16 and both rows 16-byte aligned); fp32 accumulation, warp-reduced
template <typename T>
__device__ __forceinline__ float row_dot_part(const T *a, const T *b, int n, int lane) {
    constexpr int V = 16 / sizeof(T);
    float acc = 0.f;
#pragma unroll 4  // the loads of four steps in flight at once
    for (int k = lane * V; k < n; k += 32 * V) {
        const uint4 ua = *(const uint4 *)(a + k), ub = *(const uint4 *)(b + k);
        const T *ta = (const T *)&ua, *tb = (const T *)&ub;
#pragma unroll
        for (int e = 0; e < V; ++e) acc = fmaf(to_f(ta[e]), to_f(tb[e]), acc);
    }
    return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// projection of one token per sequence: one warp per interleaved output pair
// (2i, 2i+1) of one head of one of Q, K, V, for all B sequences; lanes split
// the W inputs, fp32 accumulation; RoPE on Q and K at position t (angles in
// fp64); q to the Q region, k and v to the caches at position t.
// grid ceil(3 H d/2 / 8), 256 threads.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_dec_project(const T *__restrict__ x, const T *__restrict__ Wq,
                                                     const T *__restrict__ Wk, const T *__restrict__ Wv, T *__restrict__ q,
                                                     T *__restrict__ Kc, T *__restrict__ Vc, int t, int B, int W, int H,
                                                     int d, int S, double theta) {
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int pairs = H * d / 2;
    if (gw >= 3 * pairs) return;
    const int which = gw / pairs, pr = gw % pairs;  // 0 q, 1 k, 2 v
    const int h = (2 * pr) / d, i = pr % (d / 2);
    const int n0 = h * d + 2 * i;
    const T *Wm = which == 0 ? Wq : (which == 1 ? Wk : Wv);
    const T *w0 = Wm + (size_t)n0 * W, *w1 = w0 + W;
    // before the previous kernel of the stream completes: the weight rows into L2 and the rotation angle
    for (int o = lane * 64; o < W * (int)sizeof(T); o += 32 * 64) {
        tc::prefetch_l2((const char *)w0 + o);
        tc::prefetch_l2((const char *)w1 + o);
    }
    double c = 1.0, s = 0.0;
    if (which < 2) {
        const double ang = (double)t * pow(theta, -2.0 * (double)i / (double)d);
        c = cos(ang);
        s = sin(ang);
    }
    tc::grid_dep_wait();  // x may come from it, and the previous step's kernels read q and the caches
    tc::grid_dep_launch();
    for (int b = 0; b < B; ++b) {
        const T *xb = x + (size_t)b * W;
        const float p0 = row_dot_part(xb, w0, W, lane), p1 = row_dot_part(xb, w1, W, lane);
        const float a0 = warp_sum(p0);
        const float a1 = warp_sum(p1);
        if (lane == 0) {
            float r0 = a0, r1 = a1;
            if (which < 2) {
                r0 = (float)((double)a0 * c - (double)a1 * s);
                r1 = (float)((double)a0 * s + (double)a1 * c);
            }
            T *dst;
            if (which == 0) dst = q + ((size_t)b * H + h) * d + 2 * i;
            else dst = (which == 1 ? Kc : Vc) + (((size_t)b * H + h) * S + t) * d + 2 * i;
            dst[0] = from_f<T>(r0);
            dst[1] = from_f<T>(r1);
        }
    }
}

// summary and address of block j of (b, h): lane owns columns lane, lane+32, ...
// Same arithmetic as the batch summaries.  Returns the address (all lanes).
template <typename T>
__device__ int dec_summary(const T *Kc, const float *cb, float *kbar, int32_t *addr, size_t bh, int h, int j, int S,
                           int Bs, int d, int M, int C, int nb, float *s_kb, float *s_sc) {
    const int lane = threadIdx.x & 31;
    const T *rows = Kc + (bh * S + (size_t)j * Bs) * d;
    for (int i = lane; i < d; i += 32) {
        float acc = 0.0f;
#pragma unroll 8
        for (int tt = 0; tt < Bs; ++tt) acc = __fadd_rn(acc, to_f(rows[(size_t)tt * d + i]));
        const float v = __fdiv_rn(acc, (float)Bs);
        s_kb[i] = v;
        kbar[(bh * nb + j) * d + i] = v;
    }
    __syncwarp();
    const int dm = d / M;
    for (int mc = lane; mc < M * C; mc += 32) {
        const int m = mc / C;
        const float *w = cb + ((size_t)h * M * C + mc) * dm;
        float a = 0.0f;
        for (int i = 0; i < dm; ++i) a = __fmaf_rn(s_kb[m * dm + i], w[i], a);
        s_sc[mc] = a;
    }
    __syncwarp();
    int ad = 0;
    if (lane == 0) {
        long long a = 0;
        for (int m = 0; m < M; ++m) {
            float best = s_sc[m * C];
            int bc = 0;
            for (int c2 = 1; c2 < C; ++c2)
                if (s_sc[m * C + c2] > best) { best = s_sc[m * C + c2]; bc = c2; }
            a = a * C + bc;
        }
        ad = (int)a;
        addr[bh * nb + j] = ad;
    }
    __syncwarp();
    return __shfl_sync(0xffffffffu, ad, 0);
}

// append block j to the list of address a (one thread).  A tail outside
// [0, nb) -- a cache that mono_decode_prefill never initialised -- starts the
// list afresh instead of writing out of bounds.
__device__ __forceinline__ void dec_append(int32_t *count, int32_t *head, int32_t *tail, int32_t *next,
                                           int32_t *overflow, size_t bh, long long A, int nb, int a, int j, int cap) {
    const size_t ba = bh * A + a;
    int cnt = count[ba];
    if (cnt < 0 || (cnt > 0 && cnt < cap && (unsigned)tail[ba] >= (unsigned)nb)) cnt = 0;
    if (cnt < cap) {
        if (cnt == 0) head[ba] = j;
        else next[bh * nb + tail[ba]] = j;
        tail[ba] = j;
        next[bh * nb + j] = -1;
    } else {
        overflow[bh] += 1;
    }
    count[ba] = cnt + 1;
}

// block completed at position t (one warp per (b, h)); grid (H, B), 32 threads
template <typename T>
__global__ void __launch_bounds__(32) k_dec_block(const T *__restrict__ Kc, const float *__restrict__ cb, DecPtrs P, int t,
                                                  int S, int Bs, int d, int M, int C, int H, int nb, long long A,
                                                  int cap) {
    __shared__ float s_kb[kMaxD];
    __shared__ float s_sc[kMaxM * kMaxC];
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t bh = (size_t)b * H + h;
    const int j = t / Bs;
    tc::grid_dep_wait();  // the block's last key (projection)
    tc::grid_dep_launch();
    const int a = dec_summary<T>(Kc, cb, P.kbar, P.addr, bh, h, j, S, Bs, d, M, C, nb, s_kb, s_sc);
    if (threadIdx.x == 0) dec_append(P.count, P.head, P.tail, P.next, P.overflow, bh, A, nb, a, j, cap);
}

// prefill: summaries of blocks [0, nb0); grid (nb0, H, B), 32 threads
template <typename T>
__global__ void __launch_bounds__(32) k_dec_prefill_summaries(const T *__restrict__ Kc, const float *__restrict__ cb,
                                                              DecPtrs P, int S, int Bs, int d, int M, int C, int H,
                                                              int nb) {
    __shared__ float s_kb[kMaxD];
    __shared__ float s_sc[kMaxM * kMaxC];
    const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * H + h;
    dec_summary<T>(Kc, cb, P.kbar, P.addr, bh, h, j, S, Bs, d, M, C, nb, s_kb, s_sc);
}

// prefill: empty lists, then blocks [0, nb0) appended in ascending order; grid (H, B), 32 threads
__global__ void __launch_bounds__(32) k_dec_prefill_lists(DecPtrs P, int nb0, int H, int nb, long long A, int cap) {
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t bh = (size_t)b * H + h;
    for (long long a = threadIdx.x; a < A; a += 32) {
        P.count[bh * A + a] = 0;
        P.head[bh * A + a] = -1;
        P.tail[bh * A + a] = -1;
    }
    for (int j = threadIdx.x; j < nb; j += 32) P.next[bh * nb + j] = -1;
    __syncwarp();
    if (threadIdx.x == 0) {
        P.overflow[bh] = 0;
        for (int j = 0; j < nb0; ++j)
            dec_append(P.count, P.head, P.tail, P.next, P.overflow, bh, A, nb, P.addr[bh * nb + j], j, cap);
    }
}

__device__ __forceinline__ bool before(float v1, int a1, float v2, int a2) {
    return v1 > v2 || (v1 == v2 && a1 < a2);
}

// ---------------------------------------------------------------------------
// routing of the step's query, one warp per (b, h); grid (H, B), 32 threads,
// dynamic shared memory M C (d/M + 1) floats (the head's codewords, one
// padding float per row so that the 32 lanes' chains read 32 banks).  TPM >=
// T is the length of each lane's sorted list of its best addresses, fixed at
// compile time so that the list stays in registers (a lane's first T entries
// are its top T; the entries after them are never reached by the merge).
// ---------------------------------------------------------------------------
template <typename T, int TPM>
__global__ void __launch_bounds__(32) k_dec_route(const T *__restrict__ q, const float *__restrict__ cb,
                                                  const int32_t *__restrict__ forced, DecPtrs P, int t, int Bs, int L,
                                                  int R, int E, int M, int C, int TP, int cap, int H, int d, int nb,
                                                  long long A) {
    extern __shared__ __align__(16) float s_cb[];  // [M][C][dm + 1] of head h
    __shared__ float s_q[kMaxD];
    __shared__ float s_sc[kMaxM * kMaxC];
    __shared__ int s_top[kMaxT];
    __shared__ int s_head[kMaxT], s_cnt[kMaxT];
    __shared__ int s_cand[kMaxE];
    __shared__ int s_walk[kMaxT][kMaxE];  // the first eligible entries of each probed list
    __shared__ float s_score[kMaxE];
    __shared__ __align__(16) float s_kb[kMaxE > 8 ? 8 : kMaxE][kMaxD + 4];  // candidate kbar rows, 8 at a time
    const int lane = threadIdx.x;
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t bh = (size_t)b * H + h;
    const int lim = t / Bs - L;  // the latest block a query at t may select
    // the codewords by asynchronous copies: no lane waits for one load before issuing the next
    const int dm = d / M;
    {
        const float *src = cb + (size_t)h * C * d;
        for (int i = lane; i < C * d; i += 32)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc::smem_u32(s_cb + (i / dm) * (dm + 1) +
                                                                                       i % dm)),
                         "l"(src + i)
                         : "memory");
    }
    tc::grid_dep_wait();  // q (projection) and the lists (block update) are complete
    tc::grid_dep_launch();
    for (int i = lane; i < d; i += 32) s_q[i] = to_f(q[bh * d + i]);
    tc::cp_async_wait_all();
    __syncwarp();
    // subspace scores: fma chains in ascending element order from +0
    for (int mc = lane; mc < M * C; mc += 32) {
        const int m = mc / C;
        const float *w = s_cb + mc * (dm + 1);
        float a = 0.0f;
        for (int i = 0; i < dm; ++i) a = __fmaf_rn(s_q[m * dm + i], w[i], a);
        s_sc[mc] = a;
    }
    __syncwarp();
    // every address scored (subspace 0 most significant, summed in ascending
    // subspace order); each lane keeps its top TPM by (score desc, address asc)
    float lv[TPM];
    int la[TPM];
#pragma unroll
    for (int k = 0; k < TPM; ++k) { lv[k] = -INFINITY; la[k] = 0x7fffffff; }
    const int A32 = (int)A;  // <= 4096 on this path
    for (int a32 = lane; a32 < A32; a32 += 32) {
        int rest = a32, radix = A32 / C;
        float v = 0.0f;
        for (int m = 0; m < M; ++m) {
            const int cm = rest / radix;
            rest -= cm * radix;
            radix /= C;
            v = m == 0 ? s_sc[cm] : __fadd_rn(v, s_sc[m * C + cm]);
        }
        if (!before(v, a32, lv[TPM - 1], la[TPM - 1])) continue;
        // insertion: the new entry moves down past every entry it precedes
        float cv = v;
        int ca = a32;
#pragma unroll
        for (int k = 0; k < TPM; ++k) {
            if (before(cv, ca, lv[k], la[k])) {
                const float tv = lv[k];
                const int ta = la[k];
                lv[k] = cv;
                la[k] = ca;
                cv = tv;
                ca = ta;
            }
        }
    }
    // merge: TP rounds of a warp argmax over the lanes' heads; the winning lane drops its head
    for (int r = 0; r < TP; ++r) {
        float bv = lv[0];
        int ba = la[0];
        int bl = lane;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oa = __shfl_xor_sync(0xffffffffu, ba, o);
            const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (before(ov, oa, bv, ba)) { bv = ov; ba = oa; bl = ol; }
        }
        if (lane == 0) s_top[r] = ba;
        if (lane == bl) {
#pragma unroll
            for (int k = 0; k + 1 < TPM; ++k) {
                lv[k] = lv[k + 1];
                la[k] = la[k + 1];
            }
            lv[TPM - 1] = -INFINITY;
            la[TPM - 1] = 0x7fffffff;
        }
    }
    __syncwarp();
    // the probed lists' heads and counts, fetched at once
    if (lane < TP) {
        const int a = s_top[lane];
        const bool ok = a >= 0 && (long long)a < A;
        s_cnt[lane] = ok ? P.count[bh * A + a] : 0;
        s_head[lane] = ok ? P.head[bh * A + a] : -1;
    }
    __syncwarp();
    // union of the probed lists in probe order, causal filter, E cap: lane r walks list r (its first E eligible
    // entries at most; at most cap kept entries; an id outside [0, nb) ends a walk), so the T chains of dependent
    // loads run side by side; then the lists are concatenated in probe order up to E
    int mine = 0;
    if (lane < TP && s_cnt[lane] > 0) {
        int steps = 0;
        for (int j = s_head[lane]; (unsigned)j < (unsigned)nb && mine < E && steps < cap;
             j = P.next[bh * nb + j], ++steps) {
            if (j > lim) break;  // ascending ids: the rest are later still
            s_walk[lane][mine++] = j;
        }
    }
    int before_me = mine;  // inclusive prefix of the walked counts over the lanes in probe order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, before_me, o);
        if (lane >= o) before_me += y;
    }
    before_me -= mine;
    for (int k = 0; k < mine && before_me + k < E; ++k) s_cand[before_me + k] = s_walk[lane][k];
    int nc = __shfl_sync(0xffffffffu, before_me + mine, 31);
    nc = nc < E ? nc : E;
    __syncwarp();
    // rerank: q . kbar_j, one candidate per lane, from rows staged 8 at a time
    for (int e0 = 0; e0 < nc; e0 += 8) {
        const int ne = min(8, nc - e0);
        for (int i = lane; i < ne * d / 4; i += 32) {
            const int e = i / (d / 4), c4 = i % (d / 4);
            tc::cp_async16((float4 *)s_kb[e] + c4, (const float4 *)(P.kbar + (bh * nb + s_cand[e0 + e]) * d) + c4,
                           true);
        }
        tc::cp_async_wait_all();
        __syncwarp();
        if (lane < ne) {
            // eight runs of d/8 elements as fma chains, added as a balanced tree (the batch rerank's order)
            float run[8];
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                float a = 0.0f;
                for (int i = l * d / 8; i < (l + 1) * d / 8; ++i) a = __fmaf_rn(s_q[i], s_kb[lane][i], a);
                run[l] = a;
            }
            s_score[e0 + lane] = __fadd_rn(__fadd_rn(__fadd_rn(run[0], run[1]), __fadd_rn(run[2], run[3])),
                                           __fadd_rn(__fadd_rn(run[4], run[5]), __fadd_rn(run[6], run[7])));
        }
        __syncwarp();
    }
    if (lane == 0) {
        // top R by (score desc, id asc), in rank order
        int ra[kMaxR];
        int nr = 0;
        unsigned used = 0;  // candidates taken (E <= 32)
        for (; nr < R && nr < nc; ++nr) {
            int bi = -1;
            for (int e = 0; e < nc; ++e)
                if (!((used >> e) & 1u) && (bi < 0 || before(s_score[e], s_cand[e], s_score[bi], s_cand[bi]))) bi = e;
            used |= 1u << bi;
            ra[nr] = s_cand[bi];
        }
        if (forced) {
            const int f = forced[bh];
            if (f >= 0 && f <= lim) {
                bool present = false;
                for (int k = 0; k < nr; ++k) present |= ra[k] == f;
                if (!present && R > 0) {
                    if (nr < R) ra[nr++] = f;
                    else ra[R - 1] = f;
                }
            }
        }
        // ascending ids, -1 padding
        for (int x = 0; x < nr; ++x)
            for (int y = 0; y + 1 < nr - x; ++y)
                if (ra[y] > ra[y + 1]) { const int tmp = ra[y]; ra[y] = ra[y + 1]; ra[y + 1] = tmp; }
        for (int k = 0; k < R; ++k) P.sel[bh * R + k] = k < nr ? ra[k] : -1;
    }
}

// ---------------------------------------------------------------------------
// attention of the step's query: the key list (R remote blocks, then the local
// tokens) is walked in chunks of CH keys whose K and V rows are copied to
// shared memory (cp.async, two buffers: chunk c+1 in flight while chunk c is
// used; at the usual sizes one chunk holds every key, so all rows are in
// flight at once).  8 warps split a chunk's keys, each with an online softmax
// (lanes own d/32 dimensions); the warps merge at the end.  fp32 throughout.
// grid (H, B), 256 threads, dynamic shared memory 2 * CH * d * sizeof(T) * 2.
// ---------------------------------------------------------------------------
template <typename T>
constexpr int dec_chunk(int d) {
    return (48 * 1024) / (d * (int)sizeof(T));  // keys per buffer: 96 KB of K and V rows
}

template <typename T>
__global__ void __launch_bounds__(256) k_dec_attend(const T *__restrict__ q, const T *__restrict__ Kc,
                                                    const T *__restrict__ Vc, const int32_t *__restrict__ sel,
                                                    T *__restrict__ O, int t, int S, int Bs, int L, int R, int H, int d,
                                                    float scale) {
    constexpr int kPer = kMaxD / 32, NW = 8;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ float s_m[NW], s_l[NW];
    __shared__ float s_acc[NW][kMaxD];
    __shared__ int s_js[kMaxR];
    __shared__ int s_nr;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = blockIdx.x, b = blockIdx.y;
    const size_t bh = (size_t)b * H + h;
    const int per = d / 32;
    const int CH = dec_chunk<T>(d);
    const int rowb = d * (int)sizeof(T);      // bytes of one K or V row
    T *bufK[2] = {(T *)dsm, (T *)(dsm + 2 * CH * rowb)};
    T *bufV[2] = {(T *)(dsm + CH * rowb), (T *)(dsm + 3 * CH * rowb)};
    const int bq = t / Bs, lim = bq - L;
    tc::grid_dep_wait();  // sel (route), q and the newest key and value (projection)
    tc::grid_dep_launch();
    if (threadIdx.x == 0) {  // the selected remote blocks; ids outside [0, t/Bs - L] are skipped
        int nr = 0;
        for (int r = 0; r < R; ++r) {
            const int j = sel[bh * R + r];
            if (j >= 0 && j <= lim) s_js[nr++] = j;
        }
        s_nr = nr;
    }
    __syncthreads();
    const int nr = s_nr;
    const int lo = max(0, bq - L + 1) * Bs;
    const int nkeys = nr * Bs + (t - lo + 1);
    auto key_of = [&](int idx) { return idx < nr * Bs ? s_js[idx / Bs] * Bs + idx % Bs : lo + (idx - nr * Bs); };
    auto stage = [&](int buf, int c0) {  // rows of keys [c0, c0 + CH) into buffer buf
        const int n = min(CH, nkeys - c0), chunks = rowb / 16;
        for (int i = threadIdx.x; i < n * chunks; i += blockDim.x) {
            const int k = i / chunks, c = i % chunks;
            const size_t row = bh * S + key_of(c0 + k);
            tc::cp_async16((uint8_t *)bufK[buf] + k * rowb + 16 * c, (const uint8_t *)(Kc + row * d) + 16 * c, true);
            tc::cp_async16((uint8_t *)bufV[buf] + k * rowb + 16 * c, (const uint8_t *)(Vc + row * d) + 16 * c, true);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    float qv[kPer];
    for (int e = 0; e < per; ++e) qv[e] = to_f(q[bh * d + lane * per + e]);
    float m = -INFINITY, l = 0.f, acc[kPer];
    for (int e = 0; e < per; ++e) acc[e] = 0.f;
    stage(0, 0);
    for (int c0 = 0, cb = 0; c0 < nkeys; c0 += CH, cb ^= 1) {
        if (c0 + CH < nkeys) {
            stage(cb ^ 1, c0 + CH);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const int n = min(CH, nkeys - c0);
        for (int k = warp; k < n; k += NW) {
            const T *kr = bufK[cb] + k * d + lane * per, *vr = bufV[cb] + k * d + lane * per;
            float part = 0.f;
            for (int e = 0; e < per; ++e) part = fmaf(qv[e], to_f(kr[e]), part);
            const float s = warp_sum(part) * scale;
            const float mn = fmaxf(m, s);
            const float corr = expf(m - mn), p = expf(s - mn);
            l = l * corr + p;
            for (int e = 0; e < per; ++e) acc[e] = fmaf(p, to_f(vr[e]), acc[e] * corr);
            m = mn;
        }
        __syncthreads();  // buffer cb is refilled two chunks later
    }
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
    }
    for (int e = 0; e < per; ++e) s_acc[warp][lane * per + e] = acc[e];
    __syncthreads();
    if (warp == 0) {
        float mm = -INFINITY;
        for (int w = 0; w < NW; ++w) mm = fmaxf(mm, s_m[w]);
        float den = 0.f, o[kPer];
        for (int e = 0; e < per; ++e) o[e] = 0.f;
        for (int w = 0; w < NW; ++w) {
            if (s_m[w] == -INFINITY) continue;  // a warp without keys
            const float f = expf(s_m[w] - mm);
            den += s_l[w] * f;
            for (int e = 0; e < per; ++e) o[e] += s_acc[w][lane * per + e] * f;
        }
        for (int e = 0; e < per; ++e) O[(size_t)b * H * d + (size_t)h * d + lane * per + e] = from_f<T>(o[e] / den);
    }
}

// ---------------------------------------------------------------------------
// the same attention split over a cluster of kDecSplit CTAs per (b, h): CTA z
// of the cluster takes the z-th share of the key list, reduces it as above
// (chunks through shared memory, 8 warps with online softmaxes, merged in the
// CTA) to a partial (max, sum, unnormalised o), and CTA 0 merges the shares
// exactly, reading the others' partials from their shared memory (distributed
// shared memory of the cluster).  grid (H * kDecSplit, B), cluster
// (kDecSplit, 1, 1), 256 threads.
// ---------------------------------------------------------------------------
constexpr int kDecSplit = 4;

template <typename T>
__global__ void __launch_bounds__(256) k_dec_attend_cl(const T *__restrict__ q, const T *__restrict__ Kc,
                                                       const T *__restrict__ Vc, const int32_t *__restrict__ sel,
                                                       T *__restrict__ O, int t, int S, int Bs, int L, int R, int H,
                                                       int d, float scale, int CH) {
    constexpr int kPer = kMaxD / 32, NW = 8;
    extern __shared__ __align__(16) uint8_t dsm[];  // two buffers of CH keys' K and V rows
    __shared__ float s_m[NW], s_l[NW];
    __shared__ float s_acc[NW][kMaxD];
    __shared__ float s_part[kMaxD + 2];  // this CTA's share: o (unnormalised) [d], max, sum
    __shared__ int s_js[kMaxR];
    __shared__ int s_nr;
    cg::cluster_group cluster = cg::this_cluster();
    const int z = (int)cluster.block_rank();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = blockIdx.x / kDecSplit, b = blockIdx.y;
    const size_t bh = (size_t)b * H + h;
    const int per = d / 32;
    const int rowb = d * (int)sizeof(T);
    T *bufK[2] = {(T *)dsm, (T *)(dsm + 2 * CH * rowb)};
    T *bufV[2] = {(T *)(dsm + CH * rowb), (T *)(dsm + 3 * CH * rowb)};
    const int bq = t / Bs, lim = bq - L;
    tc::grid_dep_wait();  // sel (route), q and the newest key and value (projection)
    tc::grid_dep_launch();
    if (threadIdx.x == 0) {
        int nr = 0;
        for (int r = 0; r < R; ++r) {
            const int j = sel[bh * R + r];
            if (j >= 0 && j <= lim) s_js[nr++] = j;
        }
        s_nr = nr;
    }
    __syncthreads();
    const int nr = s_nr;
    const int lo = max(0, bq - L + 1) * Bs;
    const int nkeys = nr * Bs + (t - lo + 1);
    const int share = (nkeys + kDecSplit - 1) / kDecSplit;
    const int k_beg = min(nkeys, z * share), k_end = min(nkeys, k_beg + share);
    auto key_of = [&](int idx) { return idx < nr * Bs ? s_js[idx / Bs] * Bs + idx % Bs : lo + (idx - nr * Bs); };
    auto stage = [&](int buf, int c0) {
        const int n = min(CH, k_end - c0), chunks = rowb / 16;
        for (int i = threadIdx.x; i < n * chunks; i += blockDim.x) {
            const int k = i / chunks, c = i % chunks;
            const size_t row = bh * S + key_of(c0 + k);
            tc::cp_async16((uint8_t *)bufK[buf] + k * rowb + 16 * c, (const uint8_t *)(Kc + row * d) + 16 * c, true);
            tc::cp_async16((uint8_t *)bufV[buf] + k * rowb + 16 * c, (const uint8_t *)(Vc + row * d) + 16 * c, true);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    float qv[kPer];
    for (int e = 0; e < per; ++e) qv[e] = to_f(q[bh * d + lane * per + e]);
    float m = -INFINITY, l = 0.f, acc[kPer];
    for (int e = 0; e < per; ++e) acc[e] = 0.f;
    if (k_beg < k_end) stage(0, k_beg);
    for (int c0 = k_beg, cb = 0; c0 < k_end; c0 += CH, cb ^= 1) {
        if (c0 + CH < k_end) {
            stage(cb ^ 1, c0 + CH);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const int n = min(CH, k_end - c0);
        for (int k = warp; k < n; k += NW) {
            const T *kr = bufK[cb] + k * d + lane * per, *vr = bufV[cb] + k * d + lane * per;
            float part = 0.f;
            for (int e = 0; e < per; ++e) part = fmaf(qv[e], to_f(kr[e]), part);
            const float sc = warp_sum(part) * scale;
            const float mn = fmaxf(m, sc);
            const float corr = expf(m - mn), p = expf(sc - mn);
            l = l * corr + p;
            for (int e = 0; e < per; ++e) acc[e] = fmaf(p, to_f(vr[e]), acc[e] * corr);
            m = mn;
        }
        __syncthreads();
    }
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
    }
    for (int e = 0; e < per; ++e) s_acc[warp][lane * per + e] = acc[e];
    __syncthreads();
    if (warp == 0) {  // this CTA's share
        float mm = -INFINITY;
        for (int w = 0; w < NW; ++w) mm = fmaxf(mm, s_m[w]);
        float den = 0.f, o[kPer];
        for (int e = 0; e < per; ++e) o[e] = 0.f;
        if (mm != -INFINITY)
            for (int w = 0; w < NW; ++w) {
                if (s_m[w] == -INFINITY) continue;  // a warp without keys
                const float f = expf(s_m[w] - mm);
                den += s_l[w] * f;
                for (int e = 0; e < per; ++e) o[e] += s_acc[w][lane * per + e] * f;
            }
        for (int e = 0; e < per; ++e) s_part[lane * per + e] = o[e];
        if (lane == 0) {
            s_part[d] = mm;
            s_part[d + 1] = den;
        }
    }
    cluster.sync();  // every share is in its CTA's shared memory
    if (z == 0 && warp == 0) {
        float mm = -INFINITY;
        for (int r = 0; r < kDecSplit; ++r) mm = fmaxf(mm, cluster.map_shared_rank(s_part, r)[d]);
        float den = 0.f, o[kPer];
        for (int e = 0; e < per; ++e) o[e] = 0.f;
        for (int r = 0; r < kDecSplit; ++r) {
            const float *pr = cluster.map_shared_rank(s_part, r);
            if (pr[d] == -INFINITY) continue;  // a share without keys
            const float f = expf(pr[d] - mm);
            den += pr[d + 1] * f;
            for (int e = 0; e < per; ++e) o[e] += pr[lane * per + e] * f;
        }
        for (int e = 0; e < per; ++e) O[(size_t)b * H * d + (size_t)h * d + lane * per + e] = from_f<T>(o[e] / den);
    }
    cluster.sync();  // the shares stay readable until CTA 0 has merged them
}

// delta_t [B, W] = o [B, H d] Wo^T (Wo [W, H d]); one warp per output column
template <typename T>
__global__ void __launch_bounds__(256) k_dec_out(const T *__restrict__ o, const T *__restrict__ Wo,
                                                 T *__restrict__ delta, int B, int W, int N) {
    const int lane = threadIdx.x & 31;
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (w >= W) return;
    const T *wr = Wo + (size_t)w * N;
    for (int off = lane * 64; off < N * (int)sizeof(T); off += 32 * 64) tc::prefetch_l2((const char *)wr + off);
    tc::grid_dep_wait();  // o (attention)
    tc::grid_dep_launch();
    for (int b = 0; b < B; ++b) {
        const T *ob = o + (size_t)b * N;
        const float a = warp_sum(row_dot_part(ob, wr, N, lane));
        if (lane == 0) delta[(size_t)b * W + w] = from_f<T>(a);
    }
}

// The kernels of a decode step are launched with programmatic dependent launch: each one's blocks may start while
// the kernel before it in the stream runs, and wait (grid_dep_wait) before they touch anything that kernel writes
// or reads; the launch gaps between the step's small kernels overlap.  cluster > 1 adds a cluster dimension.
template <typename... KArgs, typename... Args>
cudaError_t dec_launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                       Args... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[2];
    int na = 0;
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cluster > 1) {
        at[na].id = cudaLaunchAttributeClusterDimension;
        at[na].val.clusterDim.x = cluster;
        at[na].val.clusterDim.y = 1;
        at[na].val.clusterDim.z = 1;
        ++na;
    }
    lc.attrs = at;
    lc.numAttrs = na;
    return cudaLaunchKernelEx(&lc, kern, (KArgs)args...);
}

int dec_check(const mono_plan_t *plan, const void *cache) {
    if (!plan) return MONO_ERR_NULL;
    if (!cache) return MONO_ERR_WORKSPACE;
    if (((uintptr_t)cache & 255) != 0) return MONO_ERR_ALIGN;
    if (plan->p.A > kDecMaxA) return MONO_ERR_UNSUPPORTED;
    if (plan->p.cfg.flags & MONO_FLAG_REDIRECT) return MONO_ERR_UNSUPPORTED;  // the cache lists append in drop mode
    return MONO_OK;
}

int dec_status(cudaError_t e) { return e == cudaSuccess ? MONO_OK : MONO_ERR_CUDA; }

bool dec_empty(const Plan &p) { return p.cfg.B == 0 || p.cfg.S == 0; }

// the row vectors are read in 16-byte chunks
int dec_ptrs16(std::initializer_list<const void *> ptrs) {
    for (const void *q : ptrs) {
        if (!q) return MONO_ERR_NULL;
        if ((uintptr_t)q & 15) return MONO_ERR_ALIGN;
    }
    return MONO_OK;
}

}  // namespace
}  // namespace mono

using namespace mono;

extern "C" {

int mono_decode_cache_bytes(const mono_plan_t *plan, size_t *bytes) {
    if (!plan || !bytes) return MONO_ERR_NULL;
    if (plan->p.A > kDecMaxA) return MONO_ERR_UNSUPPORTED;
    if (plan->p.cfg.flags & MONO_FLAG_REDIRECT) return MONO_ERR_UNSUPPORTED;
    *bytes = dec_layout(plan->p).total;
    return MONO_OK;
}

int mono_decode_cache_region(const mono_plan_t *plan, int region, size_t *offset, size_t *bytes) {
    if (!plan || !offset || !bytes) return MONO_ERR_NULL;
    if (region < 0 || region >= MONO_DEC_NREGIONS) return MONO_ERR_INVALID;
    const DecLayout L = dec_layout(plan->p);
    *offset = L.off[region];
    *bytes = L.bytes[region];
    return MONO_OK;
}

int mono_decode_prefill(const mono_plan_t *plan, int t0, const float *codebooks, void *cache, void *stream) {
    int st = dec_check(plan, cache);
    if (st) return st;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (t0 < 0 || t0 > c.S) return MONO_ERR_INVALID;
    if (dec_empty(p)) return MONO_OK;
    if (!codebooks) return MONO_ERR_NULL;
    const DecLayout L = dec_layout(p);
    const DecPtrs P = dec_ptrs(L, cache);
    cudaStream_t s = (cudaStream_t)stream;
    const int nb0 = t0 / c.Bs;
    if (nb0 > 0) {
        dim3 g(nb0, c.H, c.B);
        if (c.dtype == MONO_BF16)
            k_dec_prefill_summaries<__nv_bfloat16><<<g, 32, 0, s>>>((const __nv_bfloat16 *)P.K, codebooks, P, c.S, c.Bs,
                                                                   c.d, c.M, c.C, c.H, p.nb);
        else
            k_dec_prefill_summaries<float><<<g, 32, 0, s>>>((const float *)P.K, codebooks, P, c.S, c.Bs, c.d, c.M, c.C,
                                                            c.H, p.nb);
        count_launches(1);
    }
    k_dec_prefill_lists<<<dim3(c.H, c.B), 32, 0, s>>>(P, nb0, c.H, p.nb, p.A, c.cap);
    count_launches(1);
    return dec_status(cudaGetLastError());
}

int mono_decode_project(const mono_plan_t *plan, int t, const void *x_t, const void *Wq, const void *Wk,
                        const void *Wv, void *cache, void *stream) {
    int st = dec_check(plan, cache);
    if (st) return st;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (t < 0 || t >= c.S) return MONO_ERR_INVALID;
    if (dec_empty(p)) return MONO_OK;
    if ((st = dec_ptrs16({x_t, Wq, Wk, Wv}))) return st;
    const DecPtrs P = dec_ptrs(dec_layout(p), cache);
    const int warps = 3 * c.H * c.d / 2;
    const int grid = (warps + 7) / 8;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (c.dtype == MONO_BF16)
        e = dec_launch(k_dec_project<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1, (const __nv_bfloat16 *)x_t,
                       (const __nv_bfloat16 *)Wq, (const __nv_bfloat16 *)Wk, (const __nv_bfloat16 *)Wv,
                       (__nv_bfloat16 *)P.Q, (__nv_bfloat16 *)P.K, (__nv_bfloat16 *)P.V, t, c.B, c.W, c.H, c.d, c.S,
                       c.rope_theta);
    else
        e = dec_launch(k_dec_project<float>, dim3(grid), dim3(256), 0, s, 1, (const float *)x_t, (const float *)Wq,
                       (const float *)Wk, (const float *)Wv, (float *)P.Q, (float *)P.K, (float *)P.V, t, c.B, c.W,
                       c.H, c.d, c.S, c.rope_theta);
    count_launches(1);
    return dec_status(e != cudaSuccess ? e : cudaGetLastError());
}

int mono_decode_route(const mono_plan_t *plan, int t, const float *codebooks, const int32_t *forced_t, void *cache,
                      void *stream) {
    int st = dec_check(plan, cache);
    if (st) return st;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (t < 0 || t >= c.S) return MONO_ERR_INVALID;
    if (dec_empty(p)) return MONO_OK;
    if (!codebooks) return MONO_ERR_NULL;
    if (forced_t && ((uintptr_t)forced_t & 3)) return MONO_ERR_ALIGN;
    const DecPtrs P = dec_ptrs(dec_layout(p), cache);
    cudaStream_t s = (cudaStream_t)stream;
    const dim3 g(c.H, c.B);
    const bool bf = c.dtype == MONO_BF16;
    cudaError_t e;
    if (t % c.Bs == c.Bs - 1) {  // position t completes block t / Bs
        if (bf)
            e = dec_launch(k_dec_block<__nv_bfloat16>, g, dim3(32), 0, s, 1, (const __nv_bfloat16 *)P.K, codebooks, P,
                           t, c.S, c.Bs, c.d, c.M, c.C, c.H, p.nb, p.A, c.cap);
        else
            e = dec_launch(k_dec_block<float>, g, dim3(32), 0, s, 1, (const float *)P.K, codebooks, P, t, c.S, c.Bs,
                           c.d, c.M, c.C, c.H, p.nb, p.A, c.cap);
        count_launches(1);
        if (e != cudaSuccess) return dec_status(e);
    }
    if (c.R > 0) {
        const size_t sm = (size_t)c.M * c.C * (c.d / c.M + 1) * 4;
        static_assert(kMaxT <= 32, "per-lane address lists of at most 32 entries");
        auto route = [&](auto kern, const auto *q) -> cudaError_t {
            cudaError_t err;
            if (sm > 48 * 1024 &&
                (err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
                return err;
            return dec_launch(kern, g, dim3(32), sm, s, 1, q, codebooks, forced_t, P, t, c.Bs, c.L, c.R, c.E, c.M,
                              c.C, c.T, c.cap, c.H, c.d, p.nb, p.A);
        };
#define MONO_DEC_ROUTE(TT)                                                                                       \
    (c.T <= 4 ? route(k_dec_route<TT, 4>, (const TT *)P.Q)                                                       \
              : c.T <= 8 ? route(k_dec_route<TT, 8>, (const TT *)P.Q)                                            \
                         : c.T <= 16 ? route(k_dec_route<TT, 16>, (const TT *)P.Q)                               \
                                     : route(k_dec_route<TT, 32>, (const TT *)P.Q))
        e = bf ? MONO_DEC_ROUTE(__nv_bfloat16) : MONO_DEC_ROUTE(float);
#undef MONO_DEC_ROUTE
        count_launches(1);
        if (e != cudaSuccess) return dec_status(e);
    }
    return dec_status(cudaGetLastError());
}

int mono_decode_attend(const mono_plan_t *plan, int t, void *cache, void *stream) {
    int st = dec_check(plan, cache);
    if (st) return st;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (t < 0 || t >= c.S) return MONO_ERR_INVALID;
    if (dec_empty(p)) return MONO_OK;
    const DecPtrs P = dec_ptrs(dec_layout(p), cache);
    const float scale = (float)(1.0 / sqrt((double)c.d));
    const dim3 g(c.H, c.B);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (c.dtype == MONO_BF16) {
        // a CTA's share of at most R + L blocks of keys, in one chunk where it fits
        const int share = ((c.R + c.L) * c.Bs + kDecSplit - 1) / kDecSplit;
        const int ch = std::min(dec_chunk<__nv_bfloat16>(c.d), share);
        const size_t smc = (size_t)4 * ch * c.d * 2;
        if (smc > 48 * 1024 && (e = cudaFuncSetAttribute(k_dec_attend_cl<__nv_bfloat16>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smc)))
            return dec_status(e);
        if ((e = dec_launch(k_dec_attend_cl<__nv_bfloat16>, dim3(c.H * kDecSplit, c.B), dim3(256), smc, s, kDecSplit,
                            (const __nv_bfloat16 *)P.Q, (const __nv_bfloat16 *)P.K, (const __nv_bfloat16 *)P.V,
                            (const int32_t *)P.sel, (__nv_bfloat16 *)P.O, t, c.S, c.Bs, c.L, c.R, c.H, c.d, scale,
                            ch)))
            return dec_status(e);
    } else {
        const size_t sm = (size_t)4 * dec_chunk<float>(c.d) * c.d * 4;
        if ((e = cudaFuncSetAttribute(k_dec_attend<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)))
            return dec_status(e);
        if ((e = dec_launch(k_dec_attend<float>, g, dim3(256), sm, s, 1, (const float *)P.Q, (const float *)P.K,
                            (const float *)P.V, (const int32_t *)P.sel, (float *)P.O, t, c.S, c.Bs, c.L, c.R, c.H,
                            c.d, scale)))
            return dec_status(e);
    }
    count_launches(1);
    return dec_status(cudaGetLastError());
}

int mono_decode_step(const mono_plan_t *plan, int t, const void *x_t, const void *Wq, const void *Wk, const void *Wv,
                     const void *Wo, const float *codebooks, const int32_t *forced_t, void *delta_t, void *cache,
                     void *stream) {
    int st = dec_check(plan, cache);
    if (st) return st;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (t < 0 || t >= c.S) return MONO_ERR_INVALID;
    if (dec_empty(p)) return MONO_OK;
    if ((st = dec_ptrs16({x_t, Wq, Wk, Wv, Wo, delta_t}))) return st;
    if ((st = mono_decode_project(plan, t, x_t, Wq, Wk, Wv, cache, stream))) return st;
    if ((st = mono_decode_route(plan, t, codebooks, forced_t, cache, stream))) return st;
    if ((st = mono_decode_attend(plan, t, cache, stream))) return st;
    const DecPtrs P = dec_ptrs(dec_layout(p), cache);
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = (c.W + 7) / 8;
    cudaError_t e;
    if (c.dtype == MONO_BF16)
        e = dec_launch(k_dec_out<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, 1, (const __nv_bfloat16 *)P.O,
                       (const __nv_bfloat16 *)Wo, (__nv_bfloat16 *)delta_t, c.B, c.W, c.H * c.d);
    else
        e = dec_launch(k_dec_out<float>, dim3(grid), dim3(256), 0, s, 1, (const float *)P.O, (const float *)Wo,
                       (float *)delta_t, c.B, c.W, c.H * c.d);
    count_launches(1);
    return dec_status(e != cudaSuccess ? e : cudaGetLastError());
}

}  // extern "C"

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

namespace mono {

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
// (A4) posting lists in canonical form: ids sorted by (address, id), the
// address of each entry and its rank among the blocks of that address.  The
// lists keep the earliest `cap` blocks of each address (rank < cap); the
// others are dropped and counted.  Each block's slot is found by counting the
// blocks that sort before it, so the result is deterministic.
// grid (H, B), 1024 threads, dynamic smem nb ints.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_posting_build(const int32_t *__restrict__ addr, int32_t *__restrict__ ids,
                                                        int32_t *__restrict__ saddr, int32_t *__restrict__ rank,
                                                        int32_t *__restrict__ overflow, int nb, int cap, int H) {
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
                                                      unsigned long long *__restrict__ counters, int S, int H, int Bs,
                                                      int L, int R, int E, int M, int C, int Tp, int cap) {
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
            float acc = 0.0f;
#pragma unroll
            for (int i4 = 0; i4 < D / 4; ++i4) {
                float4 v = __ldg(kr + i4);
                acc = __fmaf_rn(q[4 * i4 + 0], v.x, acc);
                acc = __fmaf_rn(q[4 * i4 + 1], v.y, acc);
                acc = __fmaf_rn(q[4 * i4 + 2], v.z, acc);
                acc = __fmaf_rn(q[4 * i4 + 3], v.w, acc);
            }
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

cudaError_t launch_summaries(const Plan &p, const void *K, const float *cb, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    float *kbar = (float *)ws_ptr(p, ws, kRegKbar);
    int32_t *addr = (int32_t *)ws_ptr(p, ws, kRegAddr);
    unsigned long long *cnt = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    cudaError_t e = cudaMemsetAsync(cnt, 0, kCntN * 8, s);
    if (e != cudaSuccess) return e;
    dim3 g1(p.nb, c.H, c.B);
    if (c.dtype == MONO_BF16)
        k_summary_assign<__nv_bfloat16><<<g1, 128, 0, s>>>((const __nv_bfloat16 *)K, cb, kbar, addr, c.S, c.d, c.Bs,
                                                           c.M, c.C, c.H);
    else
        k_summary_assign<float><<<g1, 128, 0, s>>>((const float *)K, cb, kbar, addr, c.S, c.d, c.Bs, c.M, c.C, c.H);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_lists(const Plan &p, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    dim3 g2(c.H, c.B);
    k_posting_build<<<g2, 1024, p.nb * sizeof(int32_t), s>>>(
        (const int32_t *)ws_ptr(p, ws, kRegAddr), (int32_t *)ws_ptr(p, ws, kRegPostIds),
        (int32_t *)ws_ptr(p, ws, kRegPostAddr), (int32_t *)ws_ptr(p, ws, kRegPostRank),
        (int32_t *)ws_ptr(p, ws, kRegOverflow), p.nb, c.cap, c.H);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_queries(const Plan &p, const void *Q, const float *cb, const int32_t *forced, int32_t *sel,
                           void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    unsigned long long *cnt = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    cudaError_t e = cudaMemsetAsync(cnt, 0, 3 * 8, s);  // statistics; the error word is kept
    if (e != cudaSuccess) return e;
    if (c.R == 0) return cudaSuccess;  // nothing to select: sel has no entries
    const float *kbar = (const float *)ws_ptr(p, ws, kRegKbar);
    const int32_t *ids = (const int32_t *)ws_ptr(p, ws, kRegPostIds);
    const int32_t *saddr = (const int32_t *)ws_ptr(p, ws, kRegPostAddr);
    const size_t smem = (size_t)c.C * c.d * 4 + (size_t)p.nb * 8;
    dim3 g3((c.S + 127) / 128, c.H, c.B);
    const bool bf = c.dtype == MONO_BF16;
#define MONO_LAUNCH_PR(TT, DD)                                                                                     \
    do {                                                                                                           \
        auto kern = k_probe_rerank<TT, DD>;                                                                        \
        if (smem > 48 * 1024) {                                                                                    \
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                \
            if (e != cudaSuccess) return e;                                                                        \
        }                                                                                                          \
        kern<<<g3, 128, smem, s>>>((const TT *)Q, kbar, cb, ids, saddr, forced, sel, cnt, c.S, c.H, c.Bs, c.L,   \
                                   c.R, c.E, c.M, c.C, c.T, c.cap);                                                \
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

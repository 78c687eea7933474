// backward.cu -- gradients of the mixer for a fixed selection.
//
// The routing (summaries, addresses, posting lists, probe, rerank) is
// piecewise constant in its inputs and has no gradient, so the backward pass
// takes the selection as an input and differentiates the rest of the forward
// pass ("Monodratic Routes Sparse Attention with Learned Product Hashes", Key
// Points; the aitechinspire.com article, Snapshot): projection without bias,
// RoPE on q and k, exact softmax over the selected token set (the remote
// blocks of sel plus the local tokens [max(0, t/Bs - L + 1) * Bs, t]), output
// projection.  For one query t with probabilities P over its keys s:
//     D_t = dO_t . O_t,   dS_ts = P_ts (dO_t . v_s - D_t),
//     dQ_t = scale sum_s dS_ts k_s,   dK_s += scale dS_ts q_t,   dV_s += P_ts dO_t.
// Kernels (fp32 arithmetic, gradients in fp32):
//   k_bwd_prep   with the forward recompute's fp32 O and log-sum-exp: D per
//                row and dO head-major as two bf16 terms, for the tensor-core
//                kernels;
//   k_bwd_dq     d/16 lanes per query-head: log-sum-exp and D from recomputed
//                scores (the stored O is not needed) or from the recompute,
//                then dQ over the local keys and the remote blocks;
//   k_bwd_count / k_bwd_scan / k_bwd_fill: per (b, h) and block j, the
//                queries that selected j (lists in unspecified order);
//   k_bwd_dkdv   one CTA per (b, h) and tile of up to 64 keys of one block:
//                walks the block's local queries and its selecting queries,
//                accumulating dK and dV of its keys in registers;
//   (with bf16 storage, the forward recompute's statistics and Bs = 64 the
//   attention gradients run instead on the tensor cores: k_bwd_local_dq_tc,
//   k_bwd_local_dkdv_tc and k_bwd_remote_tc in attend_tc.cu, then
//   k_bwd_finish for the factor, the inverse rotation and the layout)
//   (dq, dk and dv leave these kernels either as [B,H,S,d] for the post-RoPE
//   q and k, or rotated back and token-major for the projection gradients)
//   k_gemm_any   the projection gradients of fp32 storage (generic strided SIMT
//                GEMM, split K with fp32 atomics where the output has few
//                tiles); with bf16 storage they run on the tensor cores
//                (k_gemm_grad_tc: bf16 operands -- the gradients before the
//                projections rounded to bf16 -- with fp32 accumulation).
#include <cuda_runtime.h>

#include <math.h>

#include <initializer_list>

#include "internal.cuh"
#include "mono.h"

namespace mono {
namespace {

struct BwdLayout {
    size_t lse, dsum, cnt, start, cursor, list, sortbuf, slab, dO, dQp, dKp, dVp, dOhi, dOlo, dQloc, dKloc, dVloc,
        dQpair, total;
    size_t slab_bytes;
};

BwdLayout bwd_layout(const Plan &p) {
    const mono_config &c = p.cfg;
    const size_t B = c.B, H = c.H, S = c.S, d = c.d, nb = p.nb, R = c.R > 0 ? c.R : 1;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    BwdLayout L{};
    L.lse = take(B * H * S * 4);
    L.dsum = take(B * H * S * 4);
    L.cnt = take(B * H * nb * 4);
    L.start = take(B * H * nb * 4);
    L.cursor = take(B * H * nb * 4);
    L.list = take(B * H * S * R * 4);
    L.sortbuf = take(2 * B * H * S * R * 4);  // a list segment too long for shared memory, padded to a power of two
    // split-K partial tiles of the weight gradients: four ranges of the three-output dWq, dWk, dWv product
    L.slab_bytes = 4 * 3 * (size_t)H * d * c.W * 4;
    L.slab = take(L.slab_bytes);
    L.dO = take(B * S * H * d * 4);
    L.dQp = take(B * S * H * d * 4);
    L.dKp = take(B * S * H * d * 4);
    L.dVp = take(B * S * H * d * 4);
    // the tensor-core path: dO as two bf16 terms, and dQ, dK, dV in fp32 (without the 1/sqrt(d) factor, before
    // the inverse rotation), all head-major [B*H, S, d]
    L.dOhi = take(B * H * S * d * 2);
    L.dOlo = take(B * H * S * d * 2);
    L.dQloc = take(B * H * S * d * 4);
    L.dKloc = take(B * H * S * d * 4);
    L.dVloc = take(B * H * S * d * 4);
    L.dQpair = take(B * H * S * R * d * 4);  // the remote blocks' dQ parts, one row per (query, slot)
    L.total = o;
    return L;
}

__device__ __forceinline__ float bwd_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ bool bwd_sel_valid(int j, int t, int Bs, int L) { return j >= 0 && j <= t / Bs - L; }

// ---------------------------------------------------------------------------
// dQ, log-sum-exp and D of every query-head: D/16 consecutive lanes per query
// (32/(D/16) queries of consecutive positions per warp), each lane holding 16
// dimensions of q, dO and the accumulators in registers; a query's partial dot
// products combine with xor shuffles.  Keys: the local ones [lo, t] first, then
// the Bs keys of each valid remote block of sel.  The warp walks the largest
// local count of its queries and every remote slot any of them holds; a key a
// lane does not own counts with probability 0.  Pass 1 (online softmax) gives
// the log-sum-exp and O in fp32, hence D = dO . O; pass 2 forms dS and dQ.
// grid ceil(B H S * D/16 / 256), 256 threads.
// ---------------------------------------------------------------------------
constexpr int kDqE = 16;

// Where the attention gradients go: [B,H,S,d] fp32 with respect to the
// post-RoPE q and k (mono_attend_backward), or with respect to the projection
// outputs before RoPE -- dq and dk rotated back by the forward's angle of their
// position (the transpose of its rotation, from its cos/sin tables), dv as is --
// token-major [B*S, H*d], in fp32 or as two bf16 terms hi = bf16(v),
// lo = bf16(v - hi) at out and out + B*S*H*d (their sum carries 16 significant
// bits) for the tensor-core GEMMs.
enum GradMode { kOutHeads = 0, kOutTokensF32 = 1, kOutTokensSplit = 2 };

struct GradOut {
    void *q, *k, *v;
    const float2 *rope_hi, *rope_lo;  // token modes: the forward's tables (positions t / 64 and t % 64)
    int mode;
};

__device__ __forceinline__ uint32_t bf16_pair(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *(uint32_t *)&h;
}

// the 16 gradient values v of dimensions e0 .. e0+15 of (b, h, position t)
template <int DD>
__device__ __forceinline__ void store_grad16(const GradOut &go, void *out, bool rotate, float *v, int b, int h, int t,
                                             int e0, int B, int H, int S) {
    if (go.mode == kOutHeads) {
        float4 *dst = (float4 *)((float *)out + (((size_t)b * H + h) * S + t) * DD + e0);
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        return;
    }
    if (rotate) {
        const float2 *hi = go.rope_hi + (size_t)(t / kRopeLo) * (DD / 2) + e0 / 2;
        const float2 *lo = go.rope_lo + (size_t)(e0 / 2) * kRopeLo + t % kRopeLo;  // frequency-major
#pragma unroll
        for (int pr = 0; pr < 8; ++pr) {
            const float2 a = __ldg(hi + pr), bb = __ldg(lo + pr * kRopeLo);
            const float c = a.x * bb.x - a.y * bb.y, sn = a.y * bb.x + a.x * bb.y;
            const float x0 = v[2 * pr], x1 = v[2 * pr + 1];
            v[2 * pr] = x0 * c + x1 * sn;
            v[2 * pr + 1] = -x0 * sn + x1 * c;
        }
    }
    const size_t dst = (((size_t)b * S + t) * H + h) * DD + e0;
    if (go.mode == kOutTokensF32) {
        float4 *o4 = (float4 *)((float *)out + dst);
#pragma unroll
        for (int c = 0; c < 4; ++c) o4[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        return;
    }
    const size_t n = (size_t)B * S * H * DD;
    uint32_t hw[8], lw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float h0 = __bfloat162float(__float2bfloat16_rn(v[2 * i]));
        const float h1 = __bfloat162float(__float2bfloat16_rn(v[2 * i + 1]));
        hw[i] = bf16_pair(h0, h1);
        lw[i] = bf16_pair(v[2 * i] - h0, v[2 * i + 1] - h1);
    }
    uint4 *oh = (uint4 *)((__nv_bfloat16 *)out + dst), *ol = (uint4 *)((__nv_bfloat16 *)out + n + dst);
    oh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    oh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    ol[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    ol[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
}

template <typename T> __device__ __forceinline__ void load16(const T *p, float *v);
template <> __device__ __forceinline__ void load16<float>(const float *p, float *v) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float4 f = __ldg((const float4 *)p + c);
        v[4 * c] = f.x; v[4 * c + 1] = f.y; v[4 * c + 2] = f.z; v[4 * c + 3] = f.w;
    }
}
template <> __device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16 *p, float *v) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const uint4 r = __ldg((const uint4 *)p + c);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[8 * c + 2 * i] = __uint_as_float(w[i] << 16);
            v[8 * c + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
}

template <int TPQ>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = 1; o < TPQ; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// dO (token-major fp32) as two bf16 terms hi = bf16(v), lo = bf16(v - hi), head-major for the tensor-core local
// dQ, and D = dO . O of each row from the forward's fp32 O.  One warp per (b, t, h) row; grid covers B*S*H rows.
template <int DD>
__global__ void __launch_bounds__(256) k_bwd_prep(const float *__restrict__ dO, const float *__restrict__ o32,
                                                  __nv_bfloat16 *__restrict__ dohi, __nv_bfloat16 *__restrict__ dolo,
                                                  float *__restrict__ dsum, int B, int H, int S) {
    constexpr int PER = DD / 32;
    const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= (long long)B * S * H) return;
    const int h = (int)(w % H);
    const long long bt = w / H;
    const int t = (int)(bt % S), b = (int)(bt / S);
    const size_t hm = (((size_t)b * H + h) * S + t) * DD;  // head-major row
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int i = lane + 32 * e;
        const float v = dO[w * DD + i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        dohi[hm + i] = hi;
        dolo[hm + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
        part = fmaf(v, o32[w * DD + i], part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) dsum[((size_t)b * H + h) * S + t] = part;
}

// The tensor-core path's last step: dQ (the local part plus the remote blocks' parts of the query's valid
// slots, in slot order) and dK (times 1/sqrt(d)) and dV from their head-major fp32 sums to the operands of the
// projection gradients (store_grad16: rotated back, token-major).  One thread per 16 dimensions of a (b, h, t)
// row.
template <int DD>
__global__ void __launch_bounds__(256) k_bwd_finish(const float *__restrict__ dq, const float *__restrict__ dk,
                                                    const float *__restrict__ dv, const float *__restrict__ dq_pair,
                                                    const int32_t *__restrict__ sel, const GradOut go, int B, int H,
                                                    int S, int Bs, int L, int R, float scale) {
    constexpr int TPR = DD / 16;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long long)B * H * S * TPR) return;
    const long long w = gid / TPR;
    const int e0 = (int)(gid % TPR) * 16;
    const int t = (int)(w % S);
    const long long bh = w / S;
    const int b = (int)(bh / H), h = (int)(bh % H);
    float q[16], k[16], v[16];
    load16<float>(dq + w * DD + e0, q);
    load16<float>(dk + w * DD + e0, k);
    load16<float>(dv + w * DD + e0, v);
    // the remote blocks' parts in slot order
    for (int r = 0; r < R; ++r) {
        if (!bwd_sel_valid(sel[w * R + r], t, Bs, L)) continue;
        float pq[16];
        load16<float>(dq_pair + (w * R + r) * DD + e0, pq);
#pragma unroll
        for (int e = 0; e < 16; ++e) q[e] += pq[e];
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        q[e] *= scale;
        k[e] *= scale;
    }
    store_grad16<DD>(go, go.q, true, q, b, h, t, e0, B, H, S);
    store_grad16<DD>(go, go.k, true, k, b, h, t, e0, B, H, S);
    store_grad16<DD>(go, go.v, false, v, b, h, t, e0, B, H, S);
}

template <typename T, int DD>
__global__ void __launch_bounds__(256) k_bwd_dq(const T *__restrict__ Q, const T *__restrict__ K,
                                                const T *__restrict__ V, const int32_t *__restrict__ sel,
                                                const float *__restrict__ dO, const GradOut go,
                                                float *__restrict__ lse_out, float *__restrict__ dsum_out,
                                                const float *__restrict__ o32, int B, int H, int S, int Bs, int L,
                                                int R, float scale) {
    constexpr int TPQ = DD / kDqE, E = kDqE, U = 2;
    const long long nq = (long long)B * H * S;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long w0 = gid / TPQ;
    const bool live = w0 < nq;
    const long long w = live ? w0 : nq - 1;  // lanes past the end shadow the last query and store nothing
    const int e0 = (int)(gid % TPQ) * E;
    const long long bh = w / S;
    const int t = (int)(w % S);
    const int b = (int)(bh / H), h = (int)(bh % H);
    const size_t base = (size_t)bh * S;
    float q[E], g[E];
    load16<T>(Q + w * DD + e0, q);
    load16<float>(dO + (((size_t)b * S + t) * H + h) * DD + e0, g);
    const int lo = max(0, t / Bs - L + 1) * Bs;
    const int nloc = t - lo + 1;
    int nloc_w = nloc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nloc_w = max(nloc_w, __shfl_xor_sync(0xffffffffu, nloc_w, o));

    // one sweep over the query's keys; f(k row, v row, valid) per group of U keys
    auto sweep = [&](auto &&f) {
        for (int i = 0; i < nloc_w; i += U) {
            const T *kr[U], *vr[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                ok[u] = i + u < nloc;
                const size_t row = (base + (ok[u] ? lo + i + u : t)) * DD + e0;
                kr[u] = K + row;
                vr[u] = V + row;
            }
            f(kr, vr, ok);
        }
        for (int r = 0; r < R; ++r) {
            const int j = sel[w * R + r];
            const bool has = bwd_sel_valid(j, t, Bs, L);
            if (!__any_sync(0xffffffffu, has)) continue;
            for (int i = 0; i < Bs; i += U) {
                const T *kr[U], *vr[U];
                bool ok[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    ok[u] = has && i + u < Bs;
                    const size_t row = (base + (ok[u] ? (size_t)j * Bs + i + u : (size_t)t)) * DD + e0;
                    kr[u] = K + row;
                    vr[u] = V + row;
                }
                f(kr, vr, ok);
            }
        }
    };

    // pass 1: log-sum-exp and O (the first group holds key lo of every query: m is finite after it); with the
    // forward's statistics (o32: O in fp32, lse_out: its log-sum-exp) only D = dO . O
    float lse, D;
    if (o32) {
        float o[E];
        load16<float>(o32 + (((size_t)b * S + t) * H + h) * DD + e0, o);
        float dpart = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) dpart = fmaf(g[e], o[e], dpart);
        D = group_sum<TPQ>(dpart);
        lse = lse_out[w];
    } else {
    float m = -INFINITY, l = 0.f, o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.f;
    sweep([&](const T *const *kr, const T *const *vr, const bool *ok) {
        float kk[U][E], sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) load16<T>(kr[u], kk[u]);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float part = 0.f, part2 = 0.f;
#pragma unroll
            for (int e = 0; e < E / 2; ++e) {
                part = fmaf(q[e], kk[u][e], part);
                part2 = fmaf(q[e + E / 2], kk[u][e + E / 2], part2);
            }
            sc[u] = group_sum<TPQ>(part + part2) * scale;
        }
        float mx = m;
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (ok[u]) mx = fmaxf(mx, sc[u]);
        const float corr = expf(m - mx);
        l *= corr;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] *= corr;
        m = mx;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float p = ok[u] ? expf(sc[u] - mx) : 0.f;
            float vv[E];
            load16<T>(vr[u], vv);
            l += p;
#pragma unroll
            for (int e = 0; e < E; ++e) o[e] = fmaf(p, vv[e], o[e]);
        }
    });
    lse = m + logf(l);
    float dpart = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) dpart = fmaf(g[e], o[e] / l, dpart);
    D = group_sum<TPQ>(dpart);
    }

    // pass 2: dS and dQ
    float dq[E];
#pragma unroll
    for (int e = 0; e < E; ++e) dq[e] = 0.f;
    sweep([&](const T *const *kr, const T *const *vr, const bool *ok) {
        float kk[U][E], sp[U], dp[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float vv[E];
            load16<T>(kr[u], kk[u]);
            load16<T>(vr[u], vv);
            float a = 0.f, c = 0.f, a2 = 0.f, c2 = 0.f;
#pragma unroll
            for (int e = 0; e < E / 2; ++e) {
                a = fmaf(q[e], kk[u][e], a);
                c = fmaf(g[e], vv[e], c);
                a2 = fmaf(q[e + E / 2], kk[u][e + E / 2], a2);
                c2 = fmaf(g[e + E / 2], vv[e + E / 2], c2);
            }
            sp[u] = a + a2;
            dp[u] = c + c2;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            sp[u] = group_sum<TPQ>(sp[u]);
            dp[u] = group_sum<TPQ>(dp[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float ds = ok[u] ? expf(sp[u] * scale - lse) * (dp[u] - D) : 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) dq[e] = fmaf(ds, kk[u][e], dq[e]);
        }
    });
    if (live) {
#pragma unroll
        for (int e = 0; e < E; ++e) dq[e] *= scale;
        store_grad16<DD>(go, go.q, true, dq, b, h, t, e0, B, H, S);
        if (e0 == 0) {
            if (!o32) lse_out[w] = lse;
            dsum_out[w] = D;
        }
    }
}

// ---------------------------------------------------------------------------
// per (b, h) and block j, the queries that selected j: count, scan, fill
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bwd_count(const int32_t *__restrict__ sel, int32_t *__restrict__ cnt,
                                                   long long n, int S, int R, int nb, int Bs, int L) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const long long w = i / R;
    const int t = (int)(w % S);
    const long long bh = w / S;
    const int j = sel[i];
    if (bwd_sel_valid(j, t, Bs, L)) atomicAdd(&cnt[bh * nb + j], 1);
}

// exclusive scan of the counts of one (b, h); grid B*H, 1024 threads
__global__ void __launch_bounds__(1024) k_bwd_scan(const int32_t *__restrict__ cnt, int32_t *__restrict__ start,
                                                   int32_t *__restrict__ cursor, int nb) {
    __shared__ int s_part[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bh = blockIdx.x;
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    const int j0 = tid * per;
    int run = 0;
    for (int j = j0; j < min(nb, j0 + per); ++j) run += cnt[bh * nb + j];
    int x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_part[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int v = lane < (int)(blockDim.x >> 5) ? s_part[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        s_part[lane] = v;
    }
    __syncthreads();
    int off = (warp ? s_part[warp - 1] : 0) + x - run;
    for (int j = j0; j < min(nb, j0 + per); ++j) {
        start[bh * nb + j] = off;
        cursor[bh * nb + j] = off;
        off += cnt[bh * nb + j];
    }
}

__global__ void __launch_bounds__(256) k_bwd_fill(const int32_t *__restrict__ sel, int32_t *__restrict__ cursor,
                                                  int32_t *__restrict__ list, long long n, int S, int R, int nb,
                                                  int Bs, int L) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const long long w = i / R;
    const int t = (int)(w % S);
    const long long bh = w / S;
    const int j = sel[i];
    if (!bwd_sel_valid(j, t, Bs, L)) return;
    const int pos = atomicAdd(&cursor[bh * nb + j], 1);
    list[bh * S * R + pos] = (int)(i - bh * S * R);  // the pair t * R + r; k_bwd_sort orders each block's list
}

// Each block's list of pairs (from k_bwd_fill, in atomic order) sorted ascending, so that every sum over a
// block's queries runs in one order on every call.  One CTA per (b, h, block): a bitonic network over the
// list padded with INT_MAX to a power of two P, in shared memory when P <= 8192, else in sortbuf (the
// segment's own 2 n ints at twice its list offset).  grid B*H*nb, 256 threads.
__global__ void __launch_bounds__(256) k_bwd_sort(int32_t *__restrict__ list, int32_t *__restrict__ sortbuf,
                                                  const int32_t *__restrict__ cnt, const int32_t *__restrict__ start,
                                                  int S, int R, int nb) {
    __shared__ int32_t sh[8192];
    const int seg = blockIdx.x, tid = threadIdx.x;
    const int n = cnt[seg];
    if (n <= 1) return;
    const size_t base = (size_t)(seg / nb) * S * R;
    int32_t *a = list + base + start[seg];
    int P = 1;
    while (P < n) P <<= 1;
    int32_t *w = P <= 8192 ? sh : sortbuf + 2 * base + 2 * (size_t)start[seg];
    for (int i = tid; i < P; i += blockDim.x) w[i] = i < n ? a[i] : 0x7fffffff;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += blockDim.x) {
                const int l = i ^ j;
                if (l > i) {
                    const int x = w[i], y = w[l];
                    if ((x > y) == ((i & k) == 0)) {
                        w[i] = y;
                        w[l] = x;
                    }
                }
            }
            __syncthreads();
        }
    for (int i = tid; i < n; i += blockDim.x) a[i] = w[i];
}

// ---------------------------------------------------------------------------
// dK and dV of a tile of up to 64 keys of block j of one (b, h): D/16 threads
// per key, each holding 16 dimensions of the key's K and V rows and of its dK
// and dV accumulators in registers; a key's threads are consecutive lanes and
// combine their partial dot products with xor shuffles.  Queries come in
// groups of 16 (q, dO, log-sum-exp and D staged in shared memory, read as
// broadcast float4; each 16-float segment of a row padded to 20 floats so
// that the segments of a key's lanes sit in distinct banks; the next group's
// rows are fetched into registers while the current one is computed,
// double-buffered): first the local ones (blocks
// j .. j+L-1; in block j itself only keys s <= t, applied as a zero
// probability so that every lane takes part in the shuffles), then those
// whose selection holds block j.
// grid (ceil(Bs/64) * nb, H, B), 64 * D/16 threads.
// ---------------------------------------------------------------------------
constexpr int kBwdKT = 64, kBwdQG = 16;

template <typename T, int DD>
__global__ void __launch_bounds__(kBwdKT * DD / 16, DD == 64 ? 2 : 1) k_bwd_dkdv(
    const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V, const float *__restrict__ dO,
    const float *__restrict__ lse, const float *__restrict__ dsum, const int32_t *__restrict__ cnt,
    const int32_t *__restrict__ start, const int32_t *__restrict__ list, const GradOut go, int B, int H, int S,
    int Bs, int L, int R, int nb, float scale) {
    constexpr int TPK = DD / 16, NT = kBwdKT * TPK, E = 16;
    constexpr int PER = kBwdQG * DD / NT;  // staged elements per thread and array (one dimension, PER queries)
    constexpr int SEG = 20, ROW = TPK * SEG;  // padded segment and row, in floats
    __shared__ __align__(16) float sq[2][kBwdQG][ROW];
    __shared__ __align__(16) float sg[2][kBwdQG][ROW];
    __shared__ float slse[2][kBwdQG], sD[2][kBwdQG];
    __shared__ int st[2][kBwdQG];
    const int tpb = (Bs + kBwdKT - 1) / kBwdKT;
    const int j = blockIdx.x / tpb, u = blockIdx.x % tpb;
    const int h = blockIdx.y, b = blockIdx.z;
    const size_t bh = (size_t)b * H + h;
    const int k0 = j * Bs + u * kBwdKT;
    const int nk = min(kBwdKT, Bs - u * kBwdKT);
    const int tid = threadIdx.x;
    const int ks = tid / TPK, part = tid % TPK, e0 = part * E;
    const bool live = ks < nk;
    const int key = k0 + ks;
    float kr[E], vr[E], dk[E], dv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        kr[e] = live ? to_f(K[(bh * S + key) * DD + e0 + e]) : 0.f;
        vr[e] = live ? to_f(V[(bh * S + key) * DD + e0 + e]) : 0.f;
        dk[e] = 0.f;
        dv[e] = 0.f;
    }
    const int t_loc0 = j * Bs, t_loc1 = min(S, (j + L) * Bs);  // local queries [t_loc0, t_loc1)
    const int nloc = t_loc1 - t_loc0;
    const int nrem = R > 0 ? cnt[bh * nb + j] : 0;
    const int rem0 = R > 0 ? start[bh * nb + j] : 0;
    const int nq = nloc + nrem;
    // thread tid stages dimension fe of queries fq0, fq0 + NT/DD, ... of a group (at padded column fc)
    const int fe = tid % DD, fq0 = tid / DD, fc = fe + (fe / E) * (SEG - E);
    float rq[PER], rg[PER], rl[PER], rd[PER];
    int rt[PER];
    auto fetch = [&](int g0) {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int n = g0 + fq0 + k * (NT / DD);
            const bool in = n < nq;
            const int t = !in ? 0 : n < nloc ? t_loc0 + n : list[bh * S * R + rem0 + (n - nloc)] / R;
            rt[k] = t;
            rq[k] = in ? to_f(Q[(bh * S + t) * DD + fe]) : 0.f;
            rg[k] = in ? dO[(((size_t)b * S + t) * H + h) * DD + fe] : 0.f;
            if (fe == 0) {
                rl[k] = in ? lse[bh * S + t] : 0.f;
                rd[k] = in ? dsum[bh * S + t] : 0.f;
            }
        }
    };
    auto stash = [&](int buf) {
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int qi = fq0 + k * (NT / DD);
            sq[buf][qi][fc] = rq[k];
            sg[buf][qi][fc] = rg[k];
            if (fe == 0) {
                st[buf][qi] = rt[k];
                slse[buf][qi] = rl[k];
                sD[buf][qi] = rd[k];
            }
        }
    };
    if (nq > 0) {
        fetch(0);
        stash(0);
    }
    __syncthreads();
    int buf = 0;
    for (int g0 = 0; g0 < nq; g0 += kBwdQG, buf ^= 1) {
        const int ng = min(kBwdQG, nq - g0);
        const bool more = g0 + kBwdQG < nq;
        if (more) fetch(g0 + kBwdQG);  // in flight while this group is computed
        for (int qi = 0; qi < ng; ++qi) {
            const float4 *q4 = (const float4 *)&sq[buf][qi][part * SEG];
            const float4 *g4 = (const float4 *)&sg[buf][qi][part * SEG];
            float qv[E], gv[E];
#pragma unroll
            for (int c = 0; c < E / 4; ++c) {
                const float4 a = q4[c], bb = g4[c];
                qv[4 * c] = a.x; qv[4 * c + 1] = a.y; qv[4 * c + 2] = a.z; qv[4 * c + 3] = a.w;
                gv[4 * c] = bb.x; gv[4 * c + 1] = bb.y; gv[4 * c + 2] = bb.z; gv[4 * c + 3] = bb.w;
            }
            float sp = 0.f, dp = 0.f, sp2 = 0.f, dp2 = 0.f;  // two chains each
#pragma unroll
            for (int e = 0; e < E / 2; ++e) {
                sp = fmaf(qv[e], kr[e], sp);
                dp = fmaf(gv[e], vr[e], dp);
                sp2 = fmaf(qv[e + E / 2], kr[e + E / 2], sp2);
                dp2 = fmaf(gv[e + E / 2], vr[e + E / 2], dp2);
            }
            sp += sp2;
            dp += dp2;
#pragma unroll
            for (int o = 1; o < TPK; o <<= 1) {
                sp += __shfl_xor_sync(0xffffffffu, sp, o);
                dp += __shfl_xor_sync(0xffffffffu, dp, o);
            }
            const bool masked = !live || (g0 + qi < nloc && key > st[buf][qi]);  // causal in the query's own block
            const float p = masked ? 0.f : expf(sp * scale - slse[buf][qi]);
            const float ds = p * (dp - sD[buf][qi]) * scale;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                dv[e] = fmaf(p, gv[e], dv[e]);
                dk[e] = fmaf(ds, qv[e], dk[e]);
            }
        }
        if (more) stash(buf ^ 1);  // every thread finished reading buf ^ 1 before the last barrier
        __syncthreads();
    }
    if (live) {
        store_grad16<DD>(go, go.k, true, dk, b, h, key, e0, B, H, S);
        store_grad16<DD>(go, go.v, false, dv, b, h, key, e0, B, H, S);
    }
}

// ---------------------------------------------------------------------------
// C[M,N] (fp32, row stride ldc) (+)= sum_k A(m,k) B(k,n), with
// A(m,k) = A[m*am + k*ak] and B(k,n) = B[k*bk + n*bn] of types TA, TB
// (fp32 accumulation).  128x128 tile per CTA, 8-deep k slices staged in shared
// memory, 8x8 outputs per thread; the tile loads walk the operand's
// unit-stride index across consecutive threads.  With split > 1 the CTA
// (blockIdx.z) takes one of `split` k ranges and adds its partial sums to C
// with fp32 atomics (C holds 0 or the sum to accumulate onto).
// grid (ceil(N/128), ceil(M/128), split), 256 threads.
// ---------------------------------------------------------------------------
template <typename TA, typename TB>
__global__ void __launch_bounds__(256) k_gemm_any(int M, int N, int Kd, const TA *__restrict__ A, long long am,
                                                  long long ak, const TB *__restrict__ Bm, long long bk, long long bn,
                                                  float *__restrict__ C, long long ldc, int kchunk, bool atomic,
                                                  long long zstride) {
    C += blockIdx.z * zstride;  // split k ranges into their own slabs
    __shared__ __align__(16) float sA[8][128 + 4];
    __shared__ __align__(16) float sB[8][128 + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
    const int kb = blockIdx.z * kchunk, ke = min(Kd, kb + kchunk);
    float acc[8][8] = {};
    for (int k0 = kb; k0 < ke; k0 += 8) {
        for (int i = tid; i < 128 * 8; i += 256) {
            int mm, kk;
            if (ak == 1) { mm = i / 8; kk = i % 8; }
            else { kk = i / 128; mm = i % 128; }
            const int m = m0 + mm, k = k0 + kk;
            sA[kk][mm] = (m < M && k < ke) ? to_f(A[(long long)m * am + (long long)k * ak]) : 0.f;
            int nn, kq;
            if (bn == 1) { kq = i / 128; nn = i % 128; }
            else { nn = i / 8; kq = i % 8; }
            const int n = n0 + nn, k2 = k0 + kq;
            sB[kq][nn] = (n < N && k2 < ke) ? to_f(Bm[(long long)k2 * bk + (long long)n * bn]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const float4 a0 = *(const float4 *)&sA[kk][ty * 8], a1 = *(const float4 *)&sA[kk][ty * 8 + 4];
            const float4 b0 = *(const float4 *)&sB[kk][tx * 8], b1 = *(const float4 *)&sB[kk][tx * 8 + 4];
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(a[r], bv[c], acc[r][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int m = m0 + ty * 8 + r;
        if (m >= M) continue;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int n = n0 + tx * 8 + c;
            if (n >= N) continue;
            float *dst = C + (long long)m * ldc + n;
            if (atomic) atomicAdd(dst, acc[r][c]);
            else *dst = acc[r][c];
        }
    }
}

// beta 0: C = A B; beta 1: C += A B.  Output tiles fewer than twice the SMs split K.
// C (+)= sum of the split slabs in ascending order (n4 float4s each)
__global__ void __launch_bounds__(256) k_slab_sum(const float4 *__restrict__ slab, float4 *__restrict__ C, long long n4,
                                                  int split, bool accumulate) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        float4 a = __ldg(slab + i);
        for (int p = 1; p < split; ++p) {
            const float4 b = __ldg(slab + (size_t)p * n4 + i);
            a = make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
        }
        if (accumulate) {
            const float4 o = C[i];
            a = make_float4(__fadd_rn(o.x, a.x), __fadd_rn(o.y, a.y), __fadd_rn(o.z, a.z), __fadd_rn(o.w, a.w));
        }
        C[i] = a;
    }
}

template <typename TA, typename TB>
cudaError_t gemm_any(int M, int N, int Kd, const TA *A, long long am, long long ak, const TB *Bm, long long bk,
                     long long bn, float *C, long long ldc, float beta, float *slab, size_t slab_bytes,
                     cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    const int tiles = ((N + 127) / 128) * ((M + 127) / 128);
    int split = 1;
    while (split < 32 && tiles * split < 2 * 148 && Kd / (split * 2) >= 256) split *= 2;
    // the k ranges' partial products go to slabs summed in range order (the same bits on every run)
    const size_t out_bytes = (size_t)M * N * sizeof(float);
    while (split > 1 && (!slab || ldc != N || split * out_bytes > slab_bytes)) split /= 2;
    const int kchunk = ((Kd + split - 1) / split + 7) / 8 * 8;
    dim3 g((N + 127) / 128, (M + 127) / 128, split);
    if (split == 1) {
        // one CTA per output element: C = product, or C += product with beta = 1
        k_gemm_any<TA, TB><<<g, 256, 0, s>>>(M, N, Kd, A, am, ak, Bm, bk, bn, C, ldc, kchunk, beta != 0.f, 0ll);
        count_launches(1);
        return cudaGetLastError();
    }
    k_gemm_any<TA, TB><<<g, 256, 0, s>>>(M, N, Kd, A, am, ak, Bm, bk, bn, slab, N, kchunk, false,
                                         (long long)M * N);
    const long long n4 = (long long)M * N / 4;
    k_slab_sum<<<(unsigned)std::min<long long>((n4 + 255) / 256, 8 * 148), 256, 0, s>>>(
        (const float4 *)slab, (float4 *)C, n4, split, beta != 0.f);
    count_launches(2);
    return cudaGetLastError();
}

// o32: the forward's O in fp32 (token-major) with its log-sum-exp already in the lse region, or null
template <typename T>
cudaError_t attend_backward(const Plan &p, const T *Q, const T *K, const T *V, const int32_t *sel, const float *dO,
                            const GradOut &go, char *bws, cudaStream_t s, const float *o32 = nullptr,
                            unsigned long long *counters = nullptr) {
    const mono_config &c = p.cfg;
    const BwdLayout L = bwd_layout(p);
    float *lse = (float *)(bws + L.lse), *dsum = (float *)(bws + L.dsum);
    int32_t *cnt = (int32_t *)(bws + L.cnt), *start = (int32_t *)(bws + L.start);
    int32_t *cursor = (int32_t *)(bws + L.cursor), *list = (int32_t *)(bws + L.list);
    const float scale = (float)(1.0 / sqrt((double)c.d));
    const long long nq = (long long)c.B * c.H * c.S;
    cudaError_t e;
    const int tpq = c.d / kDqE;
    const unsigned gq = (unsigned)((nq * tpq + 255) / 256);
    auto build_lists = [&]() -> cudaError_t {
        if (c.R == 0) return cudaSuccess;
        const long long n = nq * c.R;
        cudaError_t e2;
        if ((e2 = cudaMemsetAsync(cnt, 0, (size_t)c.B * c.H * p.nb * 4, s)) != cudaSuccess) return e2;
        k_bwd_count<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sel, cnt, n, c.S, c.R, p.nb, c.Bs, c.L);
        k_bwd_scan<<<c.B * c.H, 1024, 0, s>>>(cnt, start, cursor, p.nb);
        k_bwd_fill<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sel, cursor, list, n, c.S, c.R, p.nb, c.Bs, c.L);
        k_bwd_sort<<<(unsigned)(c.B * c.H * p.nb), 256, 0, s>>>(list, (int32_t *)(bws + L.sortbuf), cnt, start, c.S,
                                                               c.R, p.nb);
        count_launches(4);
        return cudaSuccess;
    };
    // With the forward's statistics and a shape the kernels take, every attention gradient on the tensor cores:
    // the local keys query-major (dQ) and key-major (dK, dV), then the remote blocks block by block.
    if constexpr (sizeof(T) == 2) {
        if (o32 && counters && bwd_local_dq_tc_supported(c)) {
            __nv_bfloat16 *dohi = (__nv_bfloat16 *)(bws + L.dOhi), *dolo = (__nv_bfloat16 *)(bws + L.dOlo);
            float *dq_loc = (float *)(bws + L.dQloc), *dk_loc = (float *)(bws + L.dKloc);
            float *dv_loc = (float *)(bws + L.dVloc);
            const unsigned gp = (unsigned)((nq + 7) / 8);
            if (c.d == 64)
                k_bwd_prep<64><<<gp, 256, 0, s>>>(dO, o32, dohi, dolo, dsum, c.B, c.H, c.S);
            else
                k_bwd_prep<128><<<gp, 256, 0, s>>>(dO, o32, dohi, dolo, dsum, c.B, c.H, c.S);
            count_launches(1);
            if ((e = launch_bwd_local_dq_tc(p, Q, K, V, dohi, dolo, lse, dsum, dq_loc, counters, s)) != cudaSuccess)
                return e;
            if ((e = launch_bwd_local_dkdv_tc(p, Q, K, V, dohi, dolo, lse, dsum, dk_loc, dv_loc, counters, s)) !=
                cudaSuccess)
                return e;
            if ((e = build_lists()) != cudaSuccess) return e;
            float *dq_pair = (float *)(bws + L.dQpair);
            if (c.R > 0 && (e = launch_bwd_remote_tc(p, Q, K, V, dohi, dolo, lse, dsum, cnt, start, list, dq_pair,
                                                     dk_loc, dv_loc, counters, s)) != cudaSuccess)
                return e;
            const unsigned gf = (unsigned)((nq * (c.d / 16) + 255) / 256);
            if (c.d == 64)
                k_bwd_finish<64><<<gf, 256, 0, s>>>(dq_loc, dk_loc, dv_loc, dq_pair, sel, go, c.B, c.H, c.S, c.Bs,
                                                    c.L, c.R, scale);
            else
                k_bwd_finish<128><<<gf, 256, 0, s>>>(dq_loc, dk_loc, dv_loc, dq_pair, sel, go, c.B, c.H, c.S, c.Bs,
                                                     c.L, c.R, scale);
            count_launches(1);
            return cudaGetLastError();
        }
    }
    if (c.d == 64)
        k_bwd_dq<T, 64><<<gq, 256, 0, s>>>(Q, K, V, sel, dO, go, lse, dsum, o32, c.B, c.H, c.S, c.Bs, c.L, c.R,
                                           scale);
    else
        k_bwd_dq<T, 128><<<gq, 256, 0, s>>>(Q, K, V, sel, dO, go, lse, dsum, o32, c.B, c.H, c.S, c.Bs, c.L, c.R,
                                            scale);
    count_launches(1);
    if ((e = build_lists()) != cudaSuccess) return e;
    const int tpb = (c.Bs + kBwdKT - 1) / kBwdKT;
    const dim3 gk(tpb * p.nb, c.H, c.B);
    if (c.d == 64)
        k_bwd_dkdv<T, 64><<<gk, kBwdKT * 4, 0, s>>>(Q, K, V, dO, lse, dsum, cnt, start, list, go, c.B, c.H, c.S,
                                                     c.Bs, c.L, c.R, p.nb, scale);
    else
        k_bwd_dkdv<T, 128><<<gk, kBwdKT * 8, 0, s>>>(Q, K, V, dO, lse, dsum, cnt, start, list, go, c.B, c.H, c.S,
                                                      c.Bs, c.L, c.R, p.nb, scale);
    count_launches(1);
    return cudaGetLastError();
}

// The projection gradients on the tensor cores (bf16 storage): the operands are
// the stored bf16 activations and weights, the upstream gradient ddelta (all
// exact in bf16) and the fp32 gradients before the projections, dQp, dKp, dVp,
// each as its two-term bf16 split hi + lo (in its own workspace region), so the
// products are those of fp32 operands to 16 significant bits; accumulation and
// outputs fp32.
bool grads_tc_supported(const mono_config &c) {
    const int BS = c.B * c.S, Hd = c.H * c.d, W = c.W;
    return c.dtype == MONO_BF16 && gemm_grad_tc_supported(BS, Hd, W, false, true) &&
           gemm_grad_tc_supported(W, Hd, BS, true, true) && gemm_grad_tc_supported(Hd, W, BS, true, true) &&
           gemm_grad_tc_supported(BS, W, Hd, false, true);
}

template <typename T>
cudaError_t backward_t(const Plan &p, const T *x, const T *Wq, const T *Wk, const T *Wv, const T *Wo,
                       const int32_t *sel, const T *ddelta, float *dx, float *dWq, float *dWk, float *dWv, float *dWo,
                       const T *Q, const T *K, const T *V, const T *O, char *bws, void *ws, cudaStream_t s,
                       const float *o32 = nullptr) {
    const mono_config &c = p.cfg;
    const BwdLayout L = bwd_layout(p);
    unsigned long long *counters = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    float *dO = (float *)(bws + L.dO);
    float *slab = (float *)(bws + L.slab);
    const int BS = c.B * c.S, Hd = c.H * c.d, W = c.W;
    const bool tc = grads_tc_supported(c);
    // dQp, dKp, dVp: the attention gradients before RoPE, token-major, written by the attention kernels
    GradOut go{};
    go.q = bws + L.dQp;
    go.k = bws + L.dKp;
    go.v = bws + L.dVp;
    go.rope_hi = (const float2 *)ws_ptr(p, ws, kRegRope);  // built by the projection of the forward recompute
    go.rope_lo = go.rope_hi + (size_t)((c.S + kRopeLo - 1) / kRopeLo) * (c.d / 2);
    go.mode = tc ? kOutTokensSplit : kOutTokensF32;
    cudaError_t e;
    if (tc) {
        // delta = O Wo^T:  dO = ddelta Wo (Wo MN-major),  dWo = ddelta^T O (both MN-major)
        const void *a0[1] = {ddelta}, *b0[1] = {Wo}, *b1[1] = {O};
        float *c0[1] = {dO}, *c1[1] = {dWo};
        if ((e = gemm_grad_tc(BS, Hd, W, 1, 1, a0, false, b0, true, c0, false, slab, L.slab_bytes, counters, s)) !=
            cudaSuccess)
            return e;
        if ((e = gemm_grad_tc(W, Hd, BS, 1, 1, a0, true, b1, true, c1, false, slab, L.slab_bytes, counters, s)) !=
            cudaSuccess)
            return e;
        if ((e = attend_backward<T>(p, Q, K, V, sel, dO, go, bws, s, o32, counters)) != cudaSuccess) return e;
        // q = x Wq^T (per head, then RoPE):  dWq = dQp^T x (both MN-major),  dx = dQp Wq + dKp Wk + dVp Wv,
        // each dZp as hi + lo
        using B16 = __nv_bfloat16;
        const B16 *hq = (const B16 *)go.q, *hk = (const B16 *)go.k, *hv = (const B16 *)go.v;
        const size_t n = (size_t)BS * Hd;
        const void *ah[6] = {hq, hq + n, hk, hk + n, hv, hv + n};
        const void *xs[6] = {x, x, x, x, x, x}, *wz[6] = {Wq, Wq, Wk, Wk, Wv, Wv};
        float *cw[3] = {dWq, dWk, dWv}, *cx[1] = {dx};
        if ((e = gemm_grad_tc(Hd, W, BS, 2, 3, ah, true, xs, true, cw, false, slab, L.slab_bytes, counters, s)) !=
            cudaSuccess)
            return e;
        return gemm_grad_tc(BS, W, Hd, 6, 1, ah, false, wz, true, cx, false, slab, L.slab_bytes, counters, s);
    }
    const float *dQp = (const float *)go.q, *dKp = (const float *)go.k, *dVp = (const float *)go.v;
    // delta = O Wo^T:  dO = ddelta Wo,  dWo = ddelta^T O
    if ((e = gemm_any<T, T>(BS, Hd, W, ddelta, W, 1, Wo, Hd, 1, dO, Hd, 0.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    if ((e = gemm_any<T, T>(W, Hd, BS, ddelta, 1, W, O, Hd, 1, dWo, Hd, 0.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    if ((e = attend_backward<T>(p, Q, K, V, sel, dO, go, bws, s)) != cudaSuccess) return e;
    // q = x Wq^T (per head, then RoPE):  dWq = dQp^T x,  dx = dQp Wq + dKp Wk + dVp Wv
    if ((e = gemm_any<float, T>(Hd, W, BS, dQp, 1, Hd, x, W, 1, dWq, W, 0.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    if ((e = gemm_any<float, T>(Hd, W, BS, dKp, 1, Hd, x, W, 1, dWk, W, 0.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    if ((e = gemm_any<float, T>(Hd, W, BS, dVp, 1, Hd, x, W, 1, dWv, W, 0.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    if ((e = gemm_any<float, T>(BS, W, Hd, dQp, Hd, 1, Wq, W, 1, dx, W, 0.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    if ((e = gemm_any<float, T>(BS, W, Hd, dKp, Hd, 1, Wk, W, 1, dx, W, 1.f, slab, L.slab_bytes, s)) !=
        cudaSuccess)
        return e;
    return gemm_any<float, T>(BS, W, Hd, dVp, Hd, 1, Wv, W, 1, dx, W, 1.f, slab, L.slab_bytes, s);
}

int bwd_check(std::initializer_list<const void *> ptrs) {
    for (const void *q : ptrs) {
        if (!q) return MONO_ERR_NULL;
        if ((uintptr_t)q & 15) return MONO_ERR_ALIGN;
    }
    return MONO_OK;
}

int bwd_status(cudaError_t e) { return e == cudaSuccess ? MONO_OK : MONO_ERR_CUDA; }

}  // namespace
}  // namespace mono

using namespace mono;

extern "C" {

int mono_backward_workspace_bytes(const mono_plan_t *plan, size_t *bytes) {
    if (!plan || !bytes) return MONO_ERR_NULL;
    *bytes = bwd_layout(plan->p).total;
    return MONO_OK;
}

int mono_attend_backward(const mono_plan_t *plan, const void *Q, const void *K, const void *V, const int32_t *sel,
                         const float *dO, float *dQ, float *dK, float *dV, void *bwd_workspace, void *stream) {
    if (!plan) return MONO_ERR_NULL;
    if (!bwd_workspace) return MONO_ERR_WORKSPACE;
    if ((uintptr_t)bwd_workspace & 255) return MONO_ERR_ALIGN;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (c.B == 0 || c.S == 0) return MONO_OK;
    int st = bwd_check({Q, K, V, dO, dQ, dK, dV});
    if (st) return st;
    if (c.R > 0 && (st = bwd_check({sel}))) return st;
    cudaStream_t s = (cudaStream_t)stream;
    GradOut go{};
    go.q = dQ;
    go.k = dK;
    go.v = dV;
    go.mode = kOutHeads;
    if (c.dtype == MONO_BF16)
        return bwd_status(attend_backward<__nv_bfloat16>(p, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                                                         (const __nv_bfloat16 *)V, sel, dO, go, (char *)bwd_workspace,
                                                         s));
    return bwd_status(attend_backward<float>(p, (const float *)Q, (const float *)K, (const float *)V, sel, dO, go,
                                             (char *)bwd_workspace, s));
}

int mono_backward(const mono_plan_t *plan, const void *x, const void *Wq, const void *Wk, const void *Wv,
                  const void *Wo, const int32_t *sel, const void *ddelta, float *dx, float *dWq, float *dWk,
                  float *dWv, float *dWo, void *workspace, void *bwd_workspace, void *stream) {
    if (!plan) return MONO_ERR_NULL;
    if (!workspace || !bwd_workspace) return MONO_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255) || ((uintptr_t)bwd_workspace & 255)) return MONO_ERR_ALIGN;
    const Plan &p = plan->p;
    const mono_config &c = p.cfg;
    if (c.B == 0 || c.S == 0) return MONO_OK;
    int st = bwd_check({x, Wq, Wk, Wv, Wo, ddelta, dx, dWq, dWk, dWv, dWo});
    if (st) return st;
    if (c.R > 0 && (st = bwd_check({sel}))) return st;
    // the forward activations for this selection: Q, K, V and O in the workspace
    void *Q = (char *)workspace + p.off[kRegQ], *K = (char *)workspace + p.off[kRegK];
    void *V = (char *)workspace + p.off[kRegV], *O = (char *)workspace + p.off[kRegO];
    if ((st = mono_project(plan, x, Wq, Wk, Wv, Q, K, V, workspace, stream))) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char *bws = (char *)bwd_workspace;
    // the forward attention; where its local kernel can, it also leaves O in fp32 and the log-sum-exp (in the
    // dK region, free until the dK/dV kernel, and the lse region), so the dQ kernel skips its forward pass
    const BwdLayout BL = bwd_layout(p);
    bool stats = false;
    if (p.fast) {
        if (cudaError_t e = launch_attend_tc(p, Q, K, V, sel, O, workspace, s, kAttendAll, (float *)(bws + BL.dKp),
                                             (float *)(bws + BL.lse), &stats))
            return bwd_status(e);
    } else if ((st = mono_attend(plan, Q, K, V, sel, O, workspace, stream))) {
        return st;
    }
    const float *o32 = stats ? (const float *)(bws + BL.dKp) : nullptr;
    if (c.dtype == MONO_BF16) {
        using B16 = __nv_bfloat16;
        return bwd_status(backward_t<B16>(p, (const B16 *)x, (const B16 *)Wq, (const B16 *)Wk, (const B16 *)Wv,
                                          (const B16 *)Wo, sel, (const B16 *)ddelta, dx, dWq, dWk, dWv, dWo,
                                          (const B16 *)Q, (const B16 *)K, (const B16 *)V, (const B16 *)O, bws, workspace,
                                          s, o32));
    }
    return bwd_status(backward_t<float>(p, (const float *)x, (const float *)Wq, (const float *)Wk, (const float *)Wv,
                                        (const float *)Wo, sel, (const float *)ddelta, dx, dWq, dWk, dWv, dWo,
                                        (const float *)Q, (const float *)K, (const float *)V, (const float *)O, bws,
                                        workspace, s));
}

}  // extern "C"

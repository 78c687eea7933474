// attend_simt.cu -- exact causal softmax over the selected token set,
// query-major, one warp per query-head (the plain baseline; also the fp32
// storage path, where the 1e-5 tolerance rules out bf16 tensor cores).
//
// Source: aitechinspire.com Monodratic article, "Snapshot: key facts from the
// report": each query attends, with exact causal softmax, to the tokens of its
// selected remote blocks plus its guaranteed local blocks.  Sel(t) = tokens of
// the blocks in sel[t] plus s in [max(0, bq-L+1)*Bs, t], bq = t / Bs.
#include "internal.cuh"

namespace mono {

template <typename T, int D>
__device__ __forceinline__ float dot_row(const float *qs, const T *k) {
    float acc = 0.f;
    if constexpr (sizeof(T) == 2) {
        const uint4 *kv = (const uint4 *)k;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            uint4 u = __ldg(kv + c);
            const __nv_bfloat162 *h2 = (const __nv_bfloat162 *)&u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float2 f = __bfloat1622float2(h2[e]);
                acc = fmaf(qs[8 * c + 2 * e], f.x, acc);
                acc = fmaf(qs[8 * c + 2 * e + 1], f.y, acc);
            }
        }
    } else {
        const float4 *kv = (const float4 *)k;
#pragma unroll
        for (int c = 0; c < D / 4; ++c) {
            float4 f = __ldg(kv + c);
            acc = fmaf(qs[4 * c + 0], f.x, acc);
            acc = fmaf(qs[4 * c + 1], f.y, acc);
            acc = fmaf(qs[4 * c + 2], f.z, acc);
            acc = fmaf(qs[4 * c + 3], f.w, acc);
        }
    }
    return acc;
}

// grid (ceil(S/4), H, B), 128 threads: warp w handles query t = 4*blockIdx.x + w.
template <typename T, int D>
__global__ void __launch_bounds__(128) k_attend_simt(const T *__restrict__ Q, const T *__restrict__ K,
                                                     const T *__restrict__ V, const int32_t *__restrict__ sel,
                                                     T *__restrict__ O, unsigned long long *__restrict__ counters,
                                                     int S, int H, int Bs, int L, int R, float scale) {
    constexpr int PER = D / 32;  // output dims per lane
    __shared__ float qs_all[4][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 4 + warp;
    const int h = blockIdx.y, b = blockIdx.z;
    if (t >= S) return;
    const size_t bh = (size_t)b * H + h;
    float *qs = qs_all[warp];
    const T *qp = Q + (bh * S + t) * D;
    for (int i = lane; i < D; i += 32) qs[i] = to_f(qp[i]);
    __syncwarp();
    const T *Kb = K + bh * S * D;
    const T *Vb = V + bh * S * D;
    const int bq = t / Bs;
    const int lim = bq - L;

    float m_run = -INFINITY, l_run = 0.f;
    float o[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = 0.f;

    // segments: R remote blocks, then the local window [lo*Bs, t]
    for (int seg = 0; seg <= R; ++seg) {
        int s0, s1;  // [s0, s1)
        if (seg < R) {
            const int j = sel[(bh * S + t) * R + seg];
            if (j < 0) continue;
            if (j > lim) {
                if (lane == 0) record_error(counters, kDevErrBadSel);
                continue;
            }
            s0 = j * Bs;
            s1 = s0 + Bs;
        } else {
            s0 = max(0, bq - L + 1) * Bs;
            s1 = t + 1;
        }
        for (int c0 = s0; c0 < s1; c0 += 32) {
            const int key = c0 + lane;
            const bool valid = key < s1;
            float sc = valid ? dot_row<T, D>(qs, Kb + (size_t)key * D) * scale : -INFINITY;
            float cmax = sc;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
            const float m_new = fmaxf(m_run, cmax);
            const float corr = expf(m_run - m_new);  // 0 on the first chunk (m_run = -inf)
            const float p = valid ? expf(sc - m_new) : 0.f;
            float psum = p;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
            l_run = l_run * corr + psum;
#pragma unroll
            for (int e = 0; e < PER; ++e) o[e] *= corr;
            const int n = min(32, s1 - c0);
            for (int jj = 0; jj < n; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, p, jj);
                const T *vr = Vb + (size_t)(c0 + jj) * D;
#pragma unroll
                for (int e = 0; e < PER; ++e) o[e] = fmaf(pj, to_f(vr[lane + 32 * e]), o[e]);
            }
            m_run = m_new;
        }
    }
    const float inv = 1.f / l_run;
    T *op = O + ((size_t)b * S + t) * H * D + (size_t)h * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) op[lane + 32 * e] = from_f<T>(o[e] * inv);
}

cudaError_t launch_attend_simt(const Plan &p, const void *Q, const void *K, const void *V, const int32_t *sel,
                               void *O, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    unsigned long long *cnt = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    dim3 grid((c.S + 3) / 4, c.H, c.B);
    const float scale = (float)(1.0 / sqrt((double)c.d));
    if (c.dtype == MONO_BF16) {
        if (c.d == 64)
            k_attend_simt<__nv_bfloat16, 64><<<grid, 128, 0, s>>>((const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                (const __nv_bfloat16 *)V, sel, (__nv_bfloat16 *)O, cnt, c.S, c.H, c.Bs, c.L, c.R, scale);
        else
            k_attend_simt<__nv_bfloat16, 128><<<grid, 128, 0, s>>>((const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                (const __nv_bfloat16 *)V, sel, (__nv_bfloat16 *)O, cnt, c.S, c.H, c.Bs, c.L, c.R, scale);
    } else {
        if (c.d == 64)
            k_attend_simt<float, 64><<<grid, 128, 0, s>>>((const float *)Q, (const float *)K, (const float *)V, sel,
                (float *)O, cnt, c.S, c.H, c.Bs, c.L, c.R, scale);
        else
            k_attend_simt<float, 128><<<grid, 128, 0, s>>>((const float *)Q, (const float *)K, (const float *)V, sel,
                (float *)O, cnt, c.S, c.H, c.Bs, c.L, c.R, scale);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mono

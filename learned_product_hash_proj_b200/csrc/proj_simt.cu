// proj_simt.cu -- RoPE tables and the plain (SIMT, fp32-accumulate) GEMMs
// of the projections: Q/K/V = x W^T with RoPE on Q and K, delta = O Wo^T.
// These are the fp32-storage path and the correctness baseline of the
// tensor-core GEMMs.
#include "internal.cuh"

namespace mono {

// ---------------------------------------------------------------------------
// RoPE rotation tables (interleaved pairs (2i, 2i+1), angle t * theta^(-2i/d)).
// The angle of position t = 64*th + tl is split into a coarse and a fine part;
// both tables hold (cos, sin) evaluated in fp64 and rounded to fp32, and the
// epilogue combines them with the angle-addition identity in fp32.  This keeps
// the rotation accurate to a few fp32 ulps at any position without an fp64
// sincos per element.
// hi: [nhi][d/2] float2 of (th*64) * w_i ; lo: [d/2][64] float2 of tl * w_i,
// frequency-major, so that 32 consecutive positions read 256 contiguous bytes.
// ---------------------------------------------------------------------------
__global__ void k_rope_tables(float2 *hi, float2 *lo, int nhi, int half, int d, double theta) {
    int idx = blockIdx.x * blockDim.x + threadIdx.x;
    int total = (nhi + kRopeLo) * half;
    if (idx >= total) return;
    int row = idx / half, i = idx % half;
    double w = pow(theta, -(2.0 * i) / (double)d);
    double pos = row < nhi ? (double)row * kRopeLo : (double)(row - nhi);
    double s, c;
    sincos(pos * w, &s, &c);
    float2 v = make_float2((float)c, (float)s);
    if (row < nhi) hi[(size_t)row * half + i] = v;
    else lo[(size_t)i * kRopeLo + (row - nhi)] = v;
}

cudaError_t launch_rope_tables(const Plan &p, void *ws, cudaStream_t s) {
    const int half = p.cfg.d / 2;
    const int nhi = (p.cfg.S + kRopeLo - 1) / kRopeLo;
    float2 *hi = (float2 *)ws_ptr(p, ws, kRegRope);
    float2 *lo = hi + (size_t)nhi * half;
    int total = (nhi + kRopeLo) * half;
    k_rope_tables<<<(total + 255) / 256, 256, 0, s>>>(hi, lo, nhi, half, p.cfg.d, p.cfg.rope_theta);
    count_launches(1);
    return cudaGetLastError();
}

__device__ __forceinline__ float2 rope_cs(const float2 *hi, const float2 *lo, int t, int i, int half) {
    float2 a = hi[(size_t)(t / kRopeLo) * half + i];
    float2 b = lo[(size_t)i * kRopeLo + t % kRopeLo];
    // cos(x+y) = cos x cos y - sin x sin y ; sin(x+y) = sin x cos y + cos x sin y
    return make_float2(a.x * b.x - a.y * b.y, a.y * b.x + a.x * b.y);
}

// ---------------------------------------------------------------------------
// C[m, n] = sum_k A[m, k] * Bw[n, k]; 64x64 tile, BK=16, 256 threads, 4x4 per thread.
// Epilogue modes:
//   kModeRope  : row m = b*S + t, column n = h*d + i -> out[b,h,t,i], RoPE applied
//   kModeHeads : same scatter, no rotation (V)
//   kModePlain : out[m, n] row-major (delta)
// ---------------------------------------------------------------------------
enum { kModeRope = 0, kModeHeads = 1, kModePlain = 2 };

struct GemmArgs {
    const void *A;
    const void *Bw[3];
    void *out[3];
    int mode[3];
    int Mrows, N, K;
    int S, H, d;
    const float2 *rope_hi, *rope_lo;
};

template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(GemmArgs g) {
    __shared__ float As[16][64 + 4];
    __shared__ float Bs_[16][64 + 4];
    const int z = blockIdx.z;
    const T *A = (const T *)g.A;
    const T *Bw = (const T *)g.Bw[z];
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < g.K; k0 += 16) {
        // load 64x16 of A and of B: each thread loads 4 elements of each
        for (int e = tid; e < 64 * 16; e += 256) {
            int r = e / 16, c = e % 16;
            int gm = m0 + r, gk = k0 + c;
            As[c][r] = (gm < g.Mrows && gk < g.K) ? to_f(A[(size_t)gm * g.K + gk]) : 0.f;
            int gn = n0 + r;
            Bs_[c][r] = (gn < g.N && gk < g.K) ? to_f(Bw[(size_t)gn * g.K + gk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs_[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    const int mode = g.mode[z];
    T *out = (T *)g.out[z];
    const int half = g.d / 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int m = m0 + ty * 4 + i;
        if (m >= g.Mrows) continue;
        int n = n0 + tx * 4;
        if (mode == kModePlain) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (n + j < g.N) out[(size_t)m * g.N + n + j] = from_f<T>(acc[i][j]);
            continue;
        }
        int b = m / g.S, t = m % g.S;
        int h = n / g.d, c = n % g.d;  // 4 consecutive columns never straddle a head (d % 4 == 0)
        float v[4] = {acc[i][0], acc[i][1], acc[i][2], acc[i][3]};
        if (mode == kModeRope) {
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                float2 cs = rope_cs(g.rope_hi, g.rope_lo, t, c / 2 + pr, half);
                float x0 = v[2 * pr], x1 = v[2 * pr + 1];
                v[2 * pr] = x0 * cs.x - x1 * cs.y;
                v[2 * pr + 1] = x0 * cs.y + x1 * cs.x;
            }
        }
        T *dst = out + (((size_t)b * g.H + h) * g.S + t) * g.d + c;
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = from_f<T>(v[j]);
    }
}

cudaError_t launch_project_simt(const Plan &p, const void *x, const void *Wq, const void *Wk, const void *Wv,
                                void *Q, void *K, void *V, const void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    GemmArgs g{};
    g.A = x;
    g.Bw[0] = Wq; g.Bw[1] = Wk; g.Bw[2] = Wv;
    g.out[0] = Q; g.out[1] = K; g.out[2] = V;
    g.mode[0] = kModeRope; g.mode[1] = kModeRope; g.mode[2] = kModeHeads;
    g.Mrows = c.B * c.S; g.N = c.H * c.d; g.K = c.W;
    g.S = c.S; g.H = c.H; g.d = c.d;
    const int half = c.d / 2, nhi = (c.S + kRopeLo - 1) / kRopeLo;
    g.rope_hi = (const float2 *)ws_ptr(p, (void *)ws, kRegRope);
    g.rope_lo = g.rope_hi + (size_t)nhi * half;
    dim3 grid(g.N / 64, (g.Mrows + 63) / 64, 3);
    if (c.dtype == MONO_BF16) k_gemm_simt<__nv_bfloat16><<<grid, 256, 0, s>>>(g);
    else k_gemm_simt<float><<<grid, 256, 0, s>>>(g);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_out_project_simt(const Plan &p, const void *O, const void *Wo, void *delta, cudaStream_t s) {
    const mono_config &c = p.cfg;
    GemmArgs g{};
    g.A = O;
    g.Bw[0] = Wo;
    g.out[0] = delta;
    g.mode[0] = kModePlain;
    g.Mrows = c.B * c.S; g.N = c.W; g.K = c.H * c.d;
    g.S = c.S; g.H = c.H; g.d = c.d;
    dim3 grid(g.N / 64, (g.Mrows + 63) / 64, 1);
    if (c.dtype == MONO_BF16) k_gemm_simt<__nv_bfloat16><<<grid, 256, 0, s>>>(g);
    else k_gemm_simt<float><<<grid, 256, 0, s>>>(g);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mono

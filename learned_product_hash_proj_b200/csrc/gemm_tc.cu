// gemm_tc.cu -- the projections on the tcgen05 tensor cores (bf16 storage,
// fp32 accumulation): Q/K/V = x W^T with RoPE on Q and K fused into the
// epilogue, and delta = O Wo^T.
//
// One CTA computes a 128 x 128 output tile:
//   warp 0 (one lane)  TMA producer: A and B tiles (64-wide K slices, 128-byte
//                      swizzle) into a STAGES-deep ring, completion counted on
//                      the stage's "full" mbarrier;
//   warp 1 (one lane)  MMA issuer: 4 x tcgen05.mma (K = 16 each) per slice into
//                      a 128 x 128 fp32 accumulator in TMEM, then
//                      tcgen05.commit frees the stage ("empty" mbarrier);
//   warps 2..5         epilogue: TMEM -> registers (32 columns at a time),
//                      RoPE on interleaved pairs, bf16, scatter to [B,H,S,d]
//                      or row-major [M, N].
// Every wait is bounded; on expiry the kernel records an error and finishes.
// TMA loads have no cluster multicast; each CTA loads its own tiles.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.cuh"
#include "tc.cuh"

namespace mono {

using bf16 = __nv_bfloat16;

namespace {

constexpr int BM = 128, BN = 128, BK = 64, STAGES = 3;  // 97 KB: two CTAs per SM
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2;
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + 1024;  // + alignment slack

enum { kEpiRope = 0, kEpiHeads = 1, kEpiPlain = 2, kEpiStage = 3 };
constexpr int kMaxRanks = 8;

struct TmaMaps {
    CUtensorMap a;
    CUtensorMap b[3];
};

struct Epi {
    bf16 *out[3];
    int mode[3];
    int M, N;          // rows, columns of each output
    int S, H, d;
    const float2 *rope_hi, *rope_lo;
    unsigned long long *counters;
    // kEpiStage: row m of the fp32 result goes to stage[c] (c = m / rows_chunk, possibly another GPU's memory)
    // at row rank * rows_chunk + m % rows_chunk
    float *stage[kMaxRanks];
    int rank, rows_chunk;
};

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(tc::smem_u32(mbar))
        : "memory");
}

using tc::desc_sw128;
using tc::mbar_expect_tx;

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *(uint32_t *)&h;
}

// 32 accumulator columns n .. n+31 of output row m: RoPE (kEpiRope) on
// interleaved pairs, bf16, to [B,H,S,d] (kEpiRope, kEpiHeads) or row-major
// [M, N] (kEpiPlain); fp32 to the owner's staging buffer (kEpiStage)
__device__ __forceinline__ void epi_store(const Epi &epi, int mode, bf16 *out, int half, int m, int n, float (&v)[32]) {
    if (mode == kEpiStage) {
        const int c = m / epi.rows_chunk;
        float4 *f4 = (float4 *)(epi.stage[c] + ((size_t)epi.rank * epi.rows_chunk + (m - c * epi.rows_chunk)) * epi.N +
                                n);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) f4[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        return;
    }
    bf16 *dst;
    if (mode == kEpiPlain) {
        dst = out + (size_t)m * epi.N + n;
    } else {
        const int b = m / epi.S, t = m % epi.S;
        const int h = n / epi.d, i0 = n % epi.d;
        if (mode == kEpiRope) {
            const float2 *hi = epi.rope_hi + (size_t)(t / kRopeLo) * half + i0 / 2;
            const float2 *lo = epi.rope_lo + (size_t)(i0 / 2) * kRopeLo + t % kRopeLo;  // frequency-major
#pragma unroll
            for (int pr = 0; pr < 16; ++pr) {
                const float2 a = __ldg(hi + pr), bb = __ldg(lo + pr * kRopeLo);
                const float c = a.x * bb.x - a.y * bb.y, sn = a.y * bb.x + a.x * bb.y;
                const float x0 = v[2 * pr], x1 = v[2 * pr + 1];
                v[2 * pr] = x0 * c - x1 * sn;
                v[2 * pr + 1] = x0 * sn + x1 * c;
            }
        }
        dst = out + (((size_t)b * epi.H + h) * epi.S + t) * epi.d + i0;
    }
    uint4 *d4 = (uint4 *)dst;
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8)
        d4[q8] = make_uint4(pack2(v[8 * q8], v[8 * q8 + 1]), pack2(v[8 * q8 + 2], v[8 * q8 + 3]),
                            pack2(v[8 * q8 + 4], v[8 * q8 + 5]), pack2(v[8 * q8 + 6], v[8 * q8 + 7]));
}

__global__ void __launch_bounds__(192, 2) k_gemm_tc(const __grid_constant__ TmaMaps maps, const Epi epi, int K) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[STAGES], empty[STAGES], accf;
    __shared__ uint32_t tmem_base;
    __shared__ int fail;
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int z = blockIdx.z;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int nk = K / BK;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(&accf, 1);
        tc::fence_mbar_init();
        fail = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(&tmem_base, BN);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp == 0 && lane == 0) {
        // producer
        for (int k = 0; k < nk; ++k) {
            const int s = k % STAGES;
            const uint32_t ph = (k / STAGES) & 1;
            if (k >= STAGES && !tc::mbar_wait(&empty[s], ph ^ 1)) { fail = 1; break; }
            uint8_t *sa = base + s * A_BYTES;
            uint8_t *sb = base + STAGES * A_BYTES + s * B_BYTES;
            mbar_expect_tx(&full[s], A_BYTES + B_BYTES);
            tma_load_2d(sa, &maps.a, k * BK, m0, &full[s]);
            tma_load_2d(sb, &maps.b[z], k * BK, n0, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        const uint32_t id = tc::idesc_bf16(BM, BN);
        bool ok = true;
        for (int k = 0; k < nk; ++k) {
            const int s = k % STAGES;
            const uint32_t ph = (k / STAGES) & 1;
            if (!tc::mbar_wait(&full[s], ph)) { ok = false; fail = 1; break; }
            tc::fence_after_sync();
            const uint32_t sa = tc::smem_u32(base + s * A_BYTES);
            const uint32_t sb = tc::smem_u32(base + STAGES * A_BYTES + s * B_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
                tc::mma_bf16(tmem, desc_sw128(sa + 32 * kk), desc_sw128(sb + 32 * kk), id, (k | kk) != 0);
            tc::commit(&empty[s]);
        }
        if (ok) tc::commit(&accf);
    } else if (warp >= 2) {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int m = m0 + row;
        const bool ok = tc::mbar_wait(&accf, 0, 1u << 20);
        tc::fence_after_sync();
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        const int mode = epi.mode[z];
        bf16 *out = epi.out[z];
        const int half = epi.d / 2;
        for (int c0 = 0; c0 < BN; c0 += 32) {
            float v[32];
            tc::tmem_ld32(trow + c0, v);
            if (!ok || m >= epi.M) continue;
            epi_store(epi, mode, out, half, m, n0 + c0, v);
        }
        if (!ok && lane == 0) fail = 1;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && fail) record_error(epi.counters, kDevErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tmem, BN);
}

// ---------------------------------------------------------------------------
// The same product as a persistent kernel with 128 x 256 tiles: one CTA per SM
// walks the tiles (the n tiles and outputs of one 128-row band of A first, so
// that concurrent CTAs share A in L2).  The producer runs ahead across tile
// boundaries through a 4-stage ring of 48 KB stages; the MMA issuer
// alternates two 128 x 256 fp32 accumulators in TMEM (all 512 columns), so
// the epilogue of tile i (eight warps, two per TMEM lane quarter, each half of
// the columns: TMEM -> registers -> RoPE -> bf16 stores) overlaps the MMAs of
// tile i+1.
// ---------------------------------------------------------------------------
constexpr int PBN = 256, PSTAGES = 4;
constexpr int PB_BYTES = PBN * BK * 2;
constexpr int PSMEM_BYTES = PSTAGES * (A_BYTES + PB_BYTES) + 1024;

__global__ void __launch_bounds__(320, 1) k_gemm_tcp(const __grid_constant__ TmaMaps maps, const Epi epi, int K,
                                                     int tiles_n, int tiles_m, int nz) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[PSTAGES], empty[PSTAGES], accf[2], accfree[2], drain;
    __shared__ uint32_t tmem_base;
    __shared__ int fail;
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = K / BK;
    const int total = tiles_n * tiles_m * nz;
    const int G = gridDim.x;
    auto tile_of = [&](int t, int &m0, int &n0, int &z) {
        const int per_m = tiles_n * nz;
        m0 = (t / per_m) * BM;
        const int r = t % per_m;
        z = r / tiles_n;
        n0 = (r % tiles_n) * PBN;
    };
    if (tid == 0) {
        for (int s = 0; s < PSTAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(&accf[a], 1);
            tc::mbar_init(&accfree[a], 8);
        }
        tc::mbar_init(&drain, 1);
        tc::fence_mbar_init();
        fail = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(&tmem_base, 2 * PBN);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp == 0 && lane == 0) {
        // producer: every k slice of every tile of this CTA, one ring
        int kc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += G) {
            int m0, n0, z;
            tile_of(t, m0, n0, z);
            for (int k = 0; k < nk; ++k, ++kc) {
                const int s = kc % PSTAGES;
                if (kc >= PSTAGES && !tc::mbar_wait(&empty[s], ((kc / PSTAGES) - 1) & 1)) { ok = false; break; }
                uint8_t *sa = base + s * (A_BYTES + PB_BYTES);
                uint8_t *sb = sa + A_BYTES;
                mbar_expect_tx(&full[s], A_BYTES + PB_BYTES);
                tma_load_2d(sa, &maps.a, k * BK, m0, &full[s]);
                tma_load_2d(sb, &maps.b[z], k * BK, n0, &full[s]);
            }
        }
        if (!ok) {
            fail = 1;
            // leave no copy in flight: the last load of each stage has landed
            for (int j = kc - 1; j >= 0 && j >= kc - PSTAGES; --j) tc::mbar_wait(&full[j % PSTAGES], (j / PSTAGES) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: tile lt of this CTA into accumulator lt & 1
        const uint32_t id = tc::idesc_bf16(BM, PBN);
        int kc = 0, lt = 0;
        for (int t = blockIdx.x; t < total && !fail; t += G, ++lt) {
            const int a = lt & 1;
            if (lt >= 2 && !tc::mbar_wait(&accfree[a], ((lt >> 1) - 1) & 1, 1u << 20)) { fail = 1; break; }
            tc::fence_after_sync();
            bool ok = true;
            for (int k = 0; k < nk; ++k, ++kc) {
                const int s = kc % PSTAGES;
                if (!tc::mbar_wait(&full[s], (kc / PSTAGES) & 1)) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t sa = tc::smem_u32(base + s * (A_BYTES + PB_BYTES));
                const uint32_t sb = sa + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc::mma_bf16(tmem + a * PBN, desc_sw128(sa + 32 * kk), desc_sw128(sb + 32 * kk), id,
                                 (k | kk) != 0);
                tc::commit(&empty[s]);
            }
            if (!ok) { fail = 1; break; }
            tc::commit(&accf[a]);
        }
        // every MMA issued has completed before the CTA frees its tensor memory
        tc::commit(&drain);
        if (!tc::mbar_wait(&drain, 0, 1u << 20)) fail = 1;
    } else if (warp >= 2) {
        // epilogue, eight warps: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows, columns
        // [128 c, 128 c + 128) with c = (w - 2) / 4
        const int q = warp & 3, ch = (warp - 2) >> 2;
        const int half = epi.d / 2;
        int lt = 0;
        for (int t = blockIdx.x; t < total; t += G, ++lt) {
            int m0, n0, z;
            tile_of(t, m0, n0, z);
            const int a = lt & 1;
            const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&accf[a], (lt >> 1) & 1, 1u << 20));
            if (!ok) { if (lane == 0) fail = 1; break; }
            tc::fence_after_sync();
            const uint32_t trow = tmem + a * PBN + ((uint32_t)(q * 32) << 16);
            const int m = m0 + q * 32 + lane;
            const int mode = epi.mode[z];
            bf16 *out = epi.out[z];
            for (int c0 = ch * (PBN / 2); c0 < (ch + 1) * (PBN / 2); c0 += 32) {
                float v[32];
                __syncwarp();
                tc::tmem_ld32(trow + c0, v);
                if (m < epi.M) epi_store(epi, mode, out, half, m, n0 + c0, v);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&accfree[a]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && fail) record_error(epi.counters, kDevErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tmem, 2 * PBN);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encode() {
    g_encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    return g_encode != nullptr;
}

// rows x K bf16 row-major matrix, box 64 (K) x box_rows, 128-byte swizzle
bool make_map(CUtensorMap *map, const void *ptr, long long rows, int K, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

void *tensor_map_encoder() {
    static std::once_flag once;
    static void *fn = nullptr;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = f;
    });
    return fn;
}

namespace {

cudaError_t launch(const TmaMaps &maps, const Epi &epi, int nz, int K, cudaStream_t s) {
    // set on every call: the attribute belongs to the current device, and a host call is cheap next to the GEMM
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(epi.N / BN, (epi.M + BM - 1) / BM, nz);
    k_gemm_tc<<<grid, 192, SMEM_BYTES, s>>>(maps, epi, K);
    count_launches(1);
    return cudaGetLastError();
}

// the persistent 128 x 256 kernel; `maps.b` boxes 256 rows
cudaError_t launch_persistent(const TmaMaps &maps, const Epi &epi, int nz, int K, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tcp, cudaFuncAttributeMaxDynamicSharedMemorySize, PSMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int tn = epi.N / PBN, tm = (epi.M + BM - 1) / BM;
    const int total = tn * tm * nz;
    k_gemm_tcp<<<std::min(total, sms), 320, PSMEM_BYTES, s>>>(maps, epi, K, tn, tm, nz);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool gemm_tc_supported(const mono_config &c) {
    return c.dtype == MONO_BF16 && c.W % BK == 0 && (c.H * c.d) % BN == 0 && c.W % BN == 0 &&
           (c.H * c.d) % BK == 0 && (long long)c.B * c.S < (1ll << 31);
}

cudaError_t launch_project_tc(const Plan &p, const void *x, const void *Wq, const void *Wk, const void *Wv, void *Q,
                              void *K, void *V, const void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    if (!get_encode()) return cudaErrorNotSupported;
    TmaMaps maps;
    const long long M = (long long)c.B * c.S;
    const int N = c.H * c.d;
    if (!make_map(&maps.a, x, M, c.W, BM) || !make_map(&maps.b[0], Wq, N, c.W, BN) ||
        !make_map(&maps.b[1], Wk, N, c.W, BN) || !make_map(&maps.b[2], Wv, N, c.W, BN))
        return cudaErrorInvalidValue;
    Epi epi{};
    epi.out[0] = (bf16 *)Q; epi.out[1] = (bf16 *)K; epi.out[2] = (bf16 *)V;
    epi.mode[0] = kEpiRope; epi.mode[1] = kEpiRope; epi.mode[2] = kEpiHeads;
    epi.M = (int)M; epi.N = N; epi.S = c.S; epi.H = c.H; epi.d = c.d;
    const int half = c.d / 2, nhi = (c.S + kRopeLo - 1) / kRopeLo;
    epi.rope_hi = (const float2 *)ws_ptr(p, (void *)ws, kRegRope);
    epi.rope_lo = epi.rope_hi + (size_t)nhi * half;
    epi.counters = (unsigned long long *)ws_ptr(p, (void *)ws, kRegCounters);
    if (N % PBN == 0) {
        if (!make_map(&maps.b[0], Wq, N, c.W, PBN) || !make_map(&maps.b[1], Wk, N, c.W, PBN) ||
            !make_map(&maps.b[2], Wv, N, c.W, PBN))
            return cudaErrorInvalidValue;
        return launch_persistent(maps, epi, 3, c.W, s);
    }
    return launch(maps, epi, 3, c.W, s);
}

cudaError_t launch_out_project_tc(const Plan &p, const void *O, const void *Wo, void *delta, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    if (!get_encode()) return cudaErrorNotSupported;
    TmaMaps maps;
    const long long M = (long long)c.B * c.S;
    const int Kd = c.H * c.d;
    if (!make_map(&maps.a, O, M, Kd, BM) || !make_map(&maps.b[0], Wo, c.W, Kd, BN)) return cudaErrorInvalidValue;
    maps.b[1] = maps.b[0];
    maps.b[2] = maps.b[0];
    Epi epi{};
    epi.out[0] = (bf16 *)delta;
    epi.mode[0] = kEpiPlain;
    epi.M = (int)M; epi.N = c.W; epi.S = c.S; epi.H = c.H; epi.d = c.d;
    epi.counters = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    if (c.W % PBN == 0) {
        if (!make_map(&maps.b[0], Wo, c.W, Kd, PBN)) return cudaErrorInvalidValue;
        maps.b[1] = maps.b[0];
        maps.b[2] = maps.b[0];
        return launch_persistent(maps, epi, 1, Kd, s);
    }
    return launch(maps, epi, 1, Kd, s);
}

// ---------------------------------------------------------------------------
// The gradient GEMMs on the tensor cores: C_g[M,N] (fp32, row-major) (+)=
// sum_src A_src(m,k) B_src(n,k) over bf16 operands, each stored K-major
// ([M or N rows][K], a row contiguous in k) or MN-major ([K rows][M or N], a
// row contiguous in m or n).  ngroups independent outputs (dWq, dWk, dWv),
// each the sum of nsrc products over the same K (dx = dQp Wq + dKp Wk + dVp Wv;
// an fp32 operand given as the two bf16 terms of its hi + lo split); the k
// slices are split over blockIdx.z, each range's partial tile stored in its
// own slab and the slabs summed in range order by k_split_sum (the same bits
// on every run).  Same roles as k_gemm_tc; an MN-major tile is two 64-wide column
// blocks of 64 K-rows each (128-byte swizzle), 8 KB apart.
// ---------------------------------------------------------------------------
namespace {

constexpr int kGradMaxOps = 6;

struct GradMaps {
    CUtensorMap a[kGradMaxOps];  // group-major: operand pair g * nsrc + src
    CUtensorMap b[kGradMaxOps];
};

struct GradArgs {
    float *out[3];
    int M, N, K;     // of each product
    int nsrc;        // products summed into each output
    int ngroups;     // outputs
    int split;       // k-slice ranges per output tile (blockIdx.z % split)
    int a_mn, b_mn;  // operand major-ness
    int atomic;      // add into C instead of storing
    float *slab;     // split > 1: range part of output g goes to slab + (g * split + part) * M * N
    unsigned long long *counters;
};

__device__ __forceinline__ void load_operand(uint8_t *dst, const CUtensorMap *map, bool mn, int mn0, int k0,
                                             uint64_t *bar) {
    if (mn) {
        tma_load_2d(dst, map, mn0, k0, bar);
        tma_load_2d(dst + A_BYTES / 2, map, mn0 + 64, k0, bar);
    } else {
        tma_load_2d(dst, map, k0, mn0, bar);
    }
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr, bool mn, int kk) {
    return mn ? tc::desc_sw128_mn(saddr + 2048 * kk, A_BYTES / 2) : desc_sw128(saddr + 32 * kk);
}

__global__ void __launch_bounds__(192, 2) k_gemm_grad_tc(const __grid_constant__ GradMaps maps, const GradArgs g) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[STAGES], empty[STAGES], accf;
    __shared__ uint32_t tmem_base;
    __shared__ int fail;
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = blockIdx.z / g.split, part = blockIdx.z % g.split;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int kslices = (g.K + BK - 1) / BK;
    const int total = kslices * g.nsrc;
    const int per = (total + g.split - 1) / g.split;
    const int kb = part * per;
    const int nk = max(0, min(total, kb + per) - kb);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(&accf, 1);
        tc::fence_mbar_init();
        fail = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(&tmem_base, BN);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;
    const bool amn = g.a_mn != 0, bmn = g.b_mn != 0;

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            const uint32_t ph = (i / STAGES) & 1;
            if (i >= STAGES && !tc::mbar_wait(&empty[s], ph ^ 1)) { fail = 1; break; }
            const int sl = kb + i;
            const int src = grp * g.nsrc + sl / kslices;
            const int k0 = (sl % kslices) * BK;
            uint8_t *sa = base + s * A_BYTES;
            uint8_t *sb = base + STAGES * A_BYTES + s * B_BYTES;
            mbar_expect_tx(&full[s], A_BYTES + B_BYTES);
            load_operand(sa, &maps.a[src], amn, m0, k0, &full[s]);
            load_operand(sb, &maps.b[src], bmn, n0, k0, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t id = tc::idesc_bf16(BM, BN, bmn, amn);
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
            const int s = i % STAGES;
            const uint32_t ph = (i / STAGES) & 1;
            if (!tc::mbar_wait(&full[s], ph)) { ok = false; fail = 1; break; }
            tc::fence_after_sync();
            const uint32_t sa = tc::smem_u32(base + s * A_BYTES);
            const uint32_t sb = tc::smem_u32(base + STAGES * A_BYTES + s * B_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
                tc::mma_bf16(tmem, operand_desc(sa, amn, kk), operand_desc(sb, bmn, kk), id, (i | kk) != 0);
            tc::commit(&empty[s]);
        }
        if (ok && nk > 0) tc::commit(&accf);
    } else if (warp >= 2) {
        // warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows
        const int q = warp & 3;
        const int m = m0 + q * 32 + lane;
        const bool ok = nk > 0 && tc::mbar_wait(&accf, 0, 1u << 20);
        tc::fence_after_sync();
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        float *out = g.slab ? g.slab + ((size_t)grp * g.split + part) * g.M * g.N : g.out[grp];
        for (int c0 = 0; c0 < BN; c0 += 32) {
            float v[32];
            tc::tmem_ld32(trow + c0, v);
            if (!ok || m >= g.M) continue;
            const int n = n0 + c0;
            float *dst = out + (size_t)m * g.N + n;
            if (n + 32 <= g.N) {
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const float4 f = make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
                    if (g.atomic) atomicAdd((float4 *)dst + c4, f);
                    else ((float4 *)dst)[c4] = f;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    if (n + c >= g.N) break;
                    if (g.atomic) atomicAdd(dst + c, v[c]);
                    else dst[c] = v[c];
                }
            }
        }
        if (nk > 0 && !ok && lane == 0) fail = 1;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && fail) record_error(g.counters, kDevErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tmem, BN);
}

// C_g (+)= sum over parts of slab[g][part] in ascending part order; n4 float4s per output
__global__ void __launch_bounds__(256) k_split_sum(const float4 *__restrict__ slab, float4 *__restrict__ c0,
                                                   float4 *__restrict__ c1, float4 *__restrict__ c2, long long n4,
                                                   int split, int ngroups, int accumulate) {
    const long long total = n4 * ngroups;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int g = (int)(i / n4);
        const long long e = i % n4;
        const float4 *src = slab + (size_t)g * split * n4 + e;
        float4 a = __ldg(src);
        for (int p = 1; p < split; ++p) {
            const float4 b = __ldg(src + (size_t)p * n4);
            a.x = __fadd_rn(a.x, b.x);
            a.y = __fadd_rn(a.y, b.y);
            a.z = __fadd_rn(a.z, b.z);
            a.w = __fadd_rn(a.w, b.w);
        }
        float4 *dst = (g == 0 ? c0 : g == 1 ? c1 : c2) + e;
        if (accumulate) {
            const float4 o = *dst;
            a = make_float4(__fadd_rn(o.x, a.x), __fadd_rn(o.y, a.y), __fadd_rn(o.z, a.z), __fadd_rn(o.w, a.w));
        }
        *dst = a;
    }
}

}  // namespace

bool gemm_grad_tc_supported(int M, int N, int K, bool a_mn, bool b_mn) {
    // TMA row strides are multiples of 16 bytes; fp32 rows of C hold whole float4s
    return M > 0 && N > 0 && K > 0 && (a_mn ? M % 8 : K % 8) == 0 && (b_mn ? N % 8 : K % 8) == 0 && N % 4 == 0 &&
           tensor_map_encoder() != nullptr;
}

cudaError_t gemm_grad_tc(int M, int N, int K, int nsrc, int ngroups, const void *const *A, bool a_mn,
                         const void *const *B, bool b_mn, float *const *C, bool accumulate, float *slab,
                         size_t slab_bytes, unsigned long long *counters, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (nsrc < 1 || ngroups < 1 || ngroups > 3 || nsrc * ngroups > kGradMaxOps) return cudaErrorInvalidValue;
    if (!gemm_grad_tc_supported(M, N, K, a_mn, b_mn) || !get_encode()) return cudaErrorNotSupported;
    GradMaps maps;
    const int nmaps = nsrc * ngroups;
    for (int i = 0; i < nmaps; ++i) {
        // K-major: [MN rows][K], box 64 x 128; MN-major: [K rows][MN], box 64 x 64 (two per tile)
        const bool ok_a = a_mn ? make_map(&maps.a[i], A[i], K, M, 64) : make_map(&maps.a[i], A[i], M, K, BM);
        const bool ok_b = b_mn ? make_map(&maps.b[i], B[i], K, N, 64) : make_map(&maps.b[i], B[i], N, K, BN);
        if (!ok_a || !ok_b) return cudaErrorInvalidValue;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int slots = 2 * sms;
    const int tiles = ((N + BN - 1) / BN) * ((M + BM - 1) / BM) * ngroups;
    const int total = ((K + BK - 1) / BK) * nsrc;
    // split K only where the tiles alone leave CTA slots idle (fewer tiles than slots): the smallest split
    // whose wave fill is clearly (5 %) better than every smaller one's; each split re-adds the output once
    int split = 1;
    if (tiles < slots) {
        double best = (double)tiles / (double)slots;
        for (int sp = 2; sp <= 16 && total / sp >= 4; ++sp) {
            const long long ctas = (long long)tiles * sp;
            const double fill = (double)ctas / (double)(((ctas + slots - 1) / slots) * slots);
            if (fill > best * 1.05) {
                best = fill;
                split = sp;
            }
        }
    }
    // as many slabs as the scratch holds
    const size_t out_bytes = (size_t)M * N * sizeof(float);
    while (split > 1 && (!slab || (size_t)ngroups * split * out_bytes > slab_bytes)) --split;
    const int per = (total + split - 1) / split;
    split = (total + per - 1) / per;  // every k range non-empty
    GradArgs g{};
    for (int i = 0; i < 3; ++i) g.out[i] = C[i < ngroups ? i : 0];
    g.M = M; g.N = N; g.K = K; g.nsrc = nsrc; g.ngroups = ngroups; g.split = split;
    g.a_mn = a_mn; g.b_mn = b_mn;
    g.atomic = split == 1 && accumulate;  // one CTA per output element: a deterministic add
    g.slab = split > 1 ? slab : nullptr;
    g.counters = counters;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k_gemm_grad_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, ngroups * split);
    k_gemm_grad_tc<<<grid, 192, SMEM_BYTES, s>>>(maps, g);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess || split == 1) return e;
    const long long n4 = (long long)M * N / 4;
    const int grid2 = (int)std::min<long long>((n4 * ngroups + 255) / 256, 8ll * sms);
    k_split_sum<<<grid2, 256, 0, s>>>((const float4 *)slab, (float4 *)C[0], (float4 *)C[ngroups > 1 ? 1 : 0],
                                      (float4 *)C[ngroups > 2 ? 2 : 0], n4, split, ngroups, accumulate ? 1 : 0);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mono

namespace mono {

// ---------------------------------------------------------------------------
// Output projection of one head shard fused with the scatter half of a
// reduce-scatter: the fp32 tile of rows [m0, m0 + 128) goes straight from the
// epilogue to the staging buffer of the rank that owns each row (rows split
// into nranks equal chunks), which may be another GPU's memory reached over
// NVLink (plain stores).  The transfer of a tile overlaps the MMAs of the
// next tiles; no partial is rounded to bf16.
// ---------------------------------------------------------------------------
cudaError_t launch_out_project_stage(const Plan &p, const void *O, const void *Wo, float *const *stage, int nranks,
                                     int rank, void *ws, cudaStream_t s) {
    const mono_config &c = p.cfg;
    if (!get_encode()) return cudaErrorNotSupported;
    if (nranks < 1 || nranks > kMaxRanks) return cudaErrorInvalidValue;
    TmaMaps maps;
    const long long M = (long long)c.B * c.S;
    const int Kd = c.H * c.d;
    if (!make_map(&maps.a, O, M, Kd, BM) || !make_map(&maps.b[0], Wo, c.W, Kd, BN)) return cudaErrorInvalidValue;
    maps.b[1] = maps.b[0];
    maps.b[2] = maps.b[0];
    Epi epi{};
    epi.mode[0] = kEpiStage;
    epi.M = (int)M; epi.N = c.W; epi.S = c.S; epi.H = c.H; epi.d = c.d;
    epi.counters = (unsigned long long *)ws_ptr(p, ws, kRegCounters);
    for (int r = 0; r < nranks; ++r) epi.stage[r] = stage[r];
    epi.rank = rank;
    epi.rows_chunk = (int)(M / nranks);
    return launch(maps, epi, 1, Kd, s);
}

// ---------------------------------------------------------------------------
// The reduce half: this rank's chunk is the sum of the nranks partials staged
// for it, added in fp32 in ascending rank order and rounded once to bf16.
// stage [nranks][rows][W] fp32 (this GPU's buffer), out [rows][W] bf16.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_stage_reduce(const float4 *__restrict__ stage, uint2 *__restrict__ out,
                                                      long long n4, int nranks) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        float4 a = __ldg(stage + i);
        for (int r = 1; r < nranks; ++r) {
            const float4 b = __ldg(stage + (size_t)r * n4 + i);
            a.x = __fadd_rn(a.x, b.x);
            a.y = __fadd_rn(a.y, b.y);
            a.z = __fadd_rn(a.z, b.z);
            a.w = __fadd_rn(a.w, b.w);
        }
        out[i] = make_uint2(pack2(a.x, a.y), pack2(a.z, a.w));
    }
}

cudaError_t launch_stage_reduce(const Plan &p, const float *stage, int nranks, void *out, cudaStream_t s) {
    const mono_config &c = p.cfg;
    const long long n4 = (long long)c.B * c.S / nranks * c.W / 4;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (n4 + 255) / 256;
    const int grid = (int)std::max<long long>(1, std::min<long long>(want, 8ll * sms));
    k_stage_reduce<<<grid, 256, 0, s>>>((const float4 *)stage, (uint2 *)out, n4, nranks);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mono

// tc.cuh -- thin wrappers over the sm_100a tensor-core instructions used by
// the fast kernels: tcgen05 MMA with fp32 accumulators in tensor memory
// (TMEM), TMEM allocation and loads, mbarrier completion with bounded waits,
// and the shared-memory matrix descriptors.
//
// Operand tiles in shared memory use the canonical K-major layout without
// swizzle: an 8-row x 16-byte "core matrix" is 128 contiguous bytes; core
// matrices adjacent along K are `lbo` bytes apart and 8-row groups are `sbo`
// bytes apart.  `kmajor_offset` gives the byte offset of element (row, k).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace mono {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// byte offset of bf16 element (row, k) in a K-major no-swizzle tile whose rows hold `kdim` elements
__device__ __forceinline__ uint32_t kmajor_offset(int row, int k, int kdim) {
    return (uint32_t)((row >> 3) * (kdim * 16) + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

// byte offset of the 16-byte chunk holding elements (row, 8c .. 8c+7)
__device__ __forceinline__ uint32_t kmajor_chunk(int row, int c, int kdim) {
    return (uint32_t)((row >> 3) * (kdim * 16) + c * 128 + (row & 7) * 16);
}

// shared-memory matrix descriptor, K-major, no swizzle.
// lbo: bytes between K-adjacent core matrices (128); sbo: bytes between 8-row groups (kdim * 16).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr, int kdim) {
    const uint64_t lbo = 128, sbo = (uint64_t)kdim * 16;
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)(lbo >> 4) << 16;
    d |= (uint64_t)(sbo >> 4) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    // base offset 0, lbo mode 0, layout type 0 (no swizzle)
    return d;
}

// Shared-memory descriptor of an MN-major operand without swizzle (B = V in
// O = P V, whose N = d dimension is contiguous in memory).  Here a core
// matrix is 8 K-rows x 8 MN-elements (16 bytes per K-row, 128 contiguous
// bytes); K-adjacent groups of 8 rows are `lbo` bytes apart and MN-adjacent
// groups of 8 elements are `sbo` bytes apart.  The tile of `nk` K-rows is
// laid out with lbo = 128 and sbo = nk * 16 (see mnmajor_chunk).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr, int nk) {
    const uint64_t lbo = 128, sbo = (uint64_t)nk * 16;
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)(lbo >> 4) << 16;
    d |= (uint64_t)(sbo >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// byte offset of the 16-byte chunk holding MN-elements 8c .. 8c+7 of K-row k, in an MN-major tile of nk K-rows
__device__ __forceinline__ uint32_t mnmajor_chunk(int k, int c, int nk) {
    return (uint32_t)(c * (nk * 16) + (k >> 3) * 128 + (k & 7) * 16);
}

// instruction descriptor: kind::f16, A = B = bf16, D = f32, M x N; A and B
// each K-major (false) or MN-major (true).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn = false, bool a_mn = false) {
    return (1u << 4)                    // D format f32
           | (1u << 7)                  // A format bf16
           | (1u << 10)                 // B format bf16
           | ((a_mn ? 1u : 0u) << 15)   // A major-ness
           | ((b_mn ? 1u : 0u) << 16)   // B major-ness
           | ((uint32_t)(N >> 3) << 17) //
           | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T ; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M x 16, bf16 pairs packed in 32-bit
// columns, row m in lane m) read from tensor memory; issued by one thread.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// arrive once on `mbar` when every MMA this thread issued before has completed
__device__ __forceinline__ void commit(uint64_t *mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(mbar))
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// make this thread's generic-proxy shared-memory writes visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// --- TMEM allocation (one full warp) -------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// --- TMEM -> registers: 32 lanes x 32 consecutive 32-bit columns ----------
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// --- registers -> TMEM: 32 lanes x 16 consecutive 32-bit columns ----------
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// --- asynchronous 16-byte global -> shared copies (cp.async) -------------
// `valid` false zero-fills the destination without reading the source.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
                 "r"(valid ? 16u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 32 bytes from global memory through the non-coherent path in one 256-bit
// load (sm_100); p must be 32-byte aligned
__device__ __forceinline__ void ldg_v8(const float *p, float (&v)[8]) {
    asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "l"(p));
}
__device__ __forceinline__ void ldg_v8(const void *p, uint4 &a, uint4 &b) {
    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}
// 2^x by the special-function unit (PTX ex2.approx.ftz: a few ulp, results
// below the smallest normal flushed to zero): the softmax exponentials, whose
// tolerance is that of bf16 storage
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
__device__ __forceinline__ void prefetch_l1(const void *p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// --- programmatic dependent launch --------------------------------------------
// grid_dep_wait: wait until the kernel this one was launched after (with the
// programmatic-serialisation attribute) has completed and its writes are
// visible; a no-op for a kernel launched without a programmatic predecessor.
// grid_dep_launch: let the kernel launched after this one start its own
// prologue (its blocks are scheduled once every block of this one has issued
// it or exited).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// --- TMA tile loads (no cluster multicast) --------------------------------
// `map` is the address of a CUtensorMap in parameter, constant or global memory.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *map, int x, int y, int z, uint64_t *mbar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(mbar))
        : "memory");
}

// arrive on `mbar` and add `bytes` to the transaction count its phase waits for
__device__ __forceinline__ void mbar_expect_tx(uint64_t *mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(mbar)), "r"(bytes) : "memory");
}

// Descriptors of tiles written by TMA with the 128-byte swizzle: rows of 128
// bytes (64 bf16), 8-row atoms of 1024 bytes.  K-major: an operand row is a
// tile row; K advances 32 bytes per 16-element step inside the atom.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)1 << 16;            // leading byte offset: unused for swizzled K-major
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: next 8-row atom
    d |= (uint64_t)1 << 46;            // sm_100 descriptor version
    d |= (uint64_t)2 << 61;            // SWIZZLE_128B
    return d;
}
// MN-major (B = V in O = P V): a tile row is one K index (a key) holding 64
// MN elements; 8-key atoms are 1024 bytes apart along K (stride byte
// offset), 64-element column blocks `lbo` bytes apart along MN.
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)((lbo & 0x3FFFF) >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// --- mbarrier with a bounded wait ---------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait(uint64_t *mbar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(mbar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `mbar` to complete.  Gives up after `limit`
// polls (each try_wait itself suspends for a hardware-bounded time) and
// returns false; the caller records an error and carries on so the kernel
// always terminates.
__device__ __forceinline__ bool mbar_wait(uint64_t *mbar, uint32_t parity, uint32_t limit = 1u << 16) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(mbar, parity)) return true;
    return false;
}

// the same, also giving up as soon as *abort (shared, set by another role) is nonzero
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t *mbar, uint32_t parity, const volatile int *abort,
                                                   uint32_t limit = 1u << 16) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(mbar, parity)) return true;
        if (*abort) return false;
    }
    return false;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mbar)) : "memory");
}

// ---------------------------------------------------------------------------
// Paired fp32 arithmetic of sm_100: fma.rn.f32x2 performs two independent
// IEEE fused multiply-adds, each rounded once to nearest-even, on the two
// 32-bit halves of 64-bit registers.  One instruction advances two fma chains
// by one step, with exactly the results of two __fmaf_rn calls.
// ---------------------------------------------------------------------------
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2_dup(float v) {
    f2_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ void f2_split(f2_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ f2_t f2_pack(float lo, float hi) {
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

}  // namespace tc
}  // namespace mono

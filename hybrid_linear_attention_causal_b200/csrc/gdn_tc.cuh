// tcgen05 (5th-generation tensor core) helpers for sm_100a, written as inline
// PTX from the PTX ISA's tcgen05 / mbarrier instruction descriptions.
//
// Conventions used by the GDN kernels:
//   - kind::f16 MMAs with fp16 operands and fp32 accumulators in tensor memory
//     (TMEM), one CTA (cta_group::1), one elected thread issues.  (kind::tf32
//     helpers are kept for reference products; the kernels do not use them.)
//   - shared-memory operands use the no-swizzle canonical layout built from
//     8 x 16-byte "core matrices" (128 contiguous bytes each).  A tile of R rows
//     keeps element (r, k) of a 16-bit tile at byte
//           ((k/8) * (R/8) + r/8) * 128 + (r%8) * 16 + (k%8) * 2      (kmajor_off16)
//     As a K-major operand (rows r along M or N, k along K) its descriptor has
//     LBO = (R/8) * 128 (next 8 k) and SBO = 128 (next 8 r).  The same bytes
//     serve as an MN-major operand whose K runs along the rows r and whose M or
//     N runs along k: LBO = 128 (next 8 along K), SBO = (R/8) * 128 (next 8
//     along M or N), and the instruction descriptor's transpose bit for that
//     operand set (checked on B200 against an fp64 product: max abs error 5e-7
//     on a 128 x 128 x 64 product; the other LBO/SBO assignment gives garbage).
//   - every operand value is rounded to fp16 (round to nearest even) before it
//     is stored, so the tensor core sees exactly the value the kernel chose.
//   - every wait on an mbarrier gives up after a time limit and reports it,
//     so a kernel can never hang the GPU.
#pragma once

#include <stdint.h>

namespace gdn {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float round_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

__device__ __forceinline__ float4 round_tf32(float4 v) {
    return make_float4(round_tf32(v.x), round_tf32(v.y), round_tf32(v.z), round_tf32(v.w));
}

// byte offset of element (r, k) in the K-major layout above
__device__ __forceinline__ uint32_t kmajor_off(int r, int k, int R) {
    return (uint32_t)(((k >> 2) * (R >> 3) + (r >> 3)) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

// byte offset of element (r, k) of a 16-bit K-major tile with R rows: core matrices of 8 rows x
// 8 elements (16 bytes), the same 128-byte blocks as above
__device__ __forceinline__ uint32_t kmajor_off16(int r, int k, int R) {
    return (uint32_t)(((k >> 3) * (R >> 3) + (r >> 3)) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

// 64-bit shared-memory matrix descriptor, no swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
    return d;                // base offset 0, legacy LBO mode, layout type 0 (no swizzle)
}

// ---- 128-byte swizzled tiles ------------------------------------------------
// A 16-bit tile with R rows (R a multiple of 8) and a column count that is a multiple of 64 is
// held as column blocks of 64 elements: block b is R rows of 128 bytes at b * R * 128, and inside
// an 8-row group the 16-byte chunk c of row r sits at chunk position c ^ (r % 8).  The tile must
// start on a 1024-byte boundary (the tensor core forms the XOR from address bits 7-9).  Writers
// that put 8 consecutive rows of one chunk, or one row's consecutive chunks, into a warp's lanes
// spread them over all 32 banks, so such stores run without bank conflicts.
//
// Read as a K-major operand (rows along M or N, columns along K): SBO = 1024 (next 8 rows), the
// 32-byte k-step s of a 64-wide block starts 32 s bytes into it.  Read as an MN-major operand
// (rows along K, columns along M or N): LBO = R * 128 (next 64 columns), SBO = 1024 (next 8 rows
// along K), a 16-deep k-step spans 2048 bytes.
__device__ __forceinline__ uint32_t sw128_off(int r, int k, int R) {
    return (uint32_t)((k >> 6) * (R * 128) + r * 128 + ((((k >> 3) & 7) ^ (r & 7)) << 4) + (k & 7) * 2);
}

__device__ __forceinline__ uint64_t make_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;  // layout type: 128-byte swizzle
    return d;
}

// K-major k-step `s` (16 fp16 along K) of a swizzled tile with R rows
__device__ __forceinline__ uint64_t desc_sw128_k(uint32_t base, int R, int s) {
    return make_desc_sw128(base + (uint32_t)(s >> 2) * (uint32_t)(R * 128) + (uint32_t)(s & 3) * 32, 16, 1024);
}

// A descriptor advanced by `bytes` (a multiple of 16): the start address is the low 14-bit field, in
// 16-byte units, and shared-memory addresses stay below 256 KB, so the sum never carries out of it.
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); }

// byte offset of k-step `s` (16 fp16) inside a K-major swizzled tile with R rows (see desc_sw128_k)
__host__ __device__ constexpr uint32_t sw128_kstep(int R, int s) {
    return (uint32_t)(s >> 2) * (uint32_t)(R * 128) + (uint32_t)(s & 3) * 32;
}

// MN-major k-step `s` (16 rows along K) of a swizzled tile with R rows
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t base, int R, int s) {
    return make_desc_sw128(base + (uint32_t)s * 2048, (uint32_t)(R * 128), 1024);
}

// descriptor of MMA k-step `s` (8 tf32 or 16 fp16 along K: 32 bytes) of a K-major tile with R rows
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int R, int s) {
    const uint32_t lbo = (uint32_t)(R >> 3) * 128;
    return make_desc(base + 2 * s * lbo, lbo, 128);
}

// descriptor of MMA k-step `s` (16 fp16 along K) of an MN-major operand held as a tile of R rows
// whose rows run along K (see the layout above): the step starts 16 rows (two core matrices) on
__device__ __forceinline__ uint64_t desc_mnmajor16(uint32_t base, int R, int s) {
    return make_desc(base + (uint32_t)s * 256, 128, (uint32_t)(R >> 3) * 128);
}
// instruction-descriptor bits: the A (bit 15) or B (bit 16) operand is MN-major (transposed)
constexpr uint32_t kTransposeA = 1u << 15;
constexpr uint32_t kTransposeB = 1u << 16;

// 32-bit instruction descriptor: kind::tf32, fp32 accumulate, shape M x N.
// Both operands K-major (bits 15 and 16 clear).
__device__ __forceinline__ constexpr uint32_t idesc_tf32(int M, int N) {
    return (1u << 4)                      // D format: f32
           | (2u << 7)                    // A format: tf32
           | (2u << 10)                   // B format: tf32
           | ((uint32_t)(N >> 3) << 17)
           | ((uint32_t)(M >> 4) << 24);
}

// 32-bit instruction descriptor: kind::f16 with fp16 A and B, fp32 accumulate, shape M x N,
// both operands K-major.  fp16 keeps tf32's 10-bit mantissa, so an operand rounded to fp16 is
// the value a tf32 operand would be, within fp16's range, at half the bytes and with 16 K per MMA.
__device__ __forceinline__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4)                      // D format: f32 (A, B format fields 0: f16)
           | ((uint32_t)(N >> 3) << 17)
           | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// 2^x with the hardware's approximate base-2 exponential (PTX ex2.approx.ftz.f32): one
// instruction; 2^-inf = +0 and results below the normal range flush to zero
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// two floats -> one 32-bit word of two fp16 (round to nearest even), low half first
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 unpack_f16(uint32_t w) {
    float2 f;
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(f.x), "=f"(f.y) : "r"(w));
    return f;
}

// The same MMA with the A operand in tensor memory: row m of A in lane m, two fp16 per 32-bit
// column with the even k in the low half, so a 16-deep k-step spans 8 columns (checked on B200
// against an fp64 product; the other half order gives garbage).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// Arrives on the mbarrier once every MMA this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// make generic-proxy shared-memory stores visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- TMEM allocation (one full warp) --------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- TMEM -> registers: 32 lanes x 32-bit, 16 consecutive columns ----------

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---- registers -> TMEM: 32 lanes x 32-bit, 16 consecutive columns -----------

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// One plain arrival on the mbarrier.
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// One arrival on the mbarrier that also expects `bytes` of async-copy traffic.
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}

// Asynchronous bulk copy global -> this CTA's shared memory (16-byte aligned
// addresses, size a multiple of 16), completing `bytes` on the mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// Asynchronous bulk copy of this CTA's shared memory -> global, in a bulk group.
__device__ __forceinline__ void bulk_s2g(void* gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
                 : "memory");
}
// Hint: bring `bytes` (multiple of 16, 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Per-thread asynchronous 16-byte copy global -> shared (both 16-byte aligned), cached in L2 only;
// cp_async_wait_all waits for every such copy this thread issued.
__device__ __forceinline__ void cp_async16(const void* sdst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// One non-blocking test of the phase with parity `parity` of the mbarrier.
__device__ __forceinline__ bool mbar_test(uint32_t mbar, uint32_t parity) {
    uint32_t done = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    return done != 0;
}

// Waits for the phase with parity `parity` of the mbarrier to complete.
// Gives up after `limit_ns` nanoseconds and returns false.  A phase that has already completed
// costs one test: the clock is read only once the wait is real.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, uint64_t limit_ns = 2000000000ull) {
    if (mbar_test(mbar, parity)) return true;
    uint32_t done = 0;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

}  // namespace tc
}  // namespace gdn

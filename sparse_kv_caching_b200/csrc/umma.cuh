// Thin wrappers over the sm_100a fifth-generation tensor-core instructions
// (tcgen05.*) and the mbarrier used to wait for them.
//
// Operand layout used everywhere in this library ("chunk-major", no swizzle):
// a tile of R rows x K columns is stored as K/T column chunks of R rows, each
// row chunk being 16 contiguous bytes (T = 8 bf16 or 4 f32 values):
//     byte offset of (row r, column k) = (k / T) * (R * 16) + r * 16 + (k % T) * esize
// Eight consecutive rows of one chunk form a contiguous 128-byte core matrix.
// Threads that write consecutive rows of one chunk write consecutive 16-byte
// words, so filling a tile from registers is free of bank conflicts.
//
// * As a K-major operand (rows = M or N, columns = K): leading byte offset
//   (next chunk along K) = R * 16, stride byte offset (next 8 rows) = 128.
// * As an MN-major operand (rows = K, columns = M or N): stride byte offset
//   (next chunk along M/N) = R * 16, leading byte offset (next 8 K rows) = 128.
// A K step of one MMA covers 2 chunks (32 bytes of K per row), so the K-major
// descriptor advances by 2 * R * 16 bytes per step and the MN-major one by
// 2 * 128 bytes (bf16, K = 16) or 128 bytes (tf32, K = 8).
#pragma once
#include <stdint.h>

namespace lola {
namespace umma {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Shared-memory matrix descriptor (tcgen05 format, no swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                       // descriptor version for sm_100
    return d;                                     // base offset 0, swizzle none
}

// The same descriptor for a 128-byte swizzled layout: 8-row atoms of 128-byte
// rows, 1024-byte aligned, in which the 16-byte chunk c of row r sits at chunk
// c ^ (r % 8).  K-major: sbo = stride between 8-row groups, lbo unused (the
// K extent of one MMA stays inside a row); a K step inside the row moves the
// start address by its byte offset.  MN-major: lbo = stride between 64-element
// (128-byte) blocks along M or N, sbo = stride between groups of 8 K rows.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return sdesc(saddr, lbo_bytes, sbo_bytes) | ((uint64_t)2 << 61);
}

// Byte offset of the 16-byte chunk c of row r inside a 128-byte swizzled tile
// whose rows are 128 bytes apart.
__host__ __device__ constexpr uint32_t sw128_off(uint32_t r, uint32_t c) {
    return r * 128u + (((c ^ r) & 7u) << 4);
}

enum Fmt : uint32_t { kF16 = 0, kBF16 = 1, kTF32 = 2 };

// Instruction descriptor: f32 accumulate, dense, no negation.
__host__ __device__ constexpr uint32_t idesc(uint32_t fmt, int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4)                              // D format f32
         | (fmt << 7) | (fmt << 10)               // A, B formats
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :: "r"(d_tmem), "l"(a), "l"(b), "r"(id), "r"(acc));
}
// kind::f16 serves both f16 and bf16 operands (A and B must have the same type).
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    mma_bf16(d_tmem, a, b, id, acc);
}
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
        :: "r"(d_tmem), "l"(a), "l"(b), "r"(id), "r"(acc));
}

// D[tmem] (+)= A[tmem] * B[smem] (tf32; A K-major in tensor memory: row m of A in
// lane m, one f32 element per column starting at column a_tmem).
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n"
        :: "r"(d_tmem), "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}

// D[tmem] (+)= A[tmem] * B[smem] with 16-bit operands (kind::f16: f16 or bf16 as
// the instruction descriptor says); A K-major in tensor memory: row m of A in lane
// m, two elements per 32-bit column (element 2 i in the low half of column i).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        :: "r"(d_tmem), "r"(a_tmem), "l"(b), "r"(id), "r"(acc));
}

// Arrive on an mbarrier once all previously issued MMAs of this thread complete.
__device__ __forceinline__ void commit(uint64_t* mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_addr(mbar)) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Make generic-proxy shared-memory writes visible to the tensor core.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// TMEM allocation (one full warp executes these).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_addr(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}

// 32 lanes x 16 columns of 32 bits: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t u[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
                   "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]),
                   "=r"(u[14]), "=r"(u[15])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&r)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "r"(__float_as_uint(r[0])), "r"(__float_as_uint(r[1])),
                    "r"(__float_as_uint(r[2])), "r"(__float_as_uint(r[3])), "r"(__float_as_uint(r[4])),
                    "r"(__float_as_uint(r[5])), "r"(__float_as_uint(r[6])), "r"(__float_as_uint(r[7])),
                    "r"(__float_as_uint(r[8])), "r"(__float_as_uint(r[9])), "r"(__float_as_uint(r[10])),
                    "r"(__float_as_uint(r[11])), "r"(__float_as_uint(r[12])), "r"(__float_as_uint(r[13])),
                    "r"(__float_as_uint(r[14])), "r"(__float_as_uint(r[15]))
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_addr(mbar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* mbar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(smem_addr(mbar)), "r"(phase) : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(mbar)) : "memory");
}

// Named barrier `id` over the first `nthreads` threads of the CTA (a warp-multiple),
// and its OR-reduction form.
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ bool named_sync_or(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, o;\n\t"
        "setp.ne.b32 q, %3, 0;\n\t"
        "bar.red.or.pred o, %1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, o;\n\t}\n"
        : "=r"(r) : "r"(id), "r"(nthreads), "r"(pred ? 1u : 0u) : "memory");
    return r != 0;
}

// Non-blocking test of the same condition: never suspends the thread, for a
// thread that polls several barriers in turn.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* mbar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok) : "r"(smem_addr(mbar)), "r"(phase) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait: returns false after `timeout_ns` of wall time (default 4 s),
// so a wait that can never end reports instead of hanging the GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, uint32_t phase,
                                          uint64_t timeout_ns = 4000000000ull) {
    if (mbar_try_wait(mbar, phase)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(mbar, phase))
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    return true;
}

// ---- 3xTF32 splitting ---------------------------------------------------------
// x = hi + lo with hi keeping the 10 explicit mantissa bits the tensor core
// reads (the low 13 bits of an f32 operand are ignored by kind::tf32); lo is
// exact in f32 and is itself read to tf32 precision.
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// ---- cp.async (16 bytes, L2 only) ---------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_addr(smem_dst)), "l"(gmem_src) : "memory");
}
// The same copy, or 16 zero bytes when !valid (src is then not read, but must still
// be a valid address).
__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gmem_src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(smem_addr(smem_dst)), "l"(gmem_src), "r"(valid ? 16u : 0u) : "memory");
}
// Arrive on an mbarrier once every cp.async this thread issued so far has landed
// (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* mbar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_addr(mbar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

}  // namespace umma
}  // namespace lola

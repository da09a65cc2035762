// Self-test of the tensor-core building blocks (umma.cuh): one CTA computes
// C[M x N] = A[M x K] * B with tcgen05.mma from the chunk-major shared-memory
// layouts the kernels use, the accumulator in TMEM, read back by tcgen05.ld.
// Modes: bit 0 = B is MN-major ([K][N] in global) rather than K-major
// ([N][K]); bit 1 = tf32 operands (f32 in global) rather than bf16; bit 2 =
// 3xTF32 (hi*hi + hi*lo + lo*hi, f32-accurate products); bit 3 = A is
// MN-major ([K][M] in global); bit 4 = A is read from tensor
// memory (stored there by tcgen05.st, K-major: one f32 per column for tf32,
// two bf16 per column otherwise); bit 5 = no MMA is
// issued and the completion wait gives up after about a millisecond (the
// bounded-wait failure path: *err is set, C is filled with NaN, the kernel
// frees its tensor memory and returns); bit 6 = operands in the 128-byte
// swizzled layout (128-byte rows, 8-row atoms) instead of chunk-major (tf32:
// K-major operands only); bit 7 = with bit 2, the hi parts in shared memory are
// the raw f32 values (not rounded down to tf32 first), to check that kind::tf32
// reads only their top 19 bits.
#include "device_common.cuh"
#include "umma.cuh"

namespace lola {

struct SelftestArgs {
    int mode, M, N, K;
    const void* A;
    const void* B;
    float* C;
    int* err;
};

// Copy a row-major [R][Kc] global matrix into the chunk-major tile (rows R).
template <typename T>
__device__ void fill_chunk_major(uint8_t* dst, const T* src, int R, int Kc, bool split_lo, bool split_hi) {
    constexpr int TPC = 16 / sizeof(T);           // elements per 16-byte chunk
    const int nchunks = R * (Kc / TPC);
    for (int idx = threadIdx.x; idx < nchunks; idx += blockDim.x) {
        const int r = idx % R, kc = idx / R;
        const T* s = src + (size_t)r * Kc + kc * TPC;
        T* d = reinterpret_cast<T*>(dst + (size_t)kc * R * 16 + (size_t)r * 16);
#pragma unroll
        for (int i = 0; i < TPC; ++i) {
            T x = s[i];
            if constexpr (sizeof(T) == 4) {
                if (split_hi) x = umma::tf32_hi(x);
                else if (split_lo) x = x - umma::tf32_hi(x);
            }
            d[i] = x;
        }
    }
}

// Copy a row-major [R][Kc] matrix into 128-byte swizzled blocks: block kb
// holds the kb-th 128 bytes of every row (64 bf16 or 32 f32), R rows of 128
// bytes; f32 may be split as for fill_chunk_major.
template <typename T>
__device__ void fill_sw128(uint8_t* dst, const T* src, int R, int Kc, bool split_lo = false, bool split_hi = false) {
    constexpr int TPC = 16 / sizeof(T), TPB = 128 / sizeof(T);
    const int nchunks = R * (Kc / TPC);
    for (int idx = threadIdx.x; idx < nchunks; idx += blockDim.x) {
        const int c = idx % 8, r = (idx / 8) % R, kb = idx / (8 * R);
        const T* s = src + (size_t)r * Kc + TPB * kb + TPC * c;
        T* d = reinterpret_cast<T*>(dst + (size_t)kb * R * 128 + umma::sw128_off(r, c));
#pragma unroll
        for (int i = 0; i < TPC; ++i) {
            T x = s[i];
            if constexpr (sizeof(T) == 4) {
                if (split_hi) x = umma::tf32_hi(x);
                else if (split_lo) x = x - umma::tf32_hi(x);
            }
            d[i] = x;
        }
    }
}

__global__ void __launch_bounds__(128, 1) umma_selftest_kernel(SelftestArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint64_t mbar;
    __shared__ uint32_t tbase;
    const bool bmn = a.mode & 1, tf32 = a.mode & 2, x3 = (a.mode & 4) && tf32;
    const bool amn = a.mode & 8, ats = a.mode & 16, expire = a.mode & 32;
    const bool sw = a.mode & 64;
    const bool rawhi = (a.mode & 128) && x3;                  // hi parts as raw f32
    const int M = a.M, N = a.N, K = a.K;
    const int es = tf32 ? 4 : 2;
    const size_t szA = (size_t)M * K * es, szB = (size_t)N * K * es;
    // swizzle atoms want a 1024-byte aligned base (the launch adds the slack)
    uint8_t* sA = smem + ((1024u - (umma::smem_addr(smem) & 1023u)) & 1023u);
    uint8_t* sB = smem + szA;
    uint8_t* sA2 = sB + szB;                       // lo parts (3xTF32)
    uint8_t* sB2 = sA2 + szA;
    const int warp = threadIdx.x >> 5;
    if (tf32) {
        const float* A = (const float*)a.A;
        const float* B = (const float*)a.B;
        if (sw) {    // K-major operands only
            if (!ats) {
                fill_sw128<float>(sA, A, M, K, false, x3 && !rawhi);
                if (x3) fill_sw128<float>(sA2, A, M, K, true, false);
            }
            fill_sw128<float>(sB, B, N, K, false, x3 && !rawhi);
            if (x3) fill_sw128<float>(sB2, B, N, K, true, false);
        } else if (amn) {   // A given as [K][M]: rows = K, chunks along M
            fill_chunk_major<float>(sA, A, K, M, false, x3);
            if (x3) fill_chunk_major<float>(sA2, A, K, M, true, false);
        } else if (!ats) {
            fill_chunk_major<float>(sA, A, M, K, false, x3 && !rawhi);
            if (x3) fill_chunk_major<float>(sA2, A, M, K, true, false);
        }
        if (sw) {
        } else if (bmn) {   // rows = K, chunks along N
            fill_chunk_major<float>(sB, B, K, N, false, x3);
            if (x3) fill_chunk_major<float>(sB2, B, K, N, true, false);
        } else {
            fill_chunk_major<float>(sB, B, N, K, false, x3 && !rawhi);
            if (x3) fill_chunk_major<float>(sB2, B, N, K, true, false);
        }
    } else if (sw) {
        if (amn) fill_sw128<__nv_bfloat16>(sA, (const __nv_bfloat16*)a.A, K, M);
        else fill_sw128<__nv_bfloat16>(sA, (const __nv_bfloat16*)a.A, M, K);
        if (bmn) fill_sw128<__nv_bfloat16>(sB, (const __nv_bfloat16*)a.B, K, N);
        else fill_sw128<__nv_bfloat16>(sB, (const __nv_bfloat16*)a.B, N, K);
    } else {
        if (amn) fill_chunk_major<__nv_bfloat16>(sA, (const __nv_bfloat16*)a.A, K, M, false, false);
        else fill_chunk_major<__nv_bfloat16>(sA, (const __nv_bfloat16*)a.A, M, K, false, false);
        if (bmn) fill_chunk_major<__nv_bfloat16>(sB, (const __nv_bfloat16*)a.B, K, N, false, false);
        else fill_chunk_major<__nv_bfloat16>(sB, (const __nv_bfloat16*)a.B, N, K, false, false);
    }
    umma::fence_async_smem();
    // accumulator columns [0, N); with A in tensor memory, A (hi) at column N and A_lo after it
    const int need_cols = N + (ats ? (tf32 ? K * (x3 ? 2 : 1) : K / 2) : 0);
    const uint32_t ncols = need_cols <= 32 ? 32 : need_cols <= 64 ? 64 : need_cols <= 128 ? 128
                         : need_cols <= 256 ? 256 : 512;
    if (warp == 0) umma::tmem_alloc(&tbase, ncols);
    if (threadIdx.x == 0) { umma::mbar_init(&mbar, 1); umma::fence_mbar_init(); }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = tbase;
    if (ats && !tf32) {
        // thread r of the 128 stores row r of A into lane r, two bf16 per column
        const uint16_t* A = (const uint16_t*)a.A;
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        for (int k0 = 0; k0 < K; k0 += 32) {
            float w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t lo = r < M ? A[(size_t)r * K + k0 + 2 * i] : 0u;
                const uint32_t hi = r < M ? A[(size_t)r * K + k0 + 2 * i + 1] : 0u;
                w[i] = __uint_as_float(lo | (hi << 16));
            }
            umma::tmem_st16(tmem + lane_off + N + k0 / 2, w);
        }
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncthreads();
        umma::fence_after_sync();
    } else if (ats) {
        // thread r of the 128 stores row r of A (and of A_lo) into lane r, one f32 per column
        const float* A = (const float*)a.A;
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        for (int k0 = 0; k0 < K; k0 += 16) {
            float hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float x = r < M ? A[(size_t)r * K + k0 + i] : 0.f;
                hi[i] = x3 ? umma::tf32_hi(x) : x;
                lo[i] = x - umma::tf32_hi(x);
            }
            umma::tmem_st16(tmem + lane_off + N + k0, hi);
            if (x3) umma::tmem_st16(tmem + lane_off + N + K + k0, lo);
        }
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncthreads();
        umma::fence_after_sync();
    }
    if (threadIdx.x == 0 && !expire) {
        const uint32_t id = umma::idesc(tf32 ? umma::kTF32 : umma::kBF16, M, N, amn, bmn);
        const int kstep = tf32 ? 8 : 16;
        const uint32_t a0 = umma::smem_addr(sA), b0 = umma::smem_addr(sB);
        const uint32_t a1 = umma::smem_addr(sA2), b1 = umma::smem_addr(sB2);
        const uint32_t lboA = amn ? 128 : M * 16, sboA = amn ? K * 16 : 128;
        const uint32_t lboB = bmn ? 128 : N * 16, sboB = bmn ? K * 16 : 128;
        const int passes = x3 ? 3 : 1;
        uint32_t acc = 0;
        for (int p = 0; p < passes; ++p) {
            const uint32_t abase = (p == 2) ? a1 : a0;   // pass 0: hi*hi, 1: hi*lo, 2: lo*hi
            const uint32_t bbase = (p == 1) ? b1 : b0;
            for (int ks = 0; ks < K / kstep; ++ks) {
                const uint32_t aoff = amn ? ks * kstep * 16 : ks * 2 * M * 16;
                const uint32_t boff = bmn ? ks * kstep * 16 : ks * 2 * N * 16;
                if (sw) {
                    // K-major: K steps of 32 bytes (16 bf16, 8 f32) inside a 128-byte block,
                    // blocks R x 128 bytes apart; MN-major (bf16): 16 K rows = two 1024-byte groups
                    const uint32_t ka = amn ? ks * 2048u : (ks / 4) * M * 128u + (ks % 4) * 32u;
                    const uint32_t kb = bmn ? ks * 2048u : (ks / 4) * N * 128u + (ks % 4) * 32u;
                    const uint64_t da = umma::sdesc_sw128(abase + ka, amn ? K * 128u : 16u, 1024u);
                    const uint64_t dbs = umma::sdesc_sw128(bbase + kb, bmn ? K * 128u : 16u, 1024u);
                    if (ats && tf32) umma::mma_tf32_ts(tmem, tmem + N + (p == 2 ? K : 0) + ks * kstep, dbs, id, acc);
                    else if (ats) umma::mma_f16_ts(tmem, tmem + N + ks * 8, dbs, id, acc);
                    else if (tf32) umma::mma_tf32(tmem, da, dbs, id, acc);
                    else umma::mma_bf16(tmem, da, dbs, id, acc);
                    acc = 1;
                    continue;
                }
                const uint64_t db = umma::sdesc(bbase + boff, lboB, sboB);
                if (ats && !tf32) {
                    umma::mma_f16_ts(tmem, tmem + N + ks * 8, db, id, acc);   // 16 bf16 = 8 columns
                } else if (ats) {
                    const uint32_t ta = tmem + N + (p == 2 ? K : 0) + ks * kstep;
                    umma::mma_tf32_ts(tmem, ta, db, id, acc);
                } else {
                    const uint64_t da = umma::sdesc(abase + aoff, lboA, sboA);
                    if (tf32) umma::mma_tf32(tmem, da, db, id, acc);
                    else umma::mma_bf16(tmem, da, db, id, acc);
                }
                acc = 1;
            }
        }
        umma::commit(&mbar);
    }
    const bool ok = umma::mbar_wait(&mbar, 0, expire ? 1000000ull : 4000000000ull);
    if (!ok && threadIdx.x == 0) atomicExch(a.err, 1);
    umma::fence_after_sync();
    const int row = 32 * (warp & 3) + (threadIdx.x & 31);
    for (int c0 = 0; c0 < N; c0 += 16) {
        float r[16];
        umma::tmem_ld16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + c0, r);
        umma::tmem_wait_ld();
        if (row < M)
            for (int i = 0; i < 16; ++i) a.C[(size_t)row * N + c0 + i] = ok ? r[i] : __int_as_float(0x7fc00000);
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, ncols);
}

size_t selftest_smem(int mode, int M, int N, int K) {
    const bool tf32 = mode & 2, x3 = (mode & 4) && tf32;
    const size_t es = tf32 ? 4 : 2;
    size_t b = (size_t)M * K * es + (size_t)N * K * es;
    return (x3 ? 2 * b : b) + 1024;   // + alignment slack of the operand base
}

int selftest_tmem_cols(int mode, int N, int K) {
    const bool tf32 = mode & 2, x3 = (mode & 4) && tf32, ats = mode & 16;
    return N + (ats ? (tf32 ? K * (x3 ? 2 : 1) : K / 2) : 0);
}

cudaError_t launch_selftest(int mode, const void* A, const void* B, float* C, int M, int N, int K, int* err,
                            cudaStream_t s) {
    const size_t bytes = selftest_smem(mode, M, N, K);
    cudaError_t e = cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
    if (e != cudaSuccess) return e;
    SelftestArgs a{mode, M, N, K, A, B, C, err};
    umma_selftest_kernel<<<1, 128, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lola

// Device helpers shared by the LoLA kernels: element loads, warp/block
// reductions and scans, where a KV pair lives, and the fused SRE scorer.
#pragma once
#include "lola_internal.h"

namespace lola {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Load 4 consecutive elements as float4 (p must be 4-element aligned).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    float4 r;
    r.x = __uint_as_float(u.x << 16);
    r.y = __uint_as_float(u.x & 0xFFFF0000u);
    r.z = __uint_as_float(u.y << 16);
    r.w = __uint_as_float(u.y & 0xFFFF0000u);
    return r;
}
// Load 2 consecutive elements as float2.
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Two IEEE fp32 fused multiply-adds in one sm_100 instruction: lane-wise
// d = a * b + c on pairs of floats packed in 64-bit registers.
__device__ __forceinline__ unsigned long long f2pack(float x, float y) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
    return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long r, float& x, float& y) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(r));
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// One query's term of an alternative scoring rule (LoLA notes §4.5, Table 4;
// App. F): a = exp(q.k / sqrt(d)), f = phi(q)^T phi(k).
// rule 1: (a - f)^2, 2: |a - f|, 3: f / a, 4: a.
__device__ __forceinline__ float window_term(int rule, float a, float f) {
    switch (rule) {
        case 1: { const float x = a - f; return x * x; }
        case 2: return fabsf(a - f);
        case 3: return f / a;
        default: return a;
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Exclusive prefix sum of in[0, n) into out[0, n) by the whole block
// (blockDim.x a multiple of 32, at most 1024); returns the total.  `tmp`
// holds >= 32 ints.
__device__ inline int block_exscan(const int* in, int* out, int n, int* tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NT = blockDim.x;
    const int per = (n + NT - 1) / NT;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += in[i];
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    const int NW = NT / 32;
    if (warp == 0) {
        int w = lane < NW ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        tmp[lane] = w;
    }
    __syncthreads();
    int base = (warp ? tmp[warp - 1] : 0) + x - sum;
    for (int i = lo; i < hi; ++i) { out[i] = base; base += in[i]; }
    const int total = tmp[NW - 1];
    __syncthreads();
    return total;
}

// Where the pair at position p lives during a prefill call (see lola_internal.h).
// `slot` is its cache slot when it is a cache member that predates the call.
template <typename TIn>
struct PairRef { const TIn* k; const TIn* v; const float* phik; };

template <typename TIn>
__device__ __forceinline__ PairRef<TIn> pair_ref(const PrefillArgs& a, int st, int b, int g, int p, int slot) {
    const Dims& dm = a.dm;
    PairRef<TIn> r;
    if (p >= a.t_start) {
        const size_t i = (size_t)(p - a.t_start);
        const size_t off = (((size_t)b * a.T + i) * dm.Hkv + g) * dm.d;
        r.k = (const TIn*)a.k + off;
        r.v = (const TIn*)a.v + off;
        r.phik = a.phik_new + ((size_t)st * dm.max_tokens + i) * dm.D;
    } else if (p >= a.t_start - dm.eta) {
        const size_t w = (size_t)st * dm.eta + (size_t)(p % dm.eta);
        r.k = (const TIn*)a.sp.win_k + w * dm.d;
        r.v = (const TIn*)a.sp.win_v + w * dm.d;
        r.phik = a.sp.win_phik + w * dm.D;
    } else {
        const size_t c = (size_t)st * dm.lam + (size_t)slot;
        r.k = (const TIn*)a.sp.cache_k + c * dm.d;
        r.v = (const TIn*)a.sp.cache_v + c * dm.d;
        r.phik = a.sp.cache_phik + c * dm.D;
    }
    return r;
}

// Fused Self-Recall Error of up to TE candidates against (H, s) in shared memory
// (notes §2.3, Eq. 10, squared): score_e = || H^T phi_e / (phi_e^T s) - v_e ||^2,
// with the zero prediction when phi_e^T s == 0.  fp32 FFMA throughout.
//
//   Hs   [D][DV] f32 (smem)     ss [D] f32 (smem)
//   tile [TE][D+4] f32 (smem)   phi rows of the candidates, already loaded
//   den  [TE] f32 (smem)        scratch
//   vrow(e) -> pointer to the candidate's value row (global, TIn)
//   out[e] receives the score of candidate e (e < ne)
// The thread block has kThreads threads.  Thread (ty, tx) owns output columns
// 4tx..4tx+3 of EPT candidates ty, ty+TY, ...
template <int D, int DV, typename TIn>
struct SreShape {
    static constexpr int TX = DV / 4;
    static constexpr int TY = kThreads / TX;
    static constexpr int EPT = 8;
    static constexpr int TE = TY * EPT;
    static constexpr int LD = D + 4;     // padded phi-row stride (floats)
};

template <int D, int DV, typename TIn, typename VRow>
__device__ __forceinline__ void sre_tile(const float* __restrict__ Hs, const float* __restrict__ ss,
                                         const float* __restrict__ tile, float* __restrict__ den,
                                         int ne, VRow vrow, float* __restrict__ out) {
    using Sh = SreShape<D, DV, TIn>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // den_e = phi_e . s  (one warp per candidate)
    for (int e = warp; e < ne; e += kThreads / 32) {
        float x = 0.f;
        for (int j = lane; j < D; j += 32) x = fmaf(tile[e * Sh::LD + j], ss[j], x);
        x = warp_sum(x);
        if (lane == 0) den[e] = x;
    }
    __syncthreads();
    const int tx = tid % Sh::TX, ty = tid / Sh::TX;
    float acc[Sh::EPT][4];
#pragma unroll
    for (int i = 0; i < Sh::EPT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    const float4* H4 = reinterpret_cast<const float4*>(Hs);
#pragma unroll 2
    for (int j = 0; j < D; j += 4) {
        const float4 h0 = H4[(j + 0) * (DV / 4) + tx];
        const float4 h1 = H4[(j + 1) * (DV / 4) + tx];
        const float4 h2 = H4[(j + 2) * (DV / 4) + tx];
        const float4 h3 = H4[(j + 3) * (DV / 4) + tx];
#pragma unroll
        for (int i = 0; i < Sh::EPT; ++i) {
            const int e = ty + i * Sh::TY;
            const float4 f = *reinterpret_cast<const float4*>(tile + e * Sh::LD + j);
            acc[i][0] = fmaf(f.x, h0.x, acc[i][0]); acc[i][1] = fmaf(f.x, h0.y, acc[i][1]);
            acc[i][2] = fmaf(f.x, h0.z, acc[i][2]); acc[i][3] = fmaf(f.x, h0.w, acc[i][3]);
            acc[i][0] = fmaf(f.y, h1.x, acc[i][0]); acc[i][1] = fmaf(f.y, h1.y, acc[i][1]);
            acc[i][2] = fmaf(f.y, h1.z, acc[i][2]); acc[i][3] = fmaf(f.y, h1.w, acc[i][3]);
            acc[i][0] = fmaf(f.z, h2.x, acc[i][0]); acc[i][1] = fmaf(f.z, h2.y, acc[i][1]);
            acc[i][2] = fmaf(f.z, h2.z, acc[i][2]); acc[i][3] = fmaf(f.z, h2.w, acc[i][3]);
            acc[i][0] = fmaf(f.w, h3.x, acc[i][0]); acc[i][1] = fmaf(f.w, h3.y, acc[i][1]);
            acc[i][2] = fmaf(f.w, h3.z, acc[i][2]); acc[i][3] = fmaf(f.w, h3.w, acc[i][3]);
        }
    }
#pragma unroll
    for (int i = 0; i < Sh::EPT; ++i) {
        const int e = ty + i * Sh::TY;
        float part = 0.f;
        if (e < ne) {
            const float dn = den[e];
            const float4 vv = load4(vrow(e) + 4 * tx);
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
            if (dn > 0.f) { p0 = acc[i][0] / dn; p1 = acc[i][1] / dn; p2 = acc[i][2] / dn; p3 = acc[i][3] / dn; }
            const float r0 = p0 - vv.x, r1 = p1 - vv.y, r2 = p2 - vv.z, r3 = p3 - vv.w;
            part = r0 * r0 + r1 * r1 + r2 * r2 + r3 * r3;
        }
#pragma unroll
        for (int o = Sh::TX / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (tx == 0 && e < ne) out[e] = part;
    }
    (void)lane;
    __syncthreads();
}

// Load phi rows of ne candidates into tile [ne][D+4] (phirow(e) -> global f32 pointer).
template <int D, typename PhiRow>
__device__ __forceinline__ void load_phi_tile(float* tile, int ne, PhiRow phirow) {
    constexpr int LD = D + 4;
    constexpr int Q = D / 4;
    for (int idx = threadIdx.x; idx < ne * Q; idx += kThreads) {
        const int e = idx / Q, j = (idx % Q) * 4;
        *reinterpret_cast<float4*>(tile + e * LD + j) = *reinterpret_cast<const float4*>(phirow(e) + j);
    }
}

}  // namespace lola

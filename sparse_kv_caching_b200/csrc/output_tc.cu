// Hybrid output of chunkwise LoLA prefill on the fifth-generation tensor cores
// (bf16 inputs).  Same computation as output.cu (notes §2.5 Eq. 14, §2.6):
//   y_t = (H_c^T phi(q_t) + sum_i e^{a_ti} v_i) / (phi(q_t)^T s_c + sum_i e^{a_ti})
// over i in G_c u W_c u {block keys <= t}, with one shared normaliser.
//
// One CTA serves 128 query rows (row = (head of the kv group, query of block
// c)); all of them read the same gathered keys.  Four warps; thread r owns
// row r for the softmax.  Tensor memory holds O [128 x d] f32 and S [128 x 64].
//   prologue: z = Q W_g (bf16 MMA) -> phi(q) = [softmax(z), softmax(-z)] in
//             registers -> O = phi(q) H_c (tf32 MMA, 4 K-chunks), l = phi(q).s_c
//             (the linear branch is the accumulator's initial value, logit 0)
//   per 64-key tile (double-buffered cp.async gather of K and V rows):
//             S = Q K^T (bf16 MMA) -> row max / exp2 in registers (log2 domain,
//             the reference maximum is raised lazily when a row's maximum
//             exceeds it by more than 8) -> P (f16) -> O += P V (f16 MMA; the V
//             tile is converted bf16 -> f16 in shared memory while S is computed)
//   epilogue: y = O / l.
#include "device_common.cuh"
#include "umma.cuh"

namespace lola {

template <int DIM, int DH>
struct TcShape {
    static constexpr int ROWS = 128, KT = 64, D = 2 * DH, NCH = DIM / 8;
    static constexpr int KVB = KT * DIM * 2;                  // one K or V tile (bytes)
    static constexpr int Q = 0;
    static constexpr int KV = Q + ROWS * DIM * 2;             // [2 buffers][K, V]
    static constexpr int P = KV + 4 * KVB;                    // P [128 x 64] f16; W in the prologue
    static constexpr int KPOS = P + ROWS * KT * 2;            // [2][KT] int
    static constexpr int MBAR = KPOS + 2 * KT * 4;
    static constexpr int TPTR = MBAR + 16;
    static constexpr int total = TPTR + 16;
    // prologue aliases: all D/32 chunks of H_c^T in the KV region, the phi(q) chunk
    // in the P region (after W has served the z product), s_c in the KPOS region
    static constexpr int HT = KV;                             // [D/32][DIM rows x 32 j] f32
    static constexpr int HTC = DIM * 32 * 4;                  // one chunk (bytes)
    static constexpr int PHI = P;                             // [128 rows x 32 j] f32
    static constexpr int SC = KPOS;                           // s_c [D] f32
    static constexpr int TMEM_COLS = (DIM + KT <= 128) ? 128 : 256;
    static_assert(HT + (D / 32) * HTC <= P, "H_c^T must fit in the KV region");
    static_assert(ROWS * 32 * 4 <= ROWS * KT * 2, "a phi chunk must fit in the P region");
    static_assert(D * 4 <= 2 * KT * 4, "s_c must fit in the KPOS region");
    static_assert(DIM * DH * 2 <= ROWS * KT * 2, "W must fit in the P region");
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" :: "r"(umma::smem_addr(p)), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t u) {
    return __half22float2(*reinterpret_cast<__half2*>(&u));
}
// Two bf16 values (one 32-bit word) -> two f16 values (exact for |x| < 65504).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u) {
    return pack_f16(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

template <int DIM, int DH>
__global__ void __launch_bounds__(128, 2) output_tc_kernel(const __grid_constant__ PrefillArgs a) {
    using Sh = TcShape<DIM, DH>;
    using bf16 = __nv_bfloat16;
    constexpr int ROWS = Sh::ROWS, KT = Sh::KT, D = Sh::D, NCH = Sh::NCH;
    extern __shared__ __align__(1024) uint8_t smem[];
    const Dims& dm = a.dm;
    const int rows_total = dm.Gq * dm.C;
    const int nrb = (rows_total + ROWS - 1) / ROWS;
    const int c = a.c_begin + (int)blockIdx.x / nrb, rb = blockIdx.x % nrb;
    const int g = blockIdx.y, b = blockIdx.z, st = b * dm.Hkv + g;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int t0 = a.t_start + c * dm.C;
    const int R = rb * ROWS + tid;
    const bool row_ok = R < rows_total;
    const int hh = row_ok ? R / dm.C : 0, qi = row_ok ? R % dm.C : 0;
    const int qpos = t0 + qi, h = g * dm.Gq + hh;
    const int rfirst = rb * ROWS, rlast = min(rows_total, rfirst + ROWS) - 1;
    const int qi_max = (rlast / dm.C != rfirst / dm.C) ? dm.C - 1 : rlast % dm.C;

    uint8_t* sQ = smem + Sh::Q;
    uint8_t* sKV = smem + Sh::KV;
    uint8_t* sP = smem + Sh::P;
    int* kpos = reinterpret_cast<int*>(smem + Sh::KPOS);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + Sh::MBAR);
    uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + Sh::TPTR);
    const size_t snaps = (size_t)dm.nc_max + 1;
    // something was folded before block c, and the state branch is read
    const bool has_lin = (t0 - dm.eta) > dm.lam && !(a.read_mask & 1);

    if (warp == 0) umma::tmem_alloc(tptr, Sh::TMEM_COLS);
    if (tid == 0) { umma::mbar_init(&mbar[0], 1); umma::mbar_init(&mbar[1], 1); umma::fence_mbar_init(); }

    // ---- queries (row-chunk mapping: 8 rows x 4 chunks per warp instruction) ----
    for (int idx = tid; idx < ROWS * NCH; idx += 128) {
        const int r = (idx & 7) + 8 * (idx / (8 * NCH)), j = (idx >> 3) % NCH;
        uint8_t* dst = sQ + j * ROWS * 16 + r * 16;
        const int Rr = rfirst + r;
        if (Rr < rows_total) {
            const int hr = g * dm.Gq + Rr / dm.C, ir = Rr % dm.C;
            umma::cp_async16(dst, (const bf16*)a.q + (((size_t)b * a.T + (t0 + ir - a.t_start)) * dm.Hq + hr) * DIM + 8 * j);
        } else {
            st_shared_v4(dst, 0u, 0u, 0u, 0u);
        }
    }
    const float* Hc = a.snap_H + ((size_t)st * snaps + c) * D * DIM;     // H_c^T [DIM][D]
    const float* sc_g = a.snap_s + ((size_t)st * snaps + c) * D;
    float* s_c = reinterpret_cast<float*>(smem + Sh::SC);
    if (has_lin) {
        const bf16* Wg = (const bf16*)a.sp.W + (size_t)g * DIM * DH;  // [DIM][DH]; MN-major B
        for (int idx = tid; idx < DIM * (DH / 8); idx += 128) {
            const int k = idx % DIM, n8 = idx / DIM;
            umma::cp_async16(sP + n8 * DIM * 16 + k * 16, Wg + (size_t)k * DH + 8 * n8);
        }
        for (int idx = tid; idx < D / 4; idx += 128) umma::cp_async16(s_c + 4 * idx, sc_g + 4 * idx);
        // every chunk of H_c^T at once: rows cc of 32 j each, 8 groups of 4 j
        for (int idx = tid; idx < (D / 32) * DIM * 8; idx += 128) {
            const int cc = idx % DIM, jq = (idx / DIM) % 8, ch = idx / (DIM * 8);
            umma::cp_async16(smem + Sh::HT + ch * Sh::HTC + jq * DIM * 16 + cc * 16, Hc + (size_t)cc * D + 32 * ch + 4 * jq);
        }
    }
    umma::cp_async_commit();
    umma::cp_async_wait<0>();
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tptr;
    const uint32_t tO = tmem, tS = tmem + DIM;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    uint32_t ph0 = 0, ph1 = 0;
    bool ok = true;
    float l = 0.f;

    // ---- linear branch ----
    if (has_lin) {
        if (tid == 0) {
            const uint32_t id = umma::idesc(umma::kBF16, ROWS, DH, false, true);
            for (int ks = 0; ks < DIM / 16; ++ks)
                umma::mma_bf16(tS, umma::sdesc(umma::smem_addr(sQ) + ks * 2 * ROWS * 16, ROWS * 16, 128),
                               umma::sdesc(umma::smem_addr(sP) + ks * 16 * 16, 128, DIM * 16), id, ks > 0);
            umma::commit(&mbar[0]);
        }
        ok &= umma::mbar_wait(&mbar[0], ph0); ph0 ^= 1;
        umma::fence_after_sync();
        float z[DH];
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 16) {
            float r16[16];
            umma::tmem_ld16(tS + lane_off + c0, r16);
            umma::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) z[c0 + i] = r16[i];
        }
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int i = 0; i < DH; ++i) { mx = fmaxf(mx, z[i]); mn = fminf(mn, z[i]); }
        float sp = 0.f, sn = 0.f;
#pragma unroll
        for (int i = 0; i < DH; ++i) { sp += expf(z[i] - mx); sn += expf(mn - z[i]); }
        const float isp = 1.f / sp, isn = 1.f / sn;
        uint8_t* sPhi = smem + Sh::PHI;
#pragma unroll
        for (int jc = 0; jc < D; jc += 32) {
            uint8_t* sHt = smem + Sh::HT + (jc / 32) * Sh::HTC;
#pragma unroll
            for (int jq = 0; jq < 8; ++jq) {
                float f[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = jc + 4 * jq + u;
                    f[u] = j < DH ? expf(z[j] - mx) * isp : expf(mn - z[j - DH]) * isn;
                    l = fmaf(f[u], s_c[j], l);
                }
                st_shared_v4(sPhi + jq * ROWS * 16 + tid * 16, __float_as_uint(f[0]), __float_as_uint(f[1]),
                             __float_as_uint(f[2]), __float_as_uint(f[3]));
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncthreads();
            umma::fence_after_sync();
            if (tid == 0) {
                const uint32_t id = umma::idesc(umma::kTF32, ROWS, DIM, false, false);
                for (int ks = 0; ks < 4; ++ks)
                    umma::mma_tf32(tO, umma::sdesc(umma::smem_addr(sPhi) + ks * 2 * ROWS * 16, ROWS * 16, 128),
                                   umma::sdesc(umma::smem_addr(sHt) + ks * 2 * DIM * 16, DIM * 16, 128), id,
                                   (jc > 0 || ks > 0) ? 1u : 0u);
                umma::commit(&mbar[0]);
            }
            ok &= umma::mbar_wait(&mbar[0], ph0); ph0 ^= 1;
            umma::fence_after_sync();
        }
        if (!row_ok) l = 0.f;
    }

    // ---- exact keys: cache slots, window, block keys up to the last query of the CTA ----
    const int n_g = (a.read_mask & 2) ? 0 : min(dm.lam, max(0, t0 - dm.eta));
    const int w_lo = max(0, t0 - dm.eta);
    const int n_w = t0 - w_lo;
    const int N = n_g + n_w + qi_max + 1;
    const int ntiles = (N + KT - 1) / KT;
    const int* cpos = a.snap_pos + ((size_t)st * snaps + c) * dm.lam;
    // positions of a tile's keys, one thread per key (one load per cache key, all
    // in parallel); the copies then read them from shared memory
    auto stage_pos = [&](int it, int buf) {
        if (tid < KT) {
            const int gk = it * KT + tid;
            int pos = 0x7fffffff;
            if (gk < n_g) pos = cpos[gk];
            else if (gk < n_g + n_w) pos = w_lo + (gk - n_g);
            else if (gk < N) pos = t0 + (gk - n_g - n_w);
            kpos[buf * KT + tid] = pos;
        }
    };
    auto issue_tile = [&](int it, int buf) {
        uint8_t* sK = sKV + buf * 2 * Sh::KVB;
        uint8_t* sV = sK + Sh::KVB;
        const int k0 = it * KT;
        for (int idx = tid; idx < KT * NCH; idx += 128) {
            const int kk = (idx & 7) + 8 * (idx / (8 * NCH)), j = (idx >> 3) % NCH;
            const int gk = k0 + kk;
            uint8_t* dk = sK + j * KT * 16 + kk * 16;
            uint8_t* dv = sV + j * KT * 16 + kk * 16;
            if (gk < N) {
                const PairRef<bf16> r = pair_ref<bf16>(a, st, b, g, kpos[buf * KT + kk], gk < n_g ? gk : 0);
                umma::cp_async16(dk, r.k + 8 * j);
                umma::cp_async16(dv, r.v + 8 * j);
            } else {
                st_shared_v4(dk, 0u, 0u, 0u, 0u);
                st_shared_v4(dv, 0u, 0u, 0u, 0u);
            }
        }
        umma::cp_async_commit();
    };
    const float c2 = 1.4426950408889634f / sqrtf((float)DIM);   // log2(e) / sqrt(d)
    float m_ref = 0.f;
    stage_pos(0, 0);
    __syncthreads();
    issue_tile(0, 0);
    for (int it = 0; it < ntiles; ++it) {
        const int buf = it & 1;
        if (it + 1 < ntiles) {
            stage_pos(it + 1, buf ^ 1);            // buffer buf^1 was last read by tile it-1
            __syncthreads();
            issue_tile(it + 1, buf ^ 1);
            umma::cp_async_wait<1>();
        } else {
            umma::cp_async_wait<0>();
        }
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        umma::fence_after_sync();
        const uint8_t* sK = sKV + buf * 2 * Sh::KVB;
        uint8_t* sV = sKV + buf * 2 * Sh::KVB + Sh::KVB;
        if (tid == 0) {
            const uint32_t id = umma::idesc(umma::kBF16, ROWS, KT, false, false);
            for (int ks = 0; ks < DIM / 16; ++ks)
                umma::mma_bf16(tS, umma::sdesc(umma::smem_addr(sQ) + ks * 2 * ROWS * 16, ROWS * 16, 128),
                               umma::sdesc(umma::smem_addr(sK) + ks * 2 * KT * 16, KT * 16, 128), id, ks > 0);
            umma::commit(&mbar[0]);
        }
        // While S = Q K^T runs: V tile bf16 -> f16 in place (the P V product runs in f16 so that
        // the weights P keep 10 mantissa bits).  All copies landed before the barrier above.
        for (int idx = tid; idx < KT * NCH; idx += 128) {
            uint4* pv = reinterpret_cast<uint4*>(sV + idx * 16);
            uint4 u = *pv;
            u.x = bf16x2_to_f16x2(u.x); u.y = bf16x2_to_f16x2(u.y);
            u.z = bf16x2_to_f16x2(u.z); u.w = bf16x2_to_f16x2(u.w);
            *pv = u;
        }
        ok &= umma::mbar_wait(&mbar[0], ph0); ph0 ^= 1;
        umma::fence_after_sync();
        float s[KT];
#pragma unroll
        for (int c0 = 0; c0 < KT; c0 += 16) {
            float r16[16];
            umma::tmem_ld16(tS + lane_off + c0, r16);
            umma::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) s[c0 + i] = r16[i];
        }
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < KT; ++i) {
            const bool vis = row_ok && kpos[buf * KT + i] <= qpos;
            s[i] = vis ? s[i] * c2 : -INFINITY;
            mx = fmaxf(mx, s[i]);
        }
        float factor = 1.f;
        bool rescale = false;
        if (mx != -INFINITY) {
            if (l == 0.f) m_ref = mx;                         // nothing accumulated yet
            else if (mx > m_ref + 8.f) { factor = ex2(m_ref - mx); rescale = true; m_ref = mx; }
        }
        if (__any_sync(0xffffffffu, rescale)) {                // warp-collective TMEM access
            l *= factor;
#pragma unroll
            for (int c0 = 0; c0 < DIM; c0 += 16) {
                float r16[16];
                umma::tmem_ld16(tO + lane_off + c0, r16);
                umma::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) r16[i] *= factor;
                umma::tmem_st16(tO + lane_off + c0, r16);
            }
            umma::tmem_wait_st();
        }
        // The normaliser sums the f16-rounded weights that the PV product uses, so
        // y is an exact convex combination of those weights.
        float rs = 0.f;
#pragma unroll
        for (int ch = 0; ch < KT / 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                w[u] = pack_f16(ex2(s[8 * ch + 2 * u] - m_ref), ex2(s[8 * ch + 2 * u + 1] - m_ref));
                const float2 r2 = unpack_f16(w[u]);
                rs += r2.x + r2.y;
            }
            st_shared_v4(sP + ch * ROWS * 16 + tid * 16, w[0], w[1], w[2], w[3]);
        }
        l += rs;
        umma::fence_async_smem();
        umma::fence_before_sync();
        __syncthreads();
        umma::fence_after_sync();
        if (tid == 0) {
            const uint32_t id = umma::idesc(umma::kF16, ROWS, DIM, false, true);
            for (int ks = 0; ks < KT / 16; ++ks)
                umma::mma_f16(tO, umma::sdesc(umma::smem_addr(sP) + ks * 2 * ROWS * 16, ROWS * 16, 128),
                               umma::sdesc(umma::smem_addr(sV) + ks * 16 * 16, 128, KT * 16), id,
                               (has_lin || it > 0 || ks > 0) ? 1u : 0u);
            umma::commit(&mbar[1]);
        }
        ok &= umma::mbar_wait(&mbar[1], ph1); ph1 ^= 1;
        umma::fence_after_sync();
    }

    // ---- epilogue: y = O / l ----
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* yrow = a.y + (((size_t)b * a.T + (qpos - a.t_start)) * dm.Hq + h) * DIM;
#pragma unroll
    for (int c0 = 0; c0 < DIM; c0 += 16) {
        float r16[16];
        umma::tmem_ld16(tO + lane_off + c0, r16);
        umma::tmem_wait_ld();
        if (row_ok) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(yrow + c0 + i) =
                    make_float4(r16[i] * inv, r16[i + 1] * inv, r16[i + 2] * inv, r16[i + 3] * inv);
        }
    }
    if (!ok && a.err) atomicOr(a.err, 1);
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, Sh::TMEM_COLS);
}

template <int DIM, int DH>
static cudaError_t launch_tc_t(const PrefillArgs& a, cudaStream_t s) {
    using Sh = TcShape<DIM, DH>;
    cudaError_t e = cudaFuncSetAttribute(output_tc_kernel<DIM, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Sh::total);
    if (e != cudaSuccess) return e;
    const int nrb = (a.dm.Gq * a.dm.C + Sh::ROWS - 1) / Sh::ROWS;
    dim3 grid((a.c_end - a.c_begin) * nrb, a.dm.Hkv, a.dm.B);
    output_tc_kernel<DIM, DH><<<grid, 128, Sh::total, s>>>(a);
    return cudaGetLastError();
}

// bf16 inputs on the tensor-core kernel; returns cudaErrorNotSupported for shapes it does not cover.
cudaError_t launch_output_tc(const PrefillArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (a.dm.dtype != 1) return cudaErrorNotSupported;
    {
        const cudaError_t e = launch_output_ws(a, s);
        if (e != cudaErrorNotSupported) return e;
    }
    if (d == 128 && Dh == 64) return launch_tc_t<128, 64>(a, s);
    if (d == 128 && Dh == 32) return launch_tc_t<128, 32>(a, s);
    if (d == 64 && Dh == 32) return launch_tc_t<64, 32>(a, s);
    if (d == 64 && Dh == 64) return launch_tc_t<64, 64>(a, s);
    return cudaErrorNotSupported;
}

}  // namespace lola

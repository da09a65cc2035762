// Hybrid output of chunkwise LoLA prefill (notes §2.5, Eq. 14; §2.6, Fig. 2):
//   y_t = (H_c^T phi(q_t) + sum_{i in G_c u W_c u chunk<=t} e^{a_ti} v_i)
//       / (phi(q_t)^T s_c + sum e^{a_ti}),   a_ti = q_t . k_i / sqrt(d)
// with (G_c, H_c, s_c) the memories entering block c (published by the scan)
// and W_c the eta pairs preceding the block.  One shared normaliser: the
// linear branch enters the online softmax as the initial accumulator with
// logit 0, so the running maximum m rescales it like every exact key
// (e^{-m} H^T phi, e^{-m} phi^T s).  Blocks are independent once published:
// one CTA per (32 queries of a block, query head, sequence).  fp32 FFMA.
#include "device_common.cuh"

namespace lola {

template <int DIM, int DH>
struct OutShape {
    static constexpr int QB = 32, KT = 64, D = 2 * DH, CPL = DIM / 32, QPW = 4;
    static constexpr int LDK = KT + 1;
    // smem words
    static constexpr int Qs = 0, Ph = Qs + QB * DIM, Kt = Ph + QB * D, Vs = Kt + DIM * LDK,
                         Kp = Vs + KT * DIM, total = Kp + KT;
};

template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(256) output_kernel(const __grid_constant__ PrefillArgs a) {
    using Sh = OutShape<DIM, DH>;
    constexpr int QB = Sh::QB, KT = Sh::KT, D = Sh::D, CPL = Sh::CPL, QPW = Sh::QPW, LDK = Sh::LDK;
    extern __shared__ __align__(16) float smem[];
    float* Qs = smem + Sh::Qs;
    float* Ph = smem + Sh::Ph;
    float* Kt = smem + Sh::Kt;
    float* Vs = smem + Sh::Vs;
    int* Kp = reinterpret_cast<int*>(smem + Sh::Kp);
    float* Ws = Kt;                                   // W is only needed before the key loop
    const Dims& dm = a.dm;
    const int nqb = (dm.C + QB - 1) / QB;
    const int c = a.c_begin + (int)blockIdx.x / nqb, qb = blockIdx.x % nqb;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / dm.Gq, st = b * dm.Hkv + g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = a.t_start + c * dm.C;
    const int nq = min(QB, dm.C - qb * QB);
    const int qlo = t0 + qb * QB;                    // position of the first query

    // queries and W_g
    for (int idx = tid; idx < QB * DIM / 4; idx += 256) {
        const int r = idx / (DIM / 4), j = (idx % (DIM / 4)) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < nq) {
            const size_t i = (size_t)(qlo + r - a.t_start);
            x = load4((const TIn*)a.q + (((size_t)b * a.T + i) * dm.Hq + h) * DIM + j);
        }
        *reinterpret_cast<float4*>(Qs + r * DIM + j) = x;
    }
    const TIn* Wg = (const TIn*)a.sp.W + (size_t)g * DIM * DH;
    for (int i = tid; i < DIM * DH; i += 256) Ws[i] = to_f32(Wg[i]);
    __syncthreads();

    // phi(q) for the warp's queries
    for (int qq = 0; qq < QPW; ++qq) {
        const int r = warp * QPW + qq;
        float z[DH / 32];
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) z[u] = 0.f;
        for (int j = 0; j < DIM; ++j) {
            const float xj = Qs[r * DIM + j];
#pragma unroll
            for (int u = 0; u < DH / 32; ++u) z[u] = fmaf(xj, Ws[j * DH + lane + 32 * u], z[u]);
        }
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) { mx = fmaxf(mx, z[u]); mn = fminf(mn, z[u]); }
        mx = warp_max(mx);
        mn = -warp_max(-mn);
        float ep[DH / 32], en[DH / 32], sp = 0.f, sn = 0.f;
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) {
            ep[u] = expf(z[u] - mx); en[u] = expf(mn - z[u]); sp += ep[u]; sn += en[u];
        }
        sp = warp_sum(sp);
        sn = warp_sum(sn);
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) {
            Ph[r * D + lane + 32 * u] = ep[u] / sp;
            Ph[r * D + DH + lane + 32 * u] = en[u] / sn;
        }
    }
    __syncthreads();

    // linear branch: acc = H_c^T phi(q), l = phi(q)^T s_c (H_c published as [d][D])
    const size_t snaps = (size_t)dm.nc_max + 1;
    const float* Hc = a.snap_H + ((size_t)st * snaps + c) * D * DIM;
    const float* sc = a.snap_s + ((size_t)st * snaps + c) * D;
    const bool read_state = !(a.read_mask & 1);
    float acc[QPW][CPL], m[QPW], l[QPW];
#pragma unroll
    for (int qq = 0; qq < QPW; ++qq) {
        const int r = warp * QPW + qq;
        float x = 0.f;
        if (read_state)
            for (int j = lane; j < D; j += 32) x = fmaf(Ph[r * D + j], sc[j], x);
        l[qq] = warp_sum(x);
        m[qq] = l[qq] > 0.f ? 0.f : -INFINITY;
#pragma unroll
        for (int u = 0; u < CPL; ++u) acc[qq][u] = 0.f;
    }
    constexpr int HT = KT;                            // H rows per tile (uses the Vs buffer)
    for (int j0 = 0; read_state && j0 < D; j0 += HT) {
        const int nj = min(HT, D - j0);
        __syncthreads();
        for (int idx = tid; idx < nj * DIM; idx += 256) {     // snapshot is H^T [d][D]
            const int jj = idx / DIM, cc = idx % DIM;
            Vs[jj * DIM + cc] = Hc[(size_t)cc * D + j0 + jj];
        }
        __syncthreads();
        for (int j = 0; j < nj; ++j) {
            float hv[CPL];
#pragma unroll
            for (int u = 0; u < CPL; ++u) hv[u] = Vs[j * DIM + lane * CPL + u];
#pragma unroll
            for (int qq = 0; qq < QPW; ++qq) {
                const float p = Ph[(warp * QPW + qq) * D + j0 + j];
#pragma unroll
                for (int u = 0; u < CPL; ++u) acc[qq][u] = fmaf(p, hv[u], acc[qq][u]);
            }
        }
    }

    // exact keys: cache slots, then the window, then the block up to the last query
    const int n_g = (a.read_mask & 2) ? 0 : min(dm.lam, max(0, t0 - dm.eta));
    const int w_lo = max(0, t0 - dm.eta);
    const int n_w = t0 - w_lo;
    const int n_c = qb * QB + nq;
    const int N = n_g + n_w + n_c;
    const int* cpos = a.snap_pos + ((size_t)st * snaps + c) * dm.lam;
    const float scale = 1.0f / sqrtf((float)DIM);
    for (int k0 = 0; k0 < N; k0 += KT) {
        __syncthreads();
        for (int idx = tid; idx < KT * DIM / 4; idx += 256) {
            const int kk = idx / (DIM / 4), j = (idx % (DIM / 4)) * 4;
            const int gk = k0 + kk;
            float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f), v4 = k4;
            int pos = 0x7fffffff;
            if (gk < N) {
                int slot = 0;
                if (gk < n_g) { slot = gk; pos = cpos[gk]; }
                else if (gk < n_g + n_w) pos = w_lo + (gk - n_g);
                else pos = t0 + (gk - n_g - n_w);
                const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, pos, slot);
                k4 = load4(r.k + j);
                v4 = load4(r.v + j);
            }
            Kt[(j + 0) * LDK + kk] = k4.x;
            Kt[(j + 1) * LDK + kk] = k4.y;
            Kt[(j + 2) * LDK + kk] = k4.z;
            Kt[(j + 3) * LDK + kk] = k4.w;
            *reinterpret_cast<float4*>(Vs + kk * DIM + j) = v4;
            if (j == 0) Kp[kk] = pos;
        }
        __syncthreads();
        float s0[QPW], s1[QPW];
#pragma unroll
        for (int qq = 0; qq < QPW; ++qq) s0[qq] = s1[qq] = 0.f;
        for (int j = 0; j < DIM; ++j) {
            const float k0v = Kt[j * LDK + lane], k1v = Kt[j * LDK + lane + 32];
#pragma unroll
            for (int qq = 0; qq < QPW; ++qq) {
                const float qj = Qs[(warp * QPW + qq) * DIM + j];
                s0[qq] = fmaf(qj, k0v, s0[qq]);
                s1[qq] = fmaf(qj, k1v, s1[qq]);
            }
        }
        const int p0 = Kp[lane], p1 = Kp[lane + 32];
#pragma unroll
        for (int qq = 0; qq < QPW; ++qq) {
            const int qpos = qlo + warp * QPW + qq;
            const float x0 = p0 <= qpos ? s0[qq] * scale : -INFINITY;
            const float x1 = p1 <= qpos ? s1[qq] * scale : -INFINITY;
            const float mn = fmaxf(m[qq], warp_max(fmaxf(x0, x1)));
            if (mn == -INFINITY) continue;            // nothing visible yet for this query
            const float corr = expf(m[qq] - mn);
            const float e0 = expf(x0 - mn), e1 = expf(x1 - mn);
            l[qq] = l[qq] * corr + warp_sum(e0 + e1);
            m[qq] = mn;
#pragma unroll
            for (int u = 0; u < CPL; ++u) acc[qq][u] *= corr;
            for (int kk = 0; kk < 32; ++kk) {
                const float pa = __shfl_sync(0xffffffffu, e0, kk);
                const float pb = __shfl_sync(0xffffffffu, e1, kk);
#pragma unroll
                for (int u = 0; u < CPL; ++u)
                    acc[qq][u] = fmaf(pa, Vs[kk * DIM + lane * CPL + u],
                                      fmaf(pb, Vs[(kk + 32) * DIM + lane * CPL + u], acc[qq][u]));
            }
        }
    }
#pragma unroll
    for (int qq = 0; qq < QPW; ++qq) {
        const int r = warp * QPW + qq;
        if (r >= nq) continue;
        const size_t i = (size_t)(qlo + r - a.t_start);
        float* yo = a.y + (((size_t)b * a.T + i) * dm.Hq + h) * DIM + lane * CPL;
        const float inv = 1.0f / l[qq];
#pragma unroll
        for (int u = 0; u < CPL; ++u) yo[u] = acc[qq][u] * inv;
    }
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_out_t(const PrefillArgs& a, cudaStream_t s) {
    using Sh = OutShape<DIM, DH>;
    const size_t bytes = (size_t)Sh::total * 4;
    cudaError_t e = cudaFuncSetAttribute(output_kernel<DIM, DH, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    const int nqb = (a.dm.C + Sh::QB - 1) / Sh::QB;
    dim3 grid((a.c_end - a.c_begin) * nqb, a.dm.Hq, a.dm.B);
    output_kernel<DIM, DH, TIn><<<grid, 256, bytes, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_out_d(const PrefillArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (d == 64 && Dh == 32) return launch_out_t<64, 32, TIn>(a, s);
    if (d == 64 && Dh == 64) return launch_out_t<64, 64, TIn>(a, s);
    if (d == 128 && Dh == 32) return launch_out_t<128, 32, TIn>(a, s);
    if (d == 128 && Dh == 64) return launch_out_t<128, 64, TIn>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_output(const PrefillArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_out_d<__nv_bfloat16>(a, s) : launch_out_d<float>(a, s);
}

}  // namespace lola

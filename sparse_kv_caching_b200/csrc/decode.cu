// Per-token LoLA decode step (notes §2.4, Fig. 1; one-token block of §2.6).
//
// For the new token at position t of every stream (sequence b, kv head g):
//   1. read (Eq. 14) with the memories entering the step: the cache G, the
//      window [max(0, t - eta), t), the token itself and (H, s);
//   2. the oldest window pair l = t - eta leaves; E = G u {l};
//   3. |E| <= lambda: l takes the next free cache slot; otherwise score all
//      lambda + 1 candidates by SRE against the pre-fold (H, s) (Eq. 10),
//      fold the single lowest one (ties: the newer position goes; Eqs. 11-13)
//      and, if that was not l, l takes its slot;
//   4. the new token enters the window ring at slot t % eta.
// One CTA per stream; H (D x d fp32) is staged in shared memory for the
// linear read, the SRE scoring and the rank-1 fold, then written back.
#include "device_common.cuh"

namespace lola {

template <int DIM, int DH>
struct DecShape {
    static constexpr int D = 2 * DH;
    using Sh = SreShape<D, DIM, float>;
};

struct DecOffsets {
    int Hs, ss, tile, den, qs, phq, kn, vn, phk, red, sc, sre, total;
};

__host__ __device__ inline DecOffsets dec_offsets(int DIM, int DH, int Gq, int lam, int eta) {
    const int D = 2 * DH, TE = (kThreads / (DIM / 4)) * 8, LD = D + 4;
    const int NK = lam + eta + 1;
    DecOffsets o;
    int p = 0;
    auto take = [&](int n) { int r = p; p += (n + 3) & ~3; return r; };
    o.Hs = take(D * DIM);
    o.ss = take(D);
    o.tile = take(max(TE * LD, max(DIM * DH, 2 * (kThreads / DIM) * Gq * DIM)));
    o.den = take(TE);
    o.qs = take(Gq * DIM);
    o.phq = take(Gq * D);
    o.kn = take(DIM);
    o.vn = take(DIM);
    o.phk = take(D);
    o.red = take(64);
    o.sc = take(Gq * NK);
    o.sre = take(2 * (lam + 1));
    o.total = p;
    return o;
}

template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int D = 2 * DH;
    using Sh = SreShape<D, DIM, TIn>;
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int Gq = dm.Gq, lam = dm.lam, eta = dm.eta, t = a.t;
    const int st = blockIdx.x, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const DecOffsets o = dec_offsets(DIM, DH, Gq, lam, eta);
    float* Hs = smem + o.Hs;
    float* ss = smem + o.ss;
    float* tile = smem + o.tile;
    float* den = smem + o.den;
    float* qs = smem + o.qs;
    float* phq = smem + o.phq;
    float* kn = smem + o.kn;
    float* vn = smem + o.vn;
    float* phk = smem + o.phk;
    float* red = smem + o.red;
    float* sc = smem + o.sc;
    float* sre = smem + o.sre;
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(red);   // reuses red[0..)
    float* Ws = tile;

    float* Hg = a.sp.H + (size_t)st * D * DIM;
    float* sg = a.sp.s + (size_t)st * D;
    const TIn* Wg = (const TIn*)a.sp.W + (size_t)g * DIM * DH;
    for (int i = tid; i < DIM * DH; i += kThreads) Ws[i] = to_f32(Wg[i]);
    for (int i = tid; i < D * DIM / 4; i += kThreads)
        reinterpret_cast<float4*>(Hs)[i] = reinterpret_cast<const float4*>(Hg)[i];
    for (int i = tid; i < D; i += kThreads) ss[i] = sg[i];
    const TIn* qg = (const TIn*)a.q + ((size_t)b * dm.Hq + (size_t)g * Gq) * DIM;
    for (int i = tid; i < Gq * DIM; i += kThreads) qs[i] = to_f32(qg[i]);
    const TIn* kg = (const TIn*)a.k + ((size_t)b * dm.Hkv + g) * DIM;
    const TIn* vg = (const TIn*)a.v + ((size_t)b * dm.Hkv + g) * DIM;
    for (int i = tid; i < DIM; i += kThreads) { kn[i] = to_f32(kg[i]); vn[i] = to_f32(vg[i]); }
    __syncthreads();

    // feature map of the queries and of the new key (one warp per row)
    for (int r = warp; r <= Gq; r += kThreads / 32) {
        const float* x = r < Gq ? qs + r * DIM : kn;
        float z[DH / 32];
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) z[u] = 0.f;
        for (int j = 0; j < DIM; ++j) {
#pragma unroll
            for (int u = 0; u < DH / 32; ++u) z[u] = fmaf(x[j], Ws[j * DH + lane + 32 * u], z[u]);
        }
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) { mx = fmaxf(mx, z[u]); mn = fminf(mn, z[u]); }
        mx = warp_max(mx);
        mn = -warp_max(-mn);
        float ep[DH / 32], en[DH / 32], sp = 0.f, sn = 0.f;
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) { ep[u] = expf(z[u] - mx); en[u] = expf(mn - z[u]); sp += ep[u]; sn += en[u]; }
        sp = warp_sum(sp);
        sn = warp_sum(sn);
        float* out = r < Gq ? phq + r * D : phk;
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) { out[lane + 32 * u] = ep[u] / sp; out[DH + lane + 32 * u] = en[u] / sn; }
    }
    __syncthreads();

    // ---- read: exact keys (cache, window, self) ----
    const int n_g = min(lam, max(0, t - eta));
    const int w_lo = max(0, t - eta);
    const int n_w = t - w_lo;
    const int NK = n_g + n_w + 1;
    const size_t cbase = (size_t)st * lam, wbase = (size_t)st * eta;
    auto key_row = [&](int i, const TIn*& kp, const TIn*& vp) {
        if (i < n_g) { kp = (const TIn*)a.sp.cache_k + (cbase + i) * DIM; vp = (const TIn*)a.sp.cache_v + (cbase + i) * DIM; }
        else if (i < n_g + n_w) {
            const size_t w = wbase + (size_t)((w_lo + i - n_g) % eta);
            kp = (const TIn*)a.sp.win_k + w * DIM; vp = (const TIn*)a.sp.win_v + w * DIM;
        } else { kp = kg; vp = vg; }
    };
    const float scale = 1.0f / sqrtf((float)DIM);
    for (int i = tid; i < NK; i += kThreads) {
        const TIn *kp, *vp;
        key_row(i, kp, vp);
        float accs[8];
#pragma unroll
        for (int hh = 0; hh < 8; ++hh) accs[hh] = 0.f;
        for (int j = 0; j < DIM; j += 4) {
            const float4 k4 = load4(kp + j);
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) {
                if (hh < Gq) {
                    const float* qh = qs + hh * DIM + j;
                    accs[hh] = fmaf(qh[0], k4.x, fmaf(qh[1], k4.y, fmaf(qh[2], k4.z, fmaf(qh[3], k4.w, accs[hh]))));
                }
            }
        }
        for (int hh = 0; hh < Gq; ++hh) sc[hh * NK + i] = accs[hh] * scale;
    }
    __syncthreads();
    // per head: max, exponentials, sum; linear denominator
    for (int hh = warp; hh < Gq; hh += kThreads / 32) {
        float mx = -INFINITY;
        for (int i = lane; i < NK; i += 32) mx = fmaxf(mx, sc[hh * NK + i]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < NK; i += 32) { const float e = expf(sc[hh * NK + i] - mx); sc[hh * NK + i] = e; sum += e; }
        sum = warp_sum(sum);
        float dl = 0.f;
        for (int j = lane; j < D; j += 32) dl = fmaf(phq[hh * D + j], ss[j], dl);
        dl = warp_sum(dl);
        if (lane == 0) { red[hh] = mx; red[8 + hh] = sum; red[16 + hh] = dl; }
    }
    __syncthreads();
    {
        constexpr int GR = kThreads / DIM;           // key groups
        const int cidx = tid % DIM, grp = tid / DIM;
        float aacc[8], lacc[8];
#pragma unroll
        for (int hh = 0; hh < 8; ++hh) aacc[hh] = lacc[hh] = 0.f;
        for (int i = grp; i < NK; i += GR) {
            const TIn *kp, *vp;
            key_row(i, kp, vp);
            const float vv = to_f32(vp[cidx]);
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) if (hh < Gq) aacc[hh] = fmaf(sc[hh * NK + i], vv, aacc[hh]);
        }
        for (int j = grp; j < D; j += GR) {
            const float hv = Hs[j * DIM + cidx];
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) if (hh < Gq) lacc[hh] = fmaf(phq[hh * D + j], hv, lacc[hh]);
        }
        float* ra = tile;                            // [GR][Gq][DIM]
        float* rl = tile + GR * Gq * DIM;
        for (int hh = 0; hh < Gq; ++hh) {
            ra[(grp * Gq + hh) * DIM + cidx] = aacc[hh];
            rl[(grp * Gq + hh) * DIM + cidx] = lacc[hh];
        }
        __syncthreads();
        for (int idx = tid; idx < Gq * DIM; idx += kThreads) {
            const int hh = idx / DIM, cc = idx % DIM;
            float A = 0.f, L = 0.f;
            for (int r = 0; r < GR; ++r) { A += ra[(r * Gq + hh) * DIM + cc]; L += rl[(r * Gq + hh) * DIM + cc]; }
            const float em = expf(-red[hh]);
            const float yv = (A + em * L) / (red[8 + hh] + em * red[16 + hh]);
            a.y[((size_t)b * dm.Hq + (size_t)g * Gq + hh) * DIM + cc] = yv;
        }
        __syncthreads();
    }

    // ---- update ----
    if (t >= eta) {
        const int lpos = t - eta, rs = lpos % eta;
        const size_t wsl = wbase + rs;
        if (n_g < lam) {
            const size_t cs = cbase + n_g;
            for (int i = tid; i < DIM; i += kThreads) {
                ((TIn*)a.sp.cache_k)[cs * DIM + i] = ((const TIn*)a.sp.win_k)[wsl * DIM + i];
                ((TIn*)a.sp.cache_v)[cs * DIM + i] = ((const TIn*)a.sp.win_v)[wsl * DIM + i];
            }
            for (int i = tid; i < D; i += kThreads) a.sp.cache_phik[cs * D + i] = a.sp.win_phik[wsl * D + i];
            if (tid == 0) a.sp.cache_pos[cs] = lpos;
        } else {
            const int n = lam + 1;
            auto phirow = [&](int e) -> const float* {
                return e < lam ? a.sp.cache_phik + (cbase + e) * D : a.sp.win_phik + wsl * D;
            };
            auto vrow = [&](int e) -> const TIn* {
                return e < lam ? (const TIn*)a.sp.cache_v + (cbase + e) * DIM : (const TIn*)a.sp.win_v + wsl * DIM;
            };
            for (int e0 = 0; e0 < n; e0 += Sh::TE) {
                const int ne = min(Sh::TE, n - e0);
                load_phi_tile<D>(tile, ne, [&](int e) { return phirow(e0 + e); });
                __syncthreads();
                sre_tile<D, DIM, TIn>(Hs, ss, tile, den, ne, [&](int e) { return vrow(e0 + e); }, sre + e0);
            }
            // the folded pair: lowest SRE, newer position on exact ties (keys are unique)
            auto cand_key = [&](int e) -> unsigned long long {
                const int p = e < lam ? a.sp.cache_pos[cbase + e] : lpos;
                return ((unsigned long long)__float_as_uint(sre[e]) << 32) | (unsigned long long)(~(unsigned)p);
            };
            unsigned long long best = ~0ull;
            for (int e = tid; e < n; e += kThreads) { const unsigned long long k = cand_key(e); best = k < best ? k : best; }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const unsigned long long o2 = __shfl_xor_sync(0xffffffffu, best, off);
                best = o2 < best ? o2 : best;
            }
            if (lane == 0) keys[warp] = best;
            __syncthreads();
            unsigned long long bb = keys[0];
            for (int w = 1; w < kThreads / 32; ++w) bb = keys[w] < bb ? keys[w] : bb;
            for (int e = tid; e < n; e += kThreads)
                if (cand_key(e) == bb) reinterpret_cast<int*>(red)[40] = e;
            __syncthreads();
            const int f = reinterpret_cast<int*>(red)[40];
            // stage the folded pair
            float* fphi = tile;
            float* fv = tile + D;
            for (int i = tid; i < D; i += kThreads) fphi[i] = phirow(f)[i];
            for (int i = tid; i < DIM; i += kThreads) fv[i] = to_f32(vrow(f)[i]);
            __syncthreads();
            for (int i = tid; i < D * DIM; i += kThreads) {
                const int j = i / DIM, cc = i % DIM;
                Hs[i] = fmaf(fphi[j], fv[cc], Hs[i]);
            }
            for (int i = tid; i < D; i += kThreads) ss[i] += fphi[i];
            if (f < lam) {                           // l takes the folded member's slot
                const size_t cs = cbase + f;
                for (int i = tid; i < DIM; i += kThreads) {
                    ((TIn*)a.sp.cache_k)[cs * DIM + i] = ((const TIn*)a.sp.win_k)[wsl * DIM + i];
                    ((TIn*)a.sp.cache_v)[cs * DIM + i] = ((const TIn*)a.sp.win_v)[wsl * DIM + i];
                }
                for (int i = tid; i < D; i += kThreads) a.sp.cache_phik[cs * D + i] = a.sp.win_phik[wsl * D + i];
                if (tid == 0) a.sp.cache_pos[cs] = lpos;
            }
            __syncthreads();
            for (int i = tid; i < D * DIM / 4; i += kThreads)
                reinterpret_cast<float4*>(Hg)[i] = reinterpret_cast<const float4*>(Hs)[i];
            for (int i = tid; i < D; i += kThreads) sg[i] = ss[i];
        }
    }
    __syncthreads();
    // the new token enters the window ring
    {
        const size_t ws = wbase + (size_t)(t % eta);
        for (int i = tid; i < DIM; i += kThreads) {
            ((TIn*)a.sp.win_k)[ws * DIM + i] = kg[i];
            ((TIn*)a.sp.win_v)[ws * DIM + i] = vg[i];
        }
        for (int i = tid; i < D; i += kThreads) a.sp.win_phik[ws * D + i] = phk[i];
    }
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_dec_t(const DecodeArgs& a, cudaStream_t s) {
    const size_t bytes = (size_t)dec_offsets(DIM, DH, a.dm.Gq, a.dm.lam, a.dm.eta).total * 4;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<DIM, DH, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    decode_kernel<DIM, DH, TIn><<<a.dm.S, kThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_dec_d(const DecodeArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (d == 64 && Dh == 32) return launch_dec_t<64, 32, TIn>(a, s);
    if (d == 64 && Dh == 64) return launch_dec_t<64, 64, TIn>(a, s);
    if (d == 128 && Dh == 32) return launch_dec_t<128, 32, TIn>(a, s);
    if (d == 128 && Dh == 64) return launch_dec_t<128, 64, TIn>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_dec_d<__nv_bfloat16>(a, s) : launch_dec_d<float>(a, s);
}

size_t decode_smem_bytes(const Dims& dm) {
    return (size_t)dec_offsets(dm.d, dm.Dh, dm.Gq, dm.lam, dm.eta).total * 4;
}

}  // namespace lola

// Window scores of the alternative scoring rules (LoLA notes §4.5, Table 4;
// App. F, whose Eqs. 22-25 the pages do not print).  A key's score is a sum,
// over every query that reads it exactly through the window or its own block
// (all heads of its kv group), of one term of a = exp(q.k / sqrt(d)) and
// f = phi(q)^T phi(k):
//   rule 1: (a - f)^2    rule 2: |a - f|    rule 3: f / a    rule 4: a.
// The sum stops when the key leaves the window; a cached key keeps its score.
//
// Block reading (chunk C, window eta, call starting at t_start): key i is read
// by its own block from i on and then by every block whose preceding eta
// pairs hold it, so inside the call the queries t in
//   [max(i, t_start), t_start + (floor((i + eta - t_start) / C) + 1) C)
// credit it.  Keys of the window entering the call carry the sum of earlier
// calls and decode steps (win_sc); the call's last eta keys leave theirs in
// win_sc for the next call.
//
// key_scores_kernel: one CTA per (stream, 64 keys), looping over tiles of 64
// (query, head) rows that cover the union of its keys' query ranges.  Per
// tile: the rows' phi(q) (the prefill's feature map, recomputed), then
// q.k over d and phi(q).phi(k) over D as 4 key x 4 row register tiles per
// thread, the rule's term where the query credits the key, and a per-key sum
// reduced over the 16 row groups of a half warp at the end.
#include "device_common.cuh"

namespace lola {

constexpr int kScKeys = 64;       // keys per CTA
constexpr int kScRows = 64;       // (query, head) rows per tile
constexpr int kScThreads = 256;

template <int DIM, int DH>
struct ScShape {
    static constexpr int D = 2 * DH, KL = DIM + 4, PL = D + 4;
    static constexpr int K = 0;                        // [kScKeys][KL] keys
    static constexpr int PK = K + kScKeys * KL;        // [kScKeys][PL] phi(k)
    static constexpr int Q = PK + kScKeys * PL;        // [kScRows][KL] query rows
    static constexpr int PQ = Q + kScRows * KL;        // [kScRows][PL] phi(q)
    static constexpr int W = PQ + kScRows * PL;        // [DIM][DH]
    static constexpr int total = W + DIM * DH;         // floats
};

template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(kScThreads, 1) key_scores_kernel(const __grid_constant__ PrefillArgs a) {
    using Sh = ScShape<DIM, DH>;
    constexpr int D = Sh::D, KL = Sh::KL, PL = Sh::PL, CPL = DH / 32;
    extern __shared__ __align__(16) float smem[];
    float* Ks = smem + Sh::K;
    float* PKs = smem + Sh::PK;
    float* Qs = smem + Sh::Q;
    float* PQs = smem + Sh::PQ;
    float* Ws = smem + Sh::W;
    const Dims& dm = a.dm;
    const int st = blockIdx.y, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Gq = dm.Gq, eta = dm.eta, C = dm.C;
    const int t_end = a.t_start + a.T;
    const int i0 = max(0, a.t_start - eta) + blockIdx.x * kScKeys;
    if (i0 >= t_end) return;
    const int nk = min(kScKeys, t_end - i0);
    auto q_end = [&](int i) { return min(t_end, a.t_start + ((i + eta - a.t_start) / C + 1) * C); };
    const int q_lo = max(i0, a.t_start), q_hi = q_end(i0 + nk - 1);   // q_end grows with i

    const TIn* Wg = (const TIn*)a.sp.W + (size_t)g * DIM * DH;
    for (int i = tid; i < DIM * DH; i += kScThreads) Ws[i] = to_f32(Wg[i]);
    for (int kk = warp; kk < kScKeys; kk += kScThreads / 32) {
        if (kk < nk) {
            const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, i0 + kk, 0);
            for (int j = lane; j < DIM; j += 32) Ks[kk * KL + j] = to_f32(r.k[j]);
            for (int j = lane; j < D; j += 32) PKs[kk * PL + j] = r.phik[j];
        } else {
            for (int j = lane; j < DIM; j += 32) Ks[kk * KL + j] = 0.f;
            for (int j = lane; j < D; j += 32) PKs[kk * PL + j] = 0.f;
        }
    }
    const int kq = tid >> 4, rq = tid & 15;            // keys 4 kq .. 4 kq + 3, rows rq + 16 w
    const int QT = kScRows / Gq;                        // queries per tile
    const float scale = 1.0f / sqrtf((float)DIM);
    float kacc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int tq = q_lo; tq < q_hi; tq += QT) {
        const int nq = min(QT, q_hi - tq);
        __syncthreads();                                // the previous tile's rows are consumed
        // query rows r = query * Gq + head, then their feature map (a warp per row)
        for (int r = warp; r < kScRows; r += kScThreads / 32) {
            const int qi = r / Gq, hh = r % Gq;
            if (qi < nq) {
                const TIn* x = (const TIn*)a.q +
                               (((size_t)b * a.T + (tq + qi - a.t_start)) * dm.Hq + (size_t)g * Gq + hh) * DIM;
                for (int j = lane; j < DIM; j += 32) Qs[r * KL + j] = to_f32(x[j]);
            } else {
                for (int j = lane; j < DIM; j += 32) Qs[r * KL + j] = 0.f;
            }
            __syncwarp();
            float z[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) z[c] = 0.f;
            for (int j = 0; j < DIM; ++j) {
                const float xj = Qs[r * KL + j];
#pragma unroll
                for (int c = 0; c < CPL; ++c) z[c] = fmaf(xj, Ws[j * DH + lane + 32 * c], z[c]);
            }
            float mx = -INFINITY, mn = INFINITY;
#pragma unroll
            for (int c = 0; c < CPL; ++c) { mx = fmaxf(mx, z[c]); mn = fminf(mn, z[c]); }
            mx = warp_max(mx);
            mn = -warp_max(-mn);
            float ep[CPL], en[CPL], sp = 0.f, sn = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                ep[c] = expf(z[c] - mx);
                en[c] = expf(mn - z[c]);
                sp += ep[c];
                sn += en[c];
            }
            sp = warp_sum(sp);
            sn = warp_sum(sn);
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                PQs[r * PL + lane + 32 * c] = ep[c] / sp;
                PQs[r * PL + DH + lane + 32 * c] = en[c] / sn;
            }
        }
        __syncthreads();
        // logits q.k and feature kernels phi(q).phi(k) of 4 keys x 4 rows
        float L[4][4], F[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) { L[u][w] = 0.f; F[u][w] = 0.f; }
#pragma unroll 2
        for (int j = 0; j < DIM; j += 4) {
            float4 kv[4], qv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) kv[u] = *reinterpret_cast<const float4*>(Ks + (4 * kq + u) * KL + j);
#pragma unroll
            for (int w = 0; w < 4; ++w) qv[w] = *reinterpret_cast<const float4*>(Qs + (rq + 16 * w) * KL + j);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    L[u][w] = fmaf(kv[u].x, qv[w].x, L[u][w]);
                    L[u][w] = fmaf(kv[u].y, qv[w].y, L[u][w]);
                    L[u][w] = fmaf(kv[u].z, qv[w].z, L[u][w]);
                    L[u][w] = fmaf(kv[u].w, qv[w].w, L[u][w]);
                }
        }
#pragma unroll 2
        for (int j = 0; j < D; j += 4) {
            float4 kv[4], qv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) kv[u] = *reinterpret_cast<const float4*>(PKs + (4 * kq + u) * PL + j);
#pragma unroll
            for (int w = 0; w < 4; ++w) qv[w] = *reinterpret_cast<const float4*>(PQs + (rq + 16 * w) * PL + j);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    F[u][w] = fmaf(kv[u].x, qv[w].x, F[u][w]);
                    F[u][w] = fmaf(kv[u].y, qv[w].y, F[u][w]);
                    F[u][w] = fmaf(kv[u].z, qv[w].z, F[u][w]);
                    F[u][w] = fmaf(kv[u].w, qv[w].w, F[u][w]);
                }
        }
        // terms where query t credits key i: t >= i and t before the key leaves the window
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int kk = 4 * kq + u, i = i0 + kk;
            if (kk >= nk) continue;
            const int qe = q_end(i);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int r = rq + 16 * w, qi = r / Gq, t = tq + qi;
                if (qi < nq && t >= i && t < qe) kacc[u] += window_term(a.scorer, expf(L[u][w] * scale), F[u][w]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) kacc[u] += __shfl_xor_sync(0xffffffffu, kacc[u], off);
    if (rq == 0) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int kk = 4 * kq + u, i = i0 + kk;
            if (kk >= nk) continue;
            const float prior = i < a.t_start ? a.sp.win_sc[(size_t)st * eta + (size_t)(i % eta)] : 0.f;
            a.key_sc[(size_t)st * (eta + dm.max_tokens) + (size_t)(i - a.t_start + eta)] = prior + kacc[u];
        }
    }
}

// After the call: each cache member that joined during it keeps its score with its
// slot, and the keys of the final window keep their partial sums in the ring.
__global__ void __launch_bounds__(256) finalize_scores_kernel(const __grid_constant__ PrefillArgs a) {
    const Dims& dm = a.dm;
    const int st = blockIdx.x, lam = dm.lam, eta = dm.eta;
    const size_t snaps = (size_t)dm.nc_max + 1, kb = (size_t)st * (eta + dm.max_tokens);
    const int* fin = a.snap_pos + ((size_t)st * snaps + a.nc) * lam;
    const int t_end = a.t_start + a.T;
    const int n_g = min(lam, max(0, t_end - eta));
    for (int j = threadIdx.x; j < n_g; j += blockDim.x) {
        const int p = fin[j];
        if (p >= a.t_start - eta) a.sp.cache_sc[(size_t)st * lam + j] = a.key_sc[kb + (size_t)(p - a.t_start + eta)];
    }
    for (int p = max(0, t_end - eta) + threadIdx.x; p < t_end; p += blockDim.x)
        a.sp.win_sc[(size_t)st * eta + (size_t)(p % eta)] = a.key_sc[kb + (size_t)(p - a.t_start + eta)];
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_ks_t(const PrefillArgs& a, cudaStream_t s) {
    const size_t bytes = (size_t)ScShape<DIM, DH>::total * 4;
    cudaError_t e = cudaFuncSetAttribute(key_scores_kernel<DIM, DH, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    const int nkeys = a.t_start + a.T - max(0, a.t_start - a.dm.eta);
    dim3 grid((nkeys + kScKeys - 1) / kScKeys, a.dm.S);
    key_scores_kernel<DIM, DH, TIn><<<grid, kScThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_ks_d(const PrefillArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (d == 64 && Dh == 32) return launch_ks_t<64, 32, TIn>(a, s);
    if (d == 64 && Dh == 64) return launch_ks_t<64, 64, TIn>(a, s);
    if (d == 128 && Dh == 32) return launch_ks_t<128, 32, TIn>(a, s);
    if (d == 128 && Dh == 64) return launch_ks_t<128, 64, TIn>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_key_scores(const PrefillArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_ks_d<__nv_bfloat16>(a, s) : launch_ks_d<float>(a, s);
}

cudaError_t launch_finalize_scores(const PrefillArgs& a, cudaStream_t s) {
    finalize_scores_kernel<<<a.dm.S, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lola

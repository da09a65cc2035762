// The per-stream memory-update chain of chunkwise LoLA prefill.
//
// LoLA notes §2.6 (Eq. 15, Fig. 2): after each block the pairs leaving the
// window and the cache members are scored by Self-Recall Error against the
// state (§2.3, Eq. 10), the lambda highest stay in the cache, the rest are
// folded into (H, s) (§2.4, Eqs. 11-13).  The allocation of block c depends
// on the state after block c-1, so the blocks of one stream run in order; the
// streams (one per sequence and kv head) are independent: one CTA each.
//
// The chain never reads a query.  It publishes, for every block c of the
// call, the memories ENTERING that block (cache positions by slot, H_c, s_c)
// so that the output kernel can serve all blocks in parallel afterwards.
//
// Per scored block: SRE of the n = |G| + |L| candidates in fp32 FFMA with H
// resident in shared memory; top-lambda by a 4-pass radix select over the
// score bits with exact ties broken towards the older position; slot
// bookkeeping by block scans (kept incumbents stay in their slots, kept
// newcomers fill the freed slots in slot order); the fold H += Phi_S^T V_S,
// s += sum Phi_S with H held in registers.
#include "device_common.cuh"

namespace lola {

struct ScanOffsets {          // offsets in 4-byte words
    int Hs, ss, tile, den, score, slot_pos, cand_pos, flags, ranks, keep, free_slots,
        fold_list, tmp, hist, sbits, eq_list, newslot, total;
};

__host__ __device__ inline ScanOffsets scan_offsets(int D, int DV, int lam, int C) {
    const int TE = (kThreads / (DV / 4)) * 8, LD = D + 4, NMAX = lam + C;
    ScanOffsets o;
    int p = 0;
    auto take = [&](int n) { int r = p; p += (n + 3) & ~3; return r; };
    o.Hs = take(D * DV);
    o.ss = take(D);
    o.tile = take(TE * LD);
    o.den = take(TE);
    o.score = take(NMAX);
    o.slot_pos = take(lam + 1);
    o.cand_pos = take(NMAX);
    o.flags = take(NMAX);
    o.ranks = take(NMAX);
    o.keep = take(NMAX);
    o.free_slots = take(lam + 1);
    o.fold_list = take(NMAX);
    o.tmp = take(64);
    o.hist = take(256);
    o.sbits = take(NMAX);
    o.eq_list = take(NMAX);
    o.newslot = take(C);
    o.total = p;
    return o;
}

// keep[i] = 1 for the lam candidates with the largest (score, -position);
// exact: a 4-pass MSB radix select over the fp32 score bits (scores >= 0, so
// the bit pattern orders like the value), then the candidates equal to the
// threshold are ranked by position.
__device__ void select_top(const float* score, const int* cand_pos, int n, int lam, int* keep,
                           unsigned* sbits, unsigned* hist, int* tmp, int* eq_list) {
    const int tid = threadIdx.x, lane = tid & 31;
    for (int i = tid; i < n; i += kThreads) sbits[i] = __float_as_uint(score[i]);
    unsigned prefix = 0u, mask = 0u;
    int kk = lam;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const unsigned u = sbits[i];
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            unsigned c[8], lsum = 0u;
#pragma unroll
            for (int t = 0; t < 8; ++t) { c[t] = hist[lane * 8 + t]; lsum += c[t]; }
            unsigned suf = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            unsigned above = suf - lsum;            // candidates whose digit lies in higher lanes
#pragma unroll
            for (int t = 7; t >= 0; --t) {
                if (above < (unsigned)kk && (unsigned)kk <= above + c[t]) {
                    tmp[0] = lane * 8 + t;
                    tmp[1] = kk - (int)above;
                }
                above += c[t];
            }
        }
        __syncthreads();
        prefix |= (unsigned)tmp[0] << shift;
        mask |= 255u << shift;
        kk = tmp[1];
    }
    __syncthreads();
    if (tid == 0) tmp[2] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
        const unsigned u = sbits[i];
        keep[i] = u > prefix ? 1 : 0;
        if (u == prefix) eq_list[atomicAdd(&tmp[2], 1)] = i;
    }
    __syncthreads();
    const int neq = tmp[2];
    for (int q = tid; q < neq; q += kThreads) {
        const int i = eq_list[q], p = cand_pos[i];
        int r = 0;
        for (int z = 0; z < neq; ++z) r += cand_pos[eq_list[z]] < p ? 1 : 0;
        keep[i] = r < kk ? 1 : 0;
    }
    __syncthreads();
}

template <int D, int DV, typename TIn>
__global__ void __launch_bounds__(kThreads, 1) scan_kernel(PrefillArgs a) {
    using Sh = SreShape<D, DV, TIn>;
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int lam = dm.lam, C = dm.C, eta = dm.eta;
    const int st = blockIdx.x, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x;
    const ScanOffsets o = scan_offsets(D, DV, lam, C);
    float* Hs = smem + o.Hs;
    float* ss = smem + o.ss;
    float* tile = smem + o.tile;
    float* den = smem + o.den;
    float* score = smem + o.score;
    int* slot_pos = reinterpret_cast<int*>(smem + o.slot_pos);
    int* cand_pos = reinterpret_cast<int*>(smem + o.cand_pos);
    int* flags = reinterpret_cast<int*>(smem + o.flags);
    int* ranks = reinterpret_cast<int*>(smem + o.ranks);
    int* keep = reinterpret_cast<int*>(smem + o.keep);
    int* free_slots = reinterpret_cast<int*>(smem + o.free_slots);
    int* fold_list = reinterpret_cast<int*>(smem + o.fold_list);
    int* tmp = reinterpret_cast<int*>(smem + o.tmp);
    unsigned* hist = reinterpret_cast<unsigned*>(smem + o.hist);
    unsigned* sbits = reinterpret_cast<unsigned*>(smem + o.sbits);
    int* eq_list = reinterpret_cast<int*>(smem + o.eq_list);
    int* newslot = reinterpret_cast<int*>(smem + o.newslot);

    const size_t snaps = (size_t)dm.nc_max + 1;
    const float* Hg = a.sp.H + (size_t)st * D * DV;
    const float* sg = a.sp.s + (size_t)st * D;
    for (int i = tid; i < D * DV / 4; i += kThreads)
        reinterpret_cast<float4*>(Hs)[i] = reinterpret_cast<const float4*>(Hg)[i];
    for (int i = tid; i < D; i += kThreads) ss[i] = sg[i];
    for (int j = tid; j < lam; j += kThreads) slot_pos[j] = a.sp.cache_pos[(size_t)st * lam + j];
    __syncthreads();

    auto publish = [&](int c) {
        int* sp_ = a.snap_pos + ((size_t)st * snaps + c) * lam;
        float* sH = a.snap_H + ((size_t)st * snaps + c) * D * DV;
        float* sS = a.snap_s + ((size_t)st * snaps + c) * D;
        for (int j = tid; j < lam; j += kThreads) sp_[j] = slot_pos[j];
        // H_c is published transposed, [d][D], so that a row c holds H[.][c]
        for (int i = tid; i < DV * (D / 4); i += kThreads) {
            const int cc = i % DV, j4 = (i / DV) * 4;
            reinterpret_cast<float4*>(sH + (size_t)cc * D)[j4 / 4] =
                make_float4(Hs[(j4 + 0) * DV + cc], Hs[(j4 + 1) * DV + cc], Hs[(j4 + 2) * DV + cc],
                            Hs[(j4 + 3) * DV + cc]);
        }
        for (int i = tid; i < D; i += kThreads) sS[i] = ss[i];
    };
    publish(0);

    // fold-phase thread layout: rows ty*RPT.., columns 4tx..4tx+3
    constexpr int TXF = DV / 4, TYF = kThreads / TXF, RPT = D / TYF, TF = 32, LDV = DV + 4;
    const int ftx = tid % TXF, fty = tid / TXF;

    for (int c = 0; c < a.nc; ++c) {
        const int t0 = a.t_start + c * C;
        const int n_g = min(lam, max(0, t0 - eta));
        const int l_lo = max(0, t0 - eta), l_hi = max(0, t0 + C - eta);
        const int n_l = l_hi - l_lo;
        if (n_l > 0 && n_g + n_l <= lam) {
            // every candidate fits: keep all (notes §2.4: fewer than lambda candidates)
            for (int i = tid; i < n_l; i += kThreads) slot_pos[n_g + i] = l_lo + i;
        } else if (n_l > 0) {
            const int n = n_g + n_l;
            for (int i = tid; i < n; i += kThreads) cand_pos[i] = i < n_g ? slot_pos[i] : l_lo + (i - n_g);
            __syncthreads();
            auto ref = [&](int e) { return pair_ref<TIn>(a, st, b, g, cand_pos[e], e); };
            if (lam > 0) {
                for (int e0 = 0; e0 < n; e0 += Sh::TE) {
                    const int ne = min(Sh::TE, n - e0);
                    load_phi_tile<D>(tile, ne, [&](int e) { return ref(e0 + e).phik; });
                    __syncthreads();
                    sre_tile<D, DV, TIn>(Hs, ss, tile, den, ne, [&](int e) { return ref(e0 + e).v; },
                                         score + e0);
                }
                select_top(score, cand_pos, n, lam, keep, sbits, hist, tmp, eq_list);
            } else {
                for (int i = tid; i < n; i += kThreads) keep[i] = 0;
                __syncthreads();
            }
            // freed slots (evicted incumbents and never-used slots), in slot order
            for (int j = tid; j < lam; j += kThreads) flags[j] = (j >= n_g || keep[j] == 0) ? 1 : 0;
            __syncthreads();
            block_exscan(flags, ranks, lam, tmp);
            for (int j = tid; j < lam; j += kThreads) if (flags[j]) free_slots[ranks[j]] = j;
            __syncthreads();
            // retained newcomers, in position order, take the freed slots in order
            for (int i = tid; i < n_l; i += kThreads) flags[i] = keep[n_g + i];
            __syncthreads();
            block_exscan(flags, ranks, n_l, tmp);
            for (int i = tid; i < n_l; i += kThreads) newslot[i] = flags[i] ? free_slots[ranks[i]] : -1;
            __syncthreads();
            // the folded set S = E \ G_new
            for (int e = tid; e < n; e += kThreads) flags[e] = keep[e] ? 0 : 1;
            __syncthreads();
            const int nf = block_exscan(flags, ranks, n, tmp);
            for (int e = tid; e < n; e += kThreads) if (flags[e]) fold_list[ranks[e]] = e;
            __syncthreads();
            // fold: H += phi_S^T V_S, s += sum phi_S (notes §2.4, Eqs. 12-13)
            float hreg[RPT][4];
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float4 h4 = *reinterpret_cast<const float4*>(Hs + (fty * RPT + i) * DV + 4 * ftx);
                hreg[i][0] = h4.x; hreg[i][1] = h4.y; hreg[i][2] = h4.z; hreg[i][3] = h4.w;
            }
            float sacc = 0.f;
            float* fphi = tile;
            float* fv = tile + TF * Sh::LD;
            for (int f0 = 0; f0 < nf; f0 += TF) {
                const int nff = min(TF, nf - f0);
                for (int idx = tid; idx < nff * (D / 4); idx += kThreads) {
                    const int f = idx / (D / 4), j = (idx % (D / 4)) * 4;
                    *reinterpret_cast<float4*>(fphi + f * Sh::LD + j) =
                        *reinterpret_cast<const float4*>(ref(fold_list[f0 + f]).phik + j);
                }
                for (int idx = tid; idx < nff * (DV / 4); idx += kThreads) {
                    const int f = idx / (DV / 4), j = (idx % (DV / 4)) * 4;
                    *reinterpret_cast<float4*>(fv + f * LDV + j) = load4(ref(fold_list[f0 + f]).v + j);
                }
                __syncthreads();
                for (int f = 0; f < nff; ++f) {
                    const float4 v4 = *reinterpret_cast<const float4*>(fv + f * LDV + 4 * ftx);
#pragma unroll
                    for (int i = 0; i < RPT; ++i) {
                        const float ph = fphi[f * Sh::LD + fty * RPT + i];
                        hreg[i][0] = fmaf(ph, v4.x, hreg[i][0]);
                        hreg[i][1] = fmaf(ph, v4.y, hreg[i][1]);
                        hreg[i][2] = fmaf(ph, v4.z, hreg[i][2]);
                        hreg[i][3] = fmaf(ph, v4.w, hreg[i][3]);
                    }
                }
                if (tid < D)
                    for (int f = 0; f < nff; ++f) sacc += fphi[f * Sh::LD + tid];
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < RPT; ++i)
                *reinterpret_cast<float4*>(Hs + (fty * RPT + i) * DV + 4 * ftx) =
                    make_float4(hreg[i][0], hreg[i][1], hreg[i][2], hreg[i][3]);
            if (tid < D) ss[tid] += sacc;
            for (int i = tid; i < n_l; i += kThreads)
                if (newslot[i] >= 0) slot_pos[newslot[i]] = l_lo + i;
        }
        __syncthreads();
        publish(c + 1);
        __syncthreads();
    }
    float* Ho = a.sp.H + (size_t)st * D * DV;
    float* so = a.sp.s + (size_t)st * D;
    for (int i = tid; i < D * DV / 4; i += kThreads)
        reinterpret_cast<float4*>(Ho)[i] = reinterpret_cast<const float4*>(Hs)[i];
    for (int i = tid; i < D; i += kThreads) so[i] = ss[i];
}

size_t scan_smem_bytes(const Dims& dm) {
    return (size_t)scan_offsets(dm.D, dm.d, dm.lam, dm.C).total * 4;
}

template <int D, int DV, typename TIn>
static cudaError_t launch_scan_t(const PrefillArgs& a, cudaStream_t s) {
    const size_t bytes = scan_smem_bytes(a.dm);
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<D, DV, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    scan_kernel<D, DV, TIn><<<a.dm.S, kThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_scan_d(const PrefillArgs& a, cudaStream_t s) {
    const int d = a.dm.d, D = a.dm.D;
    if (d == 64 && D == 64) return launch_scan_t<64, 64, TIn>(a, s);
    if (d == 64 && D == 128) return launch_scan_t<128, 64, TIn>(a, s);
    if (d == 128 && D == 64) return launch_scan_t<64, 128, TIn>(a, s);
    if (d == 128 && D == 128) return launch_scan_t<128, 128, TIn>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_scan(const PrefillArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_scan_d<__nv_bfloat16>(a, s) : launch_scan_d<float>(a, s);
}

}  // namespace lola

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
#include <cooperative_groups.h>

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
    const int tid = threadIdx.x, lane = tid & 31, NT = blockDim.x;
    for (int i = tid; i < n; i += NT) sbits[i] = __float_as_uint(score[i]);
    unsigned prefix = 0u, mask = 0u;
    int kk = lam;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
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
    for (int i = tid; i < n; i += NT) {
        const unsigned u = sbits[i];
        keep[i] = u > prefix ? 1 : 0;
        if (u == prefix) eq_list[atomicAdd(&tmp[2], 1)] = i;
    }
    __syncthreads();
    const int neq = tmp[2];
    for (int q = tid; q < neq; q += NT) {
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

// ---------------------------------------------------------------------------
// The same chain split over a thread-block cluster (one cluster per stream).
//
// CTA r of the cluster owns columns [r*CW, (r+1)*CW) of H.  Every CTA keeps
// the phi rows (and its columns of the value rows) of all cache members
// resident in shared memory, so a block only loads its C newcomers.  Per
// scored block each CTA computes the partial SRE of every candidate over its
// own columns; the partials are summed across the cluster through distributed
// shared memory in a fixed rank order, so every CTA holds bit-identical scores
// and takes the same (replicated) top-lambda decision; each CTA then folds
// into its own columns and publishes its rows of H_c^T.
// ---------------------------------------------------------------------------
constexpr int kClThreads = 256;

struct ClOffsets {
    int Hs, ss, phiC, vC, phiL, vL, part, den, score, slot_pos, cand_pos, flags, ranks, keep, free_slots,
        fold_list, tmp, hist, sbits, eq_list, newslot, sfold, total;
};

__host__ __device__ inline ClOffsets cl_offsets(int D, int CW, int lam, int C, int esize) {
    const int NMAX = lam + C, LD = D + 4;
    ClOffsets o;
    int p = 0;
    auto take = [&](int n) { int r = p; p += (n + 3) & ~3; return r; };
    o.Hs = take(D * CW);
    o.ss = take(D);
    o.phiC = take(lam * LD);
    o.vC = take((lam * CW * esize + 3) / 4);
    o.phiL = take(C * LD);
    o.vL = take((C * CW * esize + 3) / 4);
    o.part = take(2 * NMAX);
    o.den = take(NMAX);
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
    o.sfold = take(2 * C);
    o.total = p;
    return o;
}

template <int CW>
struct ClShape {
    static constexpr int TX = CW / 4;                          // threads across the CTA's columns
    static constexpr int TY = kClThreads / TX;
    static constexpr int EPT = CW >= 64 ? 8 : (CW == 32 ? 8 : (CW == 16 ? 4 : 2));
    static constexpr int TE = TY * EPT;                        // candidates per pass
};

template <int D, int CW, typename TIn>
__global__ void __launch_bounds__(kClThreads, 1) scan_cl_kernel(const __grid_constant__ PrefillArgs a) {
    namespace cg = cooperative_groups;
    using Sh = ClShape<CW>;
    constexpr int NT = kClThreads, LD = D + 4;
    cg::cluster_group cluster = cg::this_cluster();
    const int NCL = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int lam = dm.lam, C = dm.C, eta = dm.eta, DV = dm.d, NMAX = lam + C;
    const int st = blockIdx.x / NCL, b = st / dm.Hkv, g = st % dm.Hkv;
    const int col0 = rank * CW;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ClOffsets o = cl_offsets(D, CW, lam, C, (int)sizeof(TIn));
    float* Hs = smem + o.Hs;                                   // [D][CW]
    float* ss = smem + o.ss;
    float* phiC = smem + o.phiC;                               // [lam][LD]
    TIn* vC = reinterpret_cast<TIn*>(smem + o.vC);             // [lam][CW]
    float* phiL = smem + o.phiL;                               // [C][LD]
    TIn* vL = reinterpret_cast<TIn*>(smem + o.vL);             // [C][CW]
    float* part = smem + o.part;                               // [2][NMAX]
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
    float* sfold = smem + o.sfold;                             // fold staging: row offsets, values

    // ---- load the state: own columns of H, s, slot positions, resident rows ----
    const float* Hg = a.sp.H + (size_t)st * D * DV;
    for (int i = tid; i < D * CW; i += NT) Hs[i] = Hg[(size_t)(i / CW) * DV + col0 + i % CW];
    for (int i = tid; i < D; i += NT) ss[i] = a.sp.s[(size_t)st * D + i];
    for (int j = tid; j < lam; j += NT) slot_pos[j] = a.sp.cache_pos[(size_t)st * lam + j];
    __syncthreads();
    const int n_g0 = min(lam, max(0, a.t_start - eta));
    for (int idx = tid; idx < n_g0 * (D / 4); idx += NT) {
        const int e = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
        const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, slot_pos[e], e);
        *reinterpret_cast<float4*>(phiC + e * LD + j4) = *reinterpret_cast<const float4*>(r.phik + j4);
    }
    for (int idx = tid; idx < n_g0 * CW; idx += NT) {
        const int e = idx / CW, cl = idx % CW;
        vC[e * CW + cl] = pair_ref<TIn>(a, st, b, g, slot_pos[e], e).v[col0 + cl];
    }

    const size_t snaps = (size_t)dm.nc_max + 1;
    auto publish = [&](int c) {
        float* sH = a.snap_H + ((size_t)st * snaps + c) * D * DV;          // H_c^T [DV][D]
        for (int i = tid; i < CW * (D / 4); i += NT) {
            const int cl = i / (D / 4), j4 = (i % (D / 4)) * 4;
            reinterpret_cast<float4*>(sH + (size_t)(col0 + cl) * D)[j4 / 4] =
                make_float4(Hs[(j4 + 0) * CW + cl], Hs[(j4 + 1) * CW + cl], Hs[(j4 + 2) * CW + cl],
                            Hs[(j4 + 3) * CW + cl]);
        }
        if (rank == 0) {
            int* sp_ = a.snap_pos + ((size_t)st * snaps + c) * lam;
            float* sS = a.snap_s + ((size_t)st * snaps + c) * D;
            for (int j = tid; j < lam; j += NT) sp_[j] = slot_pos[j];
            for (int i = tid; i < D; i += NT) sS[i] = ss[i];
        }
    };
    __syncthreads();
    publish(0);

    int pb = 0;
    const int tx = tid % Sh::TX, ty = tid / Sh::TX;
    for (int c = 0; c < a.nc; ++c) {
        const int t0 = a.t_start + c * C;
        const int n_g = min(lam, max(0, t0 - eta));
        const int l_lo = max(0, t0 - eta), l_hi = max(0, t0 + C - eta);
        const int n_l = l_hi - l_lo;
        if (n_l > 0) {
            // newcomers (the pairs leaving the window): phi rows and own value columns
            for (int idx = tid; idx < n_l * (D / 4); idx += NT) {
                const int i = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
                const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, l_lo + i, 0);
                *reinterpret_cast<float4*>(phiL + i * LD + j4) = *reinterpret_cast<const float4*>(r.phik + j4);
            }
            for (int idx = tid; idx < n_l * CW; idx += NT) {
                const int i = idx / CW, cl = idx % CW;
                vL[i * CW + cl] = pair_ref<TIn>(a, st, b, g, l_lo + i, 0).v[col0 + cl];
            }
            __syncthreads();
            if (n_g + n_l <= lam) {
                // every candidate fits: all newcomers join (notes §2.4)
                for (int idx = tid; idx < n_l * (D / 4); idx += NT) {
                    const int i = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
                    *reinterpret_cast<float4*>(phiC + (n_g + i) * LD + j4) =
                        *reinterpret_cast<const float4*>(phiL + i * LD + j4);
                }
                for (int idx = tid; idx < n_l * CW; idx += NT) vC[n_g * CW + idx] = vL[idx];
                for (int i = tid; i < n_l; i += NT) slot_pos[n_g + i] = l_lo + i;
            } else {
                const int n = n_g + n_l;
                for (int i = tid; i < n; i += NT) cand_pos[i] = i < n_g ? slot_pos[i] : l_lo + (i - n_g);
                auto phirow = [&](int e) -> const float* { return e < n_g ? phiC + e * LD : phiL + (e - n_g) * LD; };
                auto vrow = [&](int e) -> const TIn* { return e < n_g ? vC + e * CW : vL + (e - n_g) * CW; };
                // den_e = phi_e . s (replicated in every CTA; one thread per candidate)
                for (int e = tid; e < n; e += NT) {
                    const float* pr = phirow(e);
                    float x = 0.f;
#pragma unroll 8
                    for (int j = 0; j < D; j += 4) {
                        const float4 f = *reinterpret_cast<const float4*>(pr + j);
                        const float4 t = *reinterpret_cast<const float4*>(ss + j);
                        x = fmaf(f.x, t.x, x); x = fmaf(f.y, t.y, x); x = fmaf(f.z, t.z, x); x = fmaf(f.w, t.w, x);
                    }
                    den[e] = x;
                }
                __syncthreads();
                // partial SRE over the CTA's columns
                float* mypart = part + pb * NMAX;
                for (int e0 = 0; e0 < n; e0 += Sh::TE) {
                    float acc[Sh::EPT][4];
                    const float* rows[Sh::EPT];
#pragma unroll
                    for (int i = 0; i < Sh::EPT; ++i) {
                        acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
                        const int e = e0 + ty + i * Sh::TY;
                        rows[i] = phirow(e < n ? e : 0);
                    }
                    for (int j = 0; j < D; j += 4) {
                        const float4 h0 = *reinterpret_cast<const float4*>(Hs + (j + 0) * CW + 4 * tx);
                        const float4 h1 = *reinterpret_cast<const float4*>(Hs + (j + 1) * CW + 4 * tx);
                        const float4 h2 = *reinterpret_cast<const float4*>(Hs + (j + 2) * CW + 4 * tx);
                        const float4 h3 = *reinterpret_cast<const float4*>(Hs + (j + 3) * CW + 4 * tx);
#pragma unroll
                        for (int i = 0; i < Sh::EPT; ++i) {
                            if (e0 + i * Sh::TY >= n) break;       // CTA-uniform: no candidate in this slot
                            const float4 f = *reinterpret_cast<const float4*>(rows[i] + j);
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
                        const int e = e0 + ty + i * Sh::TY;
                        float pt = 0.f;
                        if (e < n) {
                            const float dn = den[e];
                            const TIn* vr = vrow(e) + 4 * tx;
                            float pr[4] = {0.f, 0.f, 0.f, 0.f};
                            if (dn > 0.f) {
                                const float rdn = 1.f / dn;
#pragma unroll
                                for (int u = 0; u < 4; ++u) pr[u] = acc[i][u] * rdn;
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u) { const float r = pr[u] - to_f32(vr[u]); pt = fmaf(r, r, pt); }
                        }
#pragma unroll
                        for (int off = Sh::TX / 2; off > 0; off >>= 1) pt += __shfl_xor_sync(0xffffffffu, pt, off);
                        if (tx == 0 && e < n) mypart[e] = pt;
                    }
                }
                cluster.sync();                                 // partials visible cluster-wide
                for (int e = tid; e < n; e += NT) {
                    float sum = 0.f;
                    for (int r = 0; r < NCL; ++r) sum += cluster.map_shared_rank(mypart, r)[e];
                    score[e] = sum;
                }
                pb ^= 1;
                __syncthreads();
                if (lam > 0) {
                    select_top(score, cand_pos, n, lam, keep, sbits, hist, tmp, eq_list);
                } else {
                    for (int i = tid; i < n; i += NT) keep[i] = 0;
                    __syncthreads();
                }
                // slot bookkeeping, identical in every CTA
                for (int j = tid; j < lam; j += NT) flags[j] = (j >= n_g || keep[j] == 0) ? 1 : 0;
                __syncthreads();
                block_exscan(flags, ranks, lam, tmp);
                for (int j = tid; j < lam; j += NT) if (flags[j]) free_slots[ranks[j]] = j;
                __syncthreads();
                for (int i = tid; i < n_l; i += NT) flags[i] = keep[n_g + i];
                __syncthreads();
                block_exscan(flags, ranks, n_l, tmp);
                for (int i = tid; i < n_l; i += NT) newslot[i] = flags[i] ? free_slots[ranks[i]] : -1;
                __syncthreads();
                for (int e = tid; e < n; e += NT) flags[e] = keep[e] ? 0 : 1;
                __syncthreads();
                const int nf = block_exscan(flags, ranks, n, tmp);
                for (int e = tid; e < n; e += NT) if (flags[e]) fold_list[ranks[e]] = e;
                __syncthreads();
                // fold into the CTA's columns (notes §2.4, Eqs. 12-13): the folded rows are
                // staged contiguously, then each thread updates a block of H rows x 4
                // columns with an outer-product loop.
                int* foff = reinterpret_cast<int*>(sfold);         // [nf] phi-row offsets (floats)
                int* voff = foff + C;                              // [nf] value-row offsets (elements)
                for (int q = tid; q < nf; q += NT) {
                    foff[q] = (int)(phirow(fold_list[q]) - smem);
                    voff[q] = (int)(vrow(fold_list[q]) - reinterpret_cast<const TIn*>(smem));
                }
                __syncthreads();
                {
                    constexpr int FX = CW / 4, FY = NT / FX, RPT = (D + FY - 1) / FY;
                    const int fx = tid % FX, fy = tid / FX;
                    float hr[RPT][4];
#pragma unroll
                    for (int r = 0; r < RPT; ++r) {
                        const int j = fy + r * FY;
                        if (j < D) {
                            const float4 h4 = *reinterpret_cast<const float4*>(Hs + j * CW + 4 * fx);
                            hr[r][0] = h4.x; hr[r][1] = h4.y; hr[r][2] = h4.z; hr[r][3] = h4.w;
                        }
                    }
                    for (int q = 0; q < nf; ++q) {
                        const float4 v4 = load4(reinterpret_cast<const TIn*>(smem) + voff[q] + 4 * fx);
                        const float* fphi = smem + foff[q];
#pragma unroll
                        for (int r = 0; r < RPT; ++r) {
                            const int j = fy + r * FY;
                            if (j < D) {
                                const float ph = fphi[j];
                                hr[r][0] = fmaf(ph, v4.x, hr[r][0]); hr[r][1] = fmaf(ph, v4.y, hr[r][1]);
                                hr[r][2] = fmaf(ph, v4.z, hr[r][2]); hr[r][3] = fmaf(ph, v4.w, hr[r][3]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RPT; ++r) {
                        const int j = fy + r * FY;
                        if (j < D)
                            *reinterpret_cast<float4*>(Hs + j * CW + 4 * fx) =
                                make_float4(hr[r][0], hr[r][1], hr[r][2], hr[r][3]);
                    }
                }
                for (int j = tid; j < D; j += NT) {
                    float accs = 0.f;
                    for (int q = 0; q < nf; ++q) accs += smem[foff[q] + j];
                    ss[j] += accs;
                }
                __syncthreads();
                // retained newcomers move into the freed slots (resident rows follow)
                for (int idx = tid; idx < n_l * (D / 4); idx += NT) {
                    const int i = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
                    if (newslot[i] >= 0)
                        *reinterpret_cast<float4*>(phiC + newslot[i] * LD + j4) =
                            *reinterpret_cast<const float4*>(phiL + i * LD + j4);
                }
                for (int idx = tid; idx < n_l * CW; idx += NT) {
                    const int i = idx / CW, cl = idx % CW;
                    if (newslot[i] >= 0) vC[newslot[i] * CW + cl] = vL[i * CW + cl];
                }
                for (int i = tid; i < n_l; i += NT)
                    if (newslot[i] >= 0) slot_pos[newslot[i]] = l_lo + i;
            }
        }
        __syncthreads();
        publish(c + 1);
        __syncthreads();
    }
    float* Ho = a.sp.H + (size_t)st * D * DV;
    for (int i = tid; i < D * CW; i += NT) Ho[(size_t)(i / CW) * DV + col0 + i % CW] = Hs[i];
    if (rank == 0)
        for (int i = tid; i < D; i += NT) a.sp.s[(size_t)st * D + i] = ss[i];
    cluster.sync();                                             // peers may still read our partials
}

size_t scan_cl_smem_bytes(const Dims& dm, int CW) {
    return (size_t)cl_offsets(dm.D, CW, dm.lam, dm.C, dm.esize).total * 4;
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

template <int D, int CW, typename TIn>
static cudaError_t launch_scan_cl_t(const PrefillArgs& a, int ncl, cudaStream_t s) {
    const size_t bytes = scan_cl_smem_bytes(a.dm, CW);
    auto kern = scan_cl_kernel<D, CW, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && ncl > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.dm.S * ncl);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // every stream's cluster must be resident at once, or the chains run in waves
    int nclusters = 0;
    e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    if (e != cudaSuccess || nclusters < a.dm.S) { (void)cudaGetLastError(); return cudaErrorNotSupported; }
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D, typename TIn>
static cudaError_t launch_scan_cl_d(const PrefillArgs& a, int cw, int ncl, cudaStream_t s) {
    switch (cw) {
        case 8: return launch_scan_cl_t<D, 8, TIn>(a, ncl, s);
        case 16: return launch_scan_cl_t<D, 16, TIn>(a, ncl, s);
        case 32: return launch_scan_cl_t<D, 32, TIn>(a, ncl, s);
        case 64: return launch_scan_cl_t<D, 64, TIn>(a, ncl, s);
    }
    return cudaErrorNotSupported;
}

// Cluster size for a shape: the largest power of two <= 16 with the whole grid
// in one wave of SMs and the resident rows within shared memory; 0 = none.
static int pick_cluster(const Dims& dm, int num_sms) {
    for (int ncl = 16; ncl >= 2; ncl >>= 1) {
        const int cw = dm.d / ncl;
        if (cw < 8 || cw > 64) continue;
        if (dm.S * ncl > num_sms) continue;
        if (scan_cl_smem_bytes(dm, cw) > 227 * 1024) continue;
        return ncl;
    }
    return 0;
}

static int g_num_sms = 0;

cudaError_t launch_scan(const PrefillArgs& a, cudaStream_t s) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) g_num_sms = 1;
    }
    for (int ncl = pick_cluster(a.dm, g_num_sms); ncl >= 2; ncl >>= 1) {
        const int cw = a.dm.d / ncl;
        if (cw > 64 || scan_cl_smem_bytes(a.dm, cw) > 227 * 1024) break;
        cudaError_t e;
        if (a.dm.D == 128)
            e = a.dm.dtype == 1 ? launch_scan_cl_d<128, __nv_bfloat16>(a, cw, ncl, s) : launch_scan_cl_d<128, float>(a, cw, ncl, s);
        else
            e = a.dm.dtype == 1 ? launch_scan_cl_d<64, __nv_bfloat16>(a, cw, ncl, s) : launch_scan_cl_d<64, float>(a, cw, ncl, s);
        if (e != cudaErrorNotSupported) return e;                // launched (or a real error)
    }
    return a.dm.dtype == 1 ? launch_scan_d<__nv_bfloat16>(a, s) : launch_scan_d<float>(a, s);
}

}  // namespace lola

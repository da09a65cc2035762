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
// s += sum Phi_S with H held in registers.  Under an alternative scoring rule
// (notes §4.5, Table 4) the scores do not depend on the state: they come from
// the window-score kernel (scores.cu) and the chain only selects and folds.
#include <cooperative_groups.h>
#include <type_traits>

#include "chain_common.cuh"
#include "device_common.cuh"
#include "umma.cuh"

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
    const int* slots_in = entering_slots(a, st);
    for (int j = tid; j < lam; j += kThreads) slot_pos[j] = slots_in[j];
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
    if (a.c_begin == 0) publish(0);

    // fold-phase thread layout: rows ty*RPT.., columns 4tx..4tx+3
    constexpr int TXF = DV / 4, TYF = kThreads / TXF, RPT = D / TYF, TF = 32, LDV = DV + 4;
    const int ftx = tid % TXF, fty = tid / TXF;

    for (int c = a.c_begin; c < a.c_end; ++c) {
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
            if (lam > 0 && a.scorer != 0) {
                for (int e = tid; e < n; e += kThreads) score[e] = static_score(a, st, cand_pos[e], e);
                __syncthreads();
                select_top(score, cand_pos, n, lam, keep, sbits, hist, tmp, eq_list);
            } else if (lam > 0) {
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
// CTA r of the cluster owns columns [r*CW, (r+1)*CW) of H.  Every CTA keeps the
// phi rows, and its slice of the value rows, of the cache members in a pool of
// lambda + C shared-memory rows: a slot names a pool row, so a newcomer that
// enters the cache never moves, and the rows of folded pairs go back to a free
// stack from which the next block's newcomers are fetched with cp.async while
// the current block finishes.  Per scored block each CTA computes the partial
// SRE of every candidate over its own columns (cache members first, while the
// newcomers land); the partials are summed across the cluster through
// distributed shared memory by a fixed butterfly, so every CTA holds
// bit-identical scores and takes the same top-lambda decision (one warp selects
// and does the slot bookkeeping); each CTA then folds into its own columns and
// publishes its rows of H_c^T straight from registers.
// ---------------------------------------------------------------------------
constexpr int kClThreads = 256;

struct ClOffsets {
    int Hs, ss, phi, vv, part, score, cand_pos, cand_row, keep, slot_pos, slot_row, new_row, free_rows,
        fold_row, free_slots, hist, tmp, eq_list, total;
};

__host__ __device__ inline ClOffsets cl_offsets(int D, int CW, int lam, int C, int esize) {
    const int P = lam + C, LD = D + 4, N4 = (P + 3) & ~3;
    ClOffsets o;
    int p = 0;
    auto take = [&](int n) { int r = p; p += (n + 3) & ~3; return r; };
    o.Hs = take(D * CW);
    o.ss = take(D);
    o.phi = take(P * LD);
    o.vv = take((P * CW * esize + 3) / 4);
    o.part = take(2 * N4);
    o.score = take(N4);
    o.cand_pos = take(P);
    o.cand_row = take(P);
    o.keep = take(P);
    o.slot_pos = take(lam + 1);
    o.slot_row = take(lam + 1);
    o.new_row = take(C);
    o.free_rows = take(P);
    o.fold_row = take(P);
    o.free_slots = take(lam + 1);
    o.hist = take(256);
    o.tmp = take(32);
    o.eq_list = take(P);
    o.total = p;
    return o;
}

// Largest lambda + C the cluster scan handles (candidates held 32 per register).
template <int D>
struct ClMax {
    static constexpr int KMAX = D == 128 ? 14 : 28;
    static constexpr int NMAX = 32 * KMAX;
};

template <int D, int DV, int NCL, typename TIn>
__global__ void __launch_bounds__(kClThreads, 1) scan_cl_kernel(const __grid_constant__ PrefillArgs a) {
    namespace cg = cooperative_groups;
    constexpr int CW = DV / NCL, NT = kClThreads, NW = NT / 32, LD = D + 4;
    constexpr int CPT = 8, TX = CW / CPT, TY = NT / TX;       // SRE threads: 8 columns x EPT candidates
    constexpr int EPT = CW == 8 ? 2 : (CW == 16 ? 3 : (CW == 32 ? 5 : 8));
    constexpr int TE = TY * EPT;                              // candidates per SRE tile
    constexpr int VCH = CW * (int)sizeof(TIn) / 16;           // 16-byte pieces of a value slice
    static_assert(CW >= 8 && CW <= 64 && (CW * sizeof(TIn)) % 16 == 0 && VCH <= 32, "unsupported column split");
    static_assert(32 % NCL == 0, "butterfly groups must tile a warp");
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int lam = dm.lam, C = dm.C, eta = dm.eta, P = lam + C, N4 = (P + 3) & ~3;
    const int st = blockIdx.x / NCL, b = st / dm.Hkv, g = st % dm.Hkv;
    const int col0 = rank * CW;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ClOffsets o = cl_offsets(D, CW, lam, C, (int)sizeof(TIn));
    float* Hs = smem + o.Hs;                                   // [D][CW]
    float* ss = smem + o.ss;                                   // [D]
    float* phi = smem + o.phi;                                 // pool [P][LD]
    TIn* vv = reinterpret_cast<TIn*>(smem + o.vv);             // pool [P][CW]
    float* part = smem + o.part;                               // [2][N4] partial SRE
    float* score = smem + o.score;
    int* cand_pos = reinterpret_cast<int*>(smem + o.cand_pos);
    int* cand_row = reinterpret_cast<int*>(smem + o.cand_row);
    int* keep = reinterpret_cast<int*>(smem + o.keep);
    int* slot_pos = reinterpret_cast<int*>(smem + o.slot_pos);
    int* slot_row = reinterpret_cast<int*>(smem + o.slot_row);
    int* new_row = reinterpret_cast<int*>(smem + o.new_row);
    int* free_rows = reinterpret_cast<int*>(smem + o.free_rows);
    int* fold_row = reinterpret_cast<int*>(smem + o.fold_row);
    int* free_slots = reinterpret_cast<int*>(smem + o.free_slots);
    unsigned* hist = reinterpret_cast<unsigned*>(smem + o.hist);
    int* tmp = reinterpret_cast<int*>(smem + o.tmp);
    int* eq_list = reinterpret_cast<int*>(smem + o.eq_list);

    // cp.async the phi rows and this CTA's value slices of n_rows pairs into pool rows
    auto fetch = [&](int n_rows, auto pos_of, auto slot_of, auto row_of) {
        for (int i = warp; i < n_rows; i += NW) {                 // a warp per row
            const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, pos_of(i), slot_of(i));
            const int row = row_of(i);
            for (int q = lane; q < D / 4; q += 32) umma::cp_async16(phi + (size_t)row * LD + 4 * q, r.phik + 4 * q);
            if (lane < VCH)
                umma::cp_async16(reinterpret_cast<char*>(vv + (size_t)row * CW) + 16 * lane,
                                 reinterpret_cast<const char*>(r.v + col0) + 16 * lane);
        }
        umma::cp_async_commit();
    };

    // ---- state: own columns of H, s, slots, resident rows ----
    const float* Hg = a.sp.H + (size_t)st * D * DV;
    for (int i = tid; i < D * (CW / 4); i += NT) {
        const int j = i / (CW / 4), u = i % (CW / 4);
        umma::cp_async16(Hs + j * CW + 4 * u, Hg + (size_t)j * DV + col0 + 4 * u);
    }
    for (int i = tid; i < D / 4; i += NT) umma::cp_async16(ss + 4 * i, a.sp.s + (size_t)st * D + 4 * i);
    const int n_g0 = min(lam, max(0, a.t_start + a.c_begin * C - eta));
    const int* slots_in = entering_slots(a, st);
    for (int j = tid; j < lam; j += NT) {
        slot_pos[j] = slots_in[j];
        slot_row[j] = j;
    }
    for (int k = tid; k < P - n_g0; k += NT) free_rows[k] = P - 1 - k;      // popped from the top
    int nfree = P - n_g0;
    __syncthreads();
    fetch(n_g0, [&](int i) { return slot_pos[i]; }, [](int i) { return i; }, [](int i) { return i; });

    // the newcomers of block c (the pairs leaving the window) into rows from the free stack;
    // always commits one cp.async group
    auto prefetch = [&](int c) {
        int n_l = 0, l_lo = 0;
        if (c < a.c_end) {
            const int t0 = a.t_start + c * C;
            l_lo = max(0, t0 - eta);
            n_l = max(0, t0 + C - eta) - l_lo;
        }
        for (int i = tid; i < n_l; i += NT) new_row[i] = free_rows[nfree - 1 - i];
        fetch(n_l, [&](int i) { return l_lo + i; }, [](int) { return 0; },
              [&](int i) { return free_rows[nfree - 1 - i]; });
        nfree -= n_l;
    };
    prefetch(a.c_begin);

    const size_t snaps = (size_t)dm.nc_max + 1;
    auto snapH = [&](int c) { return a.snap_H + ((size_t)st * snaps + c) * D * DV; };   // H_c^T [DV][D]
    // slot positions by slices across the cluster, s by rank 0
    auto publish_pos_s = [&](int c, bool with_s) {
        int* sp_ = a.snap_pos + ((size_t)st * snaps + c) * lam;
        for (int j = rank * NT + tid; j < lam; j += NCL * NT) sp_[j] = slot_pos[j];
        if (with_s && rank == 0) {
            float* sS = a.snap_s + ((size_t)st * snaps + c) * D;
            for (int i = tid; i < D; i += NT) sS[i] = ss[i];
        }
    };
    auto publish_H = [&](int c) {
        float* sH = snapH(c);
        for (int i = tid; i < D * (CW / 4); i += NT) {
            const int j = i % D, u = i / D;
            const float4 h = *reinterpret_cast<const float4*>(Hs + j * CW + 4 * u);
            float* dst = sH + (size_t)(col0 + 4 * u) * D + j;
            dst[0] = h.x; dst[D] = h.y; dst[2 * D] = h.z; dst[3 * D] = h.w;
        }
    };
    umma::cp_async_wait<1>();                                  // state and resident rows landed
    __syncthreads();
    if (a.c_begin == 0) {
        publish_H(0);
        publish_pos_s(0, true);
    }

    // Partial SRE over this CTA's columns (notes §2.3, Eq. 10) of candidates [0, n):
    // for each candidate, den_e = phi_e . s and pred = H^T phi_e restricted to the
    // CTA's columns are accumulated in one pass over phi_e; the partial is
    // || pred / den_e - v_e ||^2 over those columns (the zero prediction when
    // den_e == 0).  Thread (tx, ty) takes 8 columns of EPT candidates with paired
    // fp32 FMAs; every thread of a tile works (out-of-range candidates repeat a
    // valid row and are not stored), so the inner loop has no branches.
    auto sre_all = [&](int n, float* mypart) {
        const int tx = tid % TX, ty = tid / TX;
        const float* hb = Hs + CPT * tx;
        for (int e0 = 0; e0 < n; e0 += TE) {
            unsigned long long a2[EPT][CPT / 2];
            float d0[EPT], d1[EPT];
            const float* rows[EPT];
#pragma unroll
            for (int i = 0; i < EPT; ++i) {
#pragma unroll
                for (int u = 0; u < CPT / 2; ++u) a2[i][u] = 0ull;
                d0[i] = d1[i] = 0.f;
                rows[i] = phi + (size_t)cand_row[min(e0 + ty + i * TY, n - 1)] * LD;
            }
#pragma unroll 2
            for (int j = 0; j < D; j += 4) {
                float4 h[4][2];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    h[r][0] = *reinterpret_cast<const float4*>(hb + (j + r) * CW);
                    h[r][1] = *reinterpret_cast<const float4*>(hb + (j + r) * CW + 4);
                }
                const float4 s4 = *reinterpret_cast<const float4*>(ss + j);
#pragma unroll
                for (int i = 0; i < EPT; ++i) {
                    const float4 f = *reinterpret_cast<const float4*>(rows[i] + j);
                    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const unsigned long long ff = f2pack(fv[r], fv[r]);
                        a2[i][0] = f2fma(ff, f2pack(h[r][0].x, h[r][0].y), a2[i][0]);
                        a2[i][1] = f2fma(ff, f2pack(h[r][0].z, h[r][0].w), a2[i][1]);
                        a2[i][2] = f2fma(ff, f2pack(h[r][1].x, h[r][1].y), a2[i][2]);
                        a2[i][3] = f2fma(ff, f2pack(h[r][1].z, h[r][1].w), a2[i][3]);
                    }
                    d0[i] = fmaf(f.x, s4.x, d0[i]); d1[i] = fmaf(f.y, s4.y, d1[i]);
                    d0[i] = fmaf(f.z, s4.z, d0[i]); d1[i] = fmaf(f.w, s4.w, d1[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < EPT; ++i) {
                const int e = e0 + ty + i * TY;
                float pt = 0.f;
                if (e < n) {
                    float acc[CPT];
#pragma unroll
                    for (int u = 0; u < CPT / 2; ++u) f2unpack(a2[i][u], acc[2 * u], acc[2 * u + 1]);
                    const float dn = d0[i] + d1[i];
                    const TIn* vr = vv + (size_t)cand_row[e] * CW + CPT * tx;
                    const float4 va = load4(vr), vb = load4(vr + 4);
                    const float vf[CPT] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
                    float pr[CPT];
#pragma unroll
                    for (int u = 0; u < CPT; ++u) pr[u] = 0.f;
                    if (dn > 0.f) {
                        const float rdn = 1.f / dn;
#pragma unroll
                        for (int u = 0; u < CPT; ++u) pr[u] = acc[u] * rdn;
                    }
#pragma unroll
                    for (int u = 0; u < CPT; ++u) { const float r = pr[u] - vf[u]; pt = fmaf(r, r, pt); }
                }
#pragma unroll
                for (int off = TX / 2; off > 0; off >>= 1) pt += __shfl_xor_sync(0xffffffffu, pt, off);
                if (tx == 0 && e < n) mypart[e] = pt;
            }
        }
    };

    int pb = 0;
    for (int c = a.c_begin; c < a.c_end; ++c) {
        const int t0 = a.t_start + c * C;
        const int n_g = min(lam, max(0, t0 - eta));
        const int l_lo = max(0, t0 - eta), n_l = max(0, t0 + C - eta) - l_lo;
        const int n = n_g + n_l;
        const bool scored = n_l > 0 && n > lam;
        if (n_l > 0 && !scored) {
            // every candidate fits: all newcomers join, in their pool rows (notes §2.4)
            for (int i = tid; i < n_l; i += NT) {
                slot_row[n_g + i] = new_row[i];
                slot_pos[n_g + i] = l_lo + i;
            }
        } else if (scored) {
            for (int e = tid; e < n; e += NT) {
                cand_pos[e] = e < n_g ? slot_pos[e] : l_lo + (e - n_g);
                cand_row[e] = e < n_g ? slot_row[e] : new_row[e - n_g];
            }
            __syncthreads();
            float* mypart = part + pb * N4;
            umma::cp_async_wait<0>();                          // the newcomers have landed
            __syncthreads();
            if (lam > 0 && a.scorer != 0) {
                // alternative rules: the window scores, read alike by every CTA of the cluster
                for (int e = tid; e < n; e += NT) score[e] = static_score(a, st, cand_pos[e], e);
                __syncthreads();
            } else if (lam > 0) {
                sre_all(n, mypart);
                cluster.sync();                                // partials visible cluster-wide
                // score_e = sum of the cluster's partials, by a butterfly over NCL lanes
                constexpr int GPW = 32 / NCL, KB = 4;
                const int r = lane % NCL, gs = lane / NCL;
                const float4* src = reinterpret_cast<const float4*>(cluster.map_shared_rank(mypart, r));
                const int G4 = (n + 3) / 4;
                for (int gw = warp * GPW; gw < G4; gw += KB * NW * GPW) {     // warp-uniform trip count
                    float4 x[KB];
#pragma unroll
                    for (int k = 0; k < KB; ++k) {
                        const int gi = gw + k * NW * GPW + gs;
                        x[k] = gi < G4 ? src[gi] : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int k = 0; k < KB; ++k) {
#pragma unroll
                        for (int off = NCL / 2; off > 0; off >>= 1) {
                            x[k].x += __shfl_xor_sync(0xffffffffu, x[k].x, off);
                            x[k].y += __shfl_xor_sync(0xffffffffu, x[k].y, off);
                            x[k].z += __shfl_xor_sync(0xffffffffu, x[k].z, off);
                            x[k].w += __shfl_xor_sync(0xffffffffu, x[k].w, off);
                        }
                        const int gi = gw + k * NW * GPW + gs;
                        if (r == 0 && gi < G4) reinterpret_cast<float4*>(score)[gi] = x[k];
                    }
                }
                pb ^= 1;
                __syncthreads();
            }
            if (warp == 0) {
                const int nfo = select_and_place<ClMax<D>::KMAX, true>(
                    score, cand_pos, cand_row, n, n_g, n_l, lam, l_lo, new_row, slot_row, slot_pos, fold_row,
                    free_rows, nfree, P, free_slots, hist, eq_list, keep);
                if (lane == 0) tmp[0] = nfo;
            }
            __syncthreads();
            const int nf = tmp[0];
            // fold into this CTA's columns (notes §2.4, Eqs. 12-13) and publish H_{c+1}^T
            // and s_{c+1}: a thread owns H[j][8 columns] (paired FMAs); the threads of
            // column group 0 also carry s[j].  Folded rows are taken four at a time.
            {
                float* sH = snapH(c + 1);
                float* sS = a.snap_s + ((size_t)st * snaps + (c + 1)) * D;
                const int nf4 = nf & ~3;
                for (int it = tid; it < D * (CW / 8); it += NT) {
                    const int j = it % D, c8 = (it / D) * 8;
                    float* hp = Hs + j * CW + c8;
                    const float4 h0 = *reinterpret_cast<const float4*>(hp), h1 = *reinterpret_cast<const float4*>(hp + 4);
                    unsigned long long h2[4] = {f2pack(h0.x, h0.y), f2pack(h0.z, h0.w), f2pack(h1.x, h1.y), f2pack(h1.z, h1.w)};
                    float sacc = 0.f;
                    int q = 0;
                    for (; q < nf4; q += 4) {
                        const int4 r4 = *reinterpret_cast<const int4*>(fold_row + q);
                        const int rr[4] = {r4.x, r4.y, r4.z, r4.w};
                        float p[4];
                        float4 va[4], vb[4];
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            p[t] = phi[(size_t)rr[t] * LD + j];
                            va[t] = load4(vv + (size_t)rr[t] * CW + c8);
                            vb[t] = load4(vv + (size_t)rr[t] * CW + c8 + 4);
                        }
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const unsigned long long pp = f2pack(p[t], p[t]);
                            h2[0] = f2fma(pp, f2pack(va[t].x, va[t].y), h2[0]);
                            h2[1] = f2fma(pp, f2pack(va[t].z, va[t].w), h2[1]);
                            h2[2] = f2fma(pp, f2pack(vb[t].x, vb[t].y), h2[2]);
                            h2[3] = f2fma(pp, f2pack(vb[t].z, vb[t].w), h2[3]);
                            sacc += p[t];
                        }
                    }
                    for (; q < nf; ++q) {
                        const int r = fold_row[q];
                        const float p0 = phi[(size_t)r * LD + j];
                        const float4 va = load4(vv + (size_t)r * CW + c8), vb = load4(vv + (size_t)r * CW + c8 + 4);
                        const unsigned long long pp = f2pack(p0, p0);
                        h2[0] = f2fma(pp, f2pack(va.x, va.y), h2[0]);
                        h2[1] = f2fma(pp, f2pack(va.z, va.w), h2[1]);
                        h2[2] = f2fma(pp, f2pack(vb.x, vb.y), h2[2]);
                        h2[3] = f2fma(pp, f2pack(vb.z, vb.w), h2[3]);
                        sacc += p0;
                    }
                    float hv[8];
#pragma unroll
                    for (int u = 0; u < 4; ++u) f2unpack(h2[u], hv[2 * u], hv[2 * u + 1]);
                    *reinterpret_cast<float4*>(hp) = make_float4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<float4*>(hp + 4) = make_float4(hv[4], hv[5], hv[6], hv[7]);
                    float* dst = sH + (size_t)(col0 + c8) * D + j;
#pragma unroll
                    for (int u = 0; u < 8; ++u) dst[(size_t)u * D] = hv[u];
                    if (c8 == 0) {
                        const float sj = ss[j] + sacc;
                        ss[j] = sj;
                        if (rank == 0) sS[j] = sj;
                    }
                }
            }
            nfree += nf;
            publish_pos_s(c + 1, false);
        }
        __syncthreads();
        prefetch(c + 1);
        if (!scored) {
            publish_H(c + 1);
            publish_pos_s(c + 1, true);
        }
        __syncthreads();                                       // the next block may change slot_pos
    }
    float* Ho = a.sp.H + (size_t)st * D * DV;
    for (int i = tid; i < D * CW; i += NT) Ho[(size_t)(i / CW) * DV + col0 + i % CW] = Hs[i];
    if (rank == 0)
        for (int i = tid; i < D; i += NT) a.sp.s[(size_t)st * D + i] = ss[i];
    umma::cp_async_wait<0>();
    cluster.sync();                                             // peers may still read our partials
}

// ---------------------------------------------------------------------------
// The chain over a cluster with the candidate rows left in global memory, for
// shapes whose lambda + C rows do not fit a shared-memory pool.  Same column
// split, cluster reduction, selection and fold as scan_cl_kernel; each scored
// block streams the candidates' phi rows and the CTA's value columns through a
// double-buffered shared-memory tile with cp.async (a stream's rows stay in L2
// from block to block), and stages the folded rows the same way.
// ---------------------------------------------------------------------------
constexpr int kCgTile = 128;          // candidate rows per tile
constexpr int kCgKmax = 48;           // lambda + C <= 32 * kCgKmax

struct CgOffsets {
    int Hs, ss, tphi, tv, part, score, cand_pos, keep, slot_pos, free_slots, fold_e, hist, tmp, eq_list, total;
};

__host__ __device__ inline CgOffsets cg_offsets(int D, int CW, int lam, int C, int esize) {
    const int P = lam + C, LD = D + 4, N4 = (P + 3) & ~3;
    CgOffsets o;
    int p = 0;
    auto take = [&](int n) { int r = p; p += (n + 3) & ~3; return r; };
    o.Hs = take(D * CW);
    o.ss = take(D);
    o.tphi = take(2 * kCgTile * LD);
    o.tv = take((2 * kCgTile * CW * esize + 3) / 4);
    o.part = take(2 * N4);
    o.score = take(N4);
    o.cand_pos = take(P);
    o.keep = take(P);
    o.slot_pos = take(lam + 1);
    o.free_slots = take(lam + 1);
    o.fold_e = take(P);
    o.hist = take(256);
    o.tmp = take(32);
    o.eq_list = take(P);
    o.total = p;
    return o;
}

template <int D, int DV, int NCL, typename TIn>
__global__ void __launch_bounds__(kClThreads, 1) scan_cg_kernel(const __grid_constant__ PrefillArgs a) {
    namespace cg = cooperative_groups;
    constexpr int CW = DV / NCL, NT = kClThreads, NW = NT / 32, LD = D + 4, TL = kCgTile;
    constexpr int CPT = 8, TX = CW / CPT, TY = NT / TX, EPT = TL / TY;   // one tile = one SRE pass
    constexpr int VCH = CW * (int)sizeof(TIn) / 16;                     // 16-byte pieces of a value slice
    constexpr int HI = D * (CW / 8), ITEMS = (HI + NT - 1) / NT;         // fold items per thread
    static_assert(CW >= 16 && CW <= 64 && TY * EPT == TL && VCH <= 32, "unsupported column split");
    static_assert(32 % NCL == 0, "butterfly groups must tile a warp");
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int lam = dm.lam, C = dm.C, eta = dm.eta, P = lam + C, N4 = (P + 3) & ~3;
    const int st = blockIdx.x / NCL, b = st / dm.Hkv, g = st % dm.Hkv;
    const int col0 = rank * CW;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const CgOffsets o = cg_offsets(D, CW, lam, C, (int)sizeof(TIn));
    float* Hs = smem + o.Hs;                                   // [D][CW]
    float* ss = smem + o.ss;                                   // [D]
    float* tphi = smem + o.tphi;                               // [2][TL][LD]
    TIn* tv = reinterpret_cast<TIn*>(smem + o.tv);             // [2][TL][CW]
    float* part = smem + o.part;                               // [2][N4]
    float* score = smem + o.score;
    int* cand_pos = reinterpret_cast<int*>(smem + o.cand_pos);
    int* keep = reinterpret_cast<int*>(smem + o.keep);
    int* slot_pos = reinterpret_cast<int*>(smem + o.slot_pos);
    int* free_slots = reinterpret_cast<int*>(smem + o.free_slots);
    int* fold_e = reinterpret_cast<int*>(smem + o.fold_e);
    unsigned* hist = reinterpret_cast<unsigned*>(smem + o.hist);
    int* tmp = reinterpret_cast<int*>(smem + o.tmp);
    int* eq_list = reinterpret_cast<int*>(smem + o.eq_list);

    // cp.async the phi rows and this CTA's value slices of nr candidates (list
    // index i -> candidate cand(i)) into tile buffer bi; always commits a group
    auto load_tile = [&](int bi, int nr, auto cand) {
        float* ph = tphi + (size_t)bi * TL * LD;
        TIn* vb = tv + (size_t)bi * TL * CW;
        for (int i = warp; i < nr; i += NW) {
            const int e = cand(i);
            const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, cand_pos[e], e);
            for (int q = lane; q < D / 4; q += 32) umma::cp_async16(ph + (size_t)i * LD + 4 * q, r.phik + 4 * q);
            if (lane < VCH)
                umma::cp_async16(reinterpret_cast<char*>(vb + (size_t)i * CW) + 16 * lane,
                                 reinterpret_cast<const char*>(r.v + col0) + 16 * lane);
        }
        umma::cp_async_commit();
    };

    const float* Hg = a.sp.H + (size_t)st * D * DV;
    for (int i = tid; i < D * (CW / 4); i += NT) {
        const int j = i / (CW / 4), u = i % (CW / 4);
        umma::cp_async16(Hs + j * CW + 4 * u, Hg + (size_t)j * DV + col0 + 4 * u);
    }
    for (int i = tid; i < D / 4; i += NT) umma::cp_async16(ss + 4 * i, a.sp.s + (size_t)st * D + 4 * i);
    umma::cp_async_commit();
    const int* slots_in = entering_slots(a, st);
    for (int j = tid; j < lam; j += NT) slot_pos[j] = slots_in[j];
    umma::cp_async_wait<0>();
    __syncthreads();

    const size_t snaps = (size_t)dm.nc_max + 1;
    auto snapH = [&](int c) { return a.snap_H + ((size_t)st * snaps + c) * D * DV; };
    auto publish_pos_s = [&](int c, bool with_s) {
        int* sp_ = a.snap_pos + ((size_t)st * snaps + c) * lam;
        for (int j = rank * NT + tid; j < lam; j += NCL * NT) sp_[j] = slot_pos[j];
        if (with_s && rank == 0) {
            float* sS = a.snap_s + ((size_t)st * snaps + c) * D;
            for (int i = tid; i < D; i += NT) sS[i] = ss[i];
        }
    };
    auto publish_H = [&](int c) {
        float* sH = snapH(c);
        for (int i = tid; i < D * (CW / 4); i += NT) {
            const int j = i % D, u = i / D;
            const float4 h = *reinterpret_cast<const float4*>(Hs + j * CW + 4 * u);
            float* dst = sH + (size_t)(col0 + 4 * u) * D + j;
            dst[0] = h.x; dst[D] = h.y; dst[2 * D] = h.z; dst[3 * D] = h.w;
        }
    };
    if (a.c_begin == 0) {
        publish_H(0);
        publish_pos_s(0, true);
    }

    // partial SRE (notes §2.3, Eq. 10) of the cnt candidates e0.. held in tile bi;
    // thread (tx, ty) takes 8 columns of EPT rows, out-of-range rows repeat a valid one
    auto sre_tile_cg = [&](int bi, int e0, int cnt, float* mypart) {
        const float* ph = tphi + (size_t)bi * TL * LD;
        const TIn* vb = tv + (size_t)bi * TL * CW;
        const int tx = tid % TX, ty = tid / TX;
        const float* hb = Hs + CPT * tx;
        unsigned long long a2[EPT][CPT / 2];
        float d0[EPT], d1[EPT];
        const float* rows[EPT];
#pragma unroll
        for (int i = 0; i < EPT; ++i) {
#pragma unroll
            for (int u = 0; u < CPT / 2; ++u) a2[i][u] = 0ull;
            d0[i] = d1[i] = 0.f;
            rows[i] = ph + (size_t)min(ty + i * TY, cnt - 1) * LD;
        }
#pragma unroll 2
        for (int j = 0; j < D; j += 4) {
            float4 h[4][2];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                h[r][0] = *reinterpret_cast<const float4*>(hb + (j + r) * CW);
                h[r][1] = *reinterpret_cast<const float4*>(hb + (j + r) * CW + 4);
            }
            const float4 s4 = *reinterpret_cast<const float4*>(ss + j);
#pragma unroll
            for (int i = 0; i < EPT; ++i) {
                const float4 f = *reinterpret_cast<const float4*>(rows[i] + j);
                const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const unsigned long long ff = f2pack(fv[r], fv[r]);
                    a2[i][0] = f2fma(ff, f2pack(h[r][0].x, h[r][0].y), a2[i][0]);
                    a2[i][1] = f2fma(ff, f2pack(h[r][0].z, h[r][0].w), a2[i][1]);
                    a2[i][2] = f2fma(ff, f2pack(h[r][1].x, h[r][1].y), a2[i][2]);
                    a2[i][3] = f2fma(ff, f2pack(h[r][1].z, h[r][1].w), a2[i][3]);
                }
                d0[i] = fmaf(f.x, s4.x, d0[i]); d1[i] = fmaf(f.y, s4.y, d1[i]);
                d0[i] = fmaf(f.z, s4.z, d0[i]); d1[i] = fmaf(f.w, s4.w, d1[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < EPT; ++i) {
            const int li = ty + i * TY;
            float pt = 0.f;
            if (li < cnt) {
                float acc[CPT];
#pragma unroll
                for (int u = 0; u < CPT / 2; ++u) f2unpack(a2[i][u], acc[2 * u], acc[2 * u + 1]);
                const float dn = d0[i] + d1[i];
                const TIn* vr = vb + (size_t)li * CW + CPT * tx;
                const float4 va = load4(vr), vc = load4(vr + 4);
                const float vf[CPT] = {va.x, va.y, va.z, va.w, vc.x, vc.y, vc.z, vc.w};
                float pr[CPT];
#pragma unroll
                for (int u = 0; u < CPT; ++u) pr[u] = 0.f;
                if (dn > 0.f) {
                    const float rdn = 1.f / dn;
#pragma unroll
                    for (int u = 0; u < CPT; ++u) pr[u] = acc[u] * rdn;
                }
#pragma unroll
                for (int u = 0; u < CPT; ++u) { const float r = pr[u] - vf[u]; pt = fmaf(r, r, pt); }
            }
#pragma unroll
            for (int off = TX / 2; off > 0; off >>= 1) pt += __shfl_xor_sync(0xffffffffu, pt, off);
            if (tx == 0 && li < cnt) mypart[e0 + li] = pt;
        }
    };

    int pb = 0;
    for (int c = a.c_begin; c < a.c_end; ++c) {
        const int t0 = a.t_start + c * C;
        const int n_g = min(lam, max(0, t0 - eta));
        const int l_lo = max(0, t0 - eta), n_l = max(0, t0 + C - eta) - l_lo;
        const int n = n_g + n_l;
        const bool scored = n_l > 0 && n > lam;
        if (n_l > 0 && !scored) {
            for (int i = tid; i < n_l; i += NT) slot_pos[n_g + i] = l_lo + i;   // all join (notes §2.4)
        } else if (scored) {
            for (int e = tid; e < n; e += NT) cand_pos[e] = e < n_g ? slot_pos[e] : l_lo + (e - n_g);
            __syncthreads();
            float* mypart = part + pb * N4;
            if (lam > 0) {
                const int ntile = (n + TL - 1) / TL;
                load_tile(0, min(TL, n), [](int i) { return i; });
                for (int t = 0; t < ntile; ++t) {
                    if (t + 1 < ntile)
                        load_tile((t + 1) & 1, min(TL, n - (t + 1) * TL), [t](int i) { return (t + 1) * TL + i; });
                    else
                        umma::cp_async_commit();
                    umma::cp_async_wait<1>();                  // tile t has landed
                    __syncthreads();
                    sre_tile_cg(t & 1, t * TL, min(TL, n - t * TL), mypart);
                    __syncthreads();                           // tile t's buffer is free again
                }
                cluster.sync();                                // partials visible cluster-wide
                constexpr int GPW = 32 / NCL, KB = 4;
                const int r = lane % NCL, gs = lane / NCL;
                const float4* src = reinterpret_cast<const float4*>(cluster.map_shared_rank(mypart, r));
                const int G4 = (n + 3) / 4;
                for (int gw = warp * GPW; gw < G4; gw += KB * NW * GPW) {     // warp-uniform trip count
                    float4 x[KB];
#pragma unroll
                    for (int k = 0; k < KB; ++k) {
                        const int gi = gw + k * NW * GPW + gs;
                        x[k] = gi < G4 ? src[gi] : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int k = 0; k < KB; ++k) {
#pragma unroll
                        for (int off = NCL / 2; off > 0; off >>= 1) {
                            x[k].x += __shfl_xor_sync(0xffffffffu, x[k].x, off);
                            x[k].y += __shfl_xor_sync(0xffffffffu, x[k].y, off);
                            x[k].z += __shfl_xor_sync(0xffffffffu, x[k].z, off);
                            x[k].w += __shfl_xor_sync(0xffffffffu, x[k].w, off);
                        }
                        const int gi = gw + k * NW * GPW + gs;
                        if (r == 0 && gi < G4) reinterpret_cast<float4*>(score)[gi] = x[k];
                    }
                }
                pb ^= 1;
                __syncthreads();
            }
            if (warp == 0) {
                const int nfo = select_and_place<kCgKmax, false>(
                    score, cand_pos, nullptr, n, n_g, n_l, lam, l_lo, nullptr, nullptr, slot_pos, fold_e,
                    nullptr, 0, P, free_slots, hist, eq_list, keep);
                if (lane == 0) tmp[0] = nfo;
            }
            __syncthreads();
            const int nf = tmp[0];
            // fold (notes §2.4, Eqs. 12-13), folded rows streamed through the tiles: a
            // thread owns ITEMS x (row j, 8 columns) of H; column group 0 also carries s[j]
            unsigned long long h2[ITEMS][4];
            float sacc[ITEMS];
#pragma unroll
            for (int k = 0; k < ITEMS; ++k) {
                const int it = tid + k * NT;
                sacc[k] = 0.f;
                if (it < HI) {
                    const float* hp = Hs + (it % D) * CW + (it / D) * 8;
                    const float4 h0 = *reinterpret_cast<const float4*>(hp), h1 = *reinterpret_cast<const float4*>(hp + 4);
                    h2[k][0] = f2pack(h0.x, h0.y); h2[k][1] = f2pack(h0.z, h0.w);
                    h2[k][2] = f2pack(h1.x, h1.y); h2[k][3] = f2pack(h1.z, h1.w);
                }
            }
            const int nft = (nf + TL - 1) / TL;
            if (nft > 0) load_tile(0, min(TL, nf), [&](int i) { return fold_e[i]; });
            for (int t = 0; t < nft; ++t) {
                if (t + 1 < nft)
                    load_tile((t + 1) & 1, min(TL, nf - (t + 1) * TL), [&, t](int i) { return fold_e[(t + 1) * TL + i]; });
                else
                    umma::cp_async_commit();
                umma::cp_async_wait<1>();
                __syncthreads();
                const float* ph = tphi + (size_t)(t & 1) * TL * LD;
                const TIn* vb = tv + (size_t)(t & 1) * TL * CW;
                const int cnt = min(TL, nf - t * TL);
#pragma unroll
                for (int k = 0; k < ITEMS; ++k) {
                    const int it = tid + k * NT;
                    if (it >= HI) continue;
                    const int j = it % D, c8 = (it / D) * 8;
                    for (int q = 0; q < cnt; ++q) {
                        const float p0 = ph[(size_t)q * LD + j];
                        const float4 va = load4(vb + (size_t)q * CW + c8), vc = load4(vb + (size_t)q * CW + c8 + 4);
                        const unsigned long long pp = f2pack(p0, p0);
                        h2[k][0] = f2fma(pp, f2pack(va.x, va.y), h2[k][0]);
                        h2[k][1] = f2fma(pp, f2pack(va.z, va.w), h2[k][1]);
                        h2[k][2] = f2fma(pp, f2pack(vc.x, vc.y), h2[k][2]);
                        h2[k][3] = f2fma(pp, f2pack(vc.z, vc.w), h2[k][3]);
                        sacc[k] += p0;
                    }
                }
                __syncthreads();
            }
            {
                float* sH = snapH(c + 1);
                float* sS = a.snap_s + ((size_t)st * snaps + (c + 1)) * D;
#pragma unroll
                for (int k = 0; k < ITEMS; ++k) {
                    const int it = tid + k * NT;
                    if (it >= HI) continue;
                    const int j = it % D, c8 = (it / D) * 8;
                    float hv[8];
#pragma unroll
                    for (int u = 0; u < 4; ++u) f2unpack(h2[k][u], hv[2 * u], hv[2 * u + 1]);
                    float* hp = Hs + j * CW + c8;
                    *reinterpret_cast<float4*>(hp) = make_float4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<float4*>(hp + 4) = make_float4(hv[4], hv[5], hv[6], hv[7]);
                    float* dst = sH + (size_t)(col0 + c8) * D + j;
#pragma unroll
                    for (int u = 0; u < 8; ++u) dst[(size_t)u * D] = hv[u];
                    if (c8 == 0) {
                        const float sj = ss[j] + sacc[k];
                        ss[j] = sj;
                        if (rank == 0) sS[j] = sj;
                    }
                }
            }
            publish_pos_s(c + 1, false);
        }
        __syncthreads();
        if (!scored) {
            publish_H(c + 1);
            publish_pos_s(c + 1, true);
        }
        __syncthreads();                                       // the next block may change slot_pos
    }
    float* Ho = a.sp.H + (size_t)st * D * DV;
    for (int i = tid; i < D * CW; i += NT) Ho[(size_t)(i / CW) * DV + col0 + i % CW] = Hs[i];
    if (rank == 0)
        for (int i = tid; i < D; i += NT) a.sp.s[(size_t)st * D + i] = ss[i];
    umma::cp_async_wait<0>();
    cluster.sync();                                             // peers may still read our partials
}

size_t scan_cg_smem_bytes(const Dims& dm, int CW) {
    return (size_t)cg_offsets(dm.D, CW, dm.lam, dm.C, dm.esize).total * 4;
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

template <int D, int DV, int NCL, typename TIn>
static cudaError_t launch_scan_cl_t(const PrefillArgs& a, cudaStream_t s) {
    const size_t bytes = scan_cl_smem_bytes(a.dm, DV / NCL);
    auto kern = scan_cl_kernel<D, DV, NCL, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && NCL > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.dm.S * NCL);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NCL;
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
static cudaError_t launch_scan_cl_d(const PrefillArgs& a, int ncl, cudaStream_t s) {
    if (a.dm.d == 128) {
        switch (ncl) {
            case 2: return launch_scan_cl_t<D, 128, 2, TIn>(a, s);
            case 4: return launch_scan_cl_t<D, 128, 4, TIn>(a, s);
            case 8: return launch_scan_cl_t<D, 128, 8, TIn>(a, s);
            case 16: return launch_scan_cl_t<D, 128, 16, TIn>(a, s);
        }
    } else if (a.dm.d == 64) {
        switch (ncl) {
            case 2: return launch_scan_cl_t<D, 64, 2, TIn>(a, s);
            case 4: return launch_scan_cl_t<D, 64, 4, TIn>(a, s);
            case 8: return launch_scan_cl_t<D, 64, 8, TIn>(a, s);
        }
    }
    return cudaErrorNotSupported;
}

// Cluster size for a shape: the largest power of two <= 16 with the whole grid
// in one wave of SMs and the row pool within shared memory; 0 = none.
static int pick_cluster(const Dims& dm, int num_sms) {
    for (int ncl = 16; ncl >= 2; ncl >>= 1) {
        const int cw = dm.d / ncl;
        if (cw < 8 || cw > 64) continue;
        if (dm.S * ncl > num_sms) continue;
        if (scan_cl_smem_bytes(dm, cw) > 227 * 1024) continue;
        if (dm.lam + dm.C > (dm.D == 128 ? ClMax<128>::NMAX : ClMax<64>::NMAX)) continue;
        return ncl;
    }
    return 0;
}

template <int D, int DV, int NCL, typename TIn>
static cudaError_t launch_scan_cg_t(const PrefillArgs& a, cudaStream_t s) {
    const size_t bytes = scan_cg_smem_bytes(a.dm, DV / NCL);
    auto kern = scan_cg_kernel<D, DV, NCL, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && NCL > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.dm.S * NCL);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NCL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    if (e != cudaSuccess || nclusters < a.dm.S) { (void)cudaGetLastError(); return cudaErrorNotSupported; }
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D, typename TIn>
static cudaError_t launch_scan_cg_d(const PrefillArgs& a, int ncl, cudaStream_t s) {
    if (a.dm.d == 128) {
        switch (ncl) {
            case 2: return launch_scan_cg_t<D, 128, 2, TIn>(a, s);
            case 4: return launch_scan_cg_t<D, 128, 4, TIn>(a, s);
            case 8: return launch_scan_cg_t<D, 128, 8, TIn>(a, s);
        }
    } else if (a.dm.d == 64) {
        switch (ncl) {
            case 2: return launch_scan_cg_t<D, 64, 2, TIn>(a, s);
            case 4: return launch_scan_cg_t<D, 64, 4, TIn>(a, s);
        }
    }
    return cudaErrorNotSupported;
}

static int g_num_sms = 0;

cudaError_t launch_scan(const PrefillArgs& a, cudaStream_t s) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) g_num_sms = 1;
    }
    {
        const cudaError_t e = launch_scan_tc(a, g_num_sms, s);
        if (e != cudaErrorNotSupported) return e;               // launched (or a real error)
    }
    for (int ncl = pick_cluster(a.dm, g_num_sms); ncl >= 2; ncl >>= 1) {
        const int cw = a.dm.d / ncl;
        if (cw > 64 || scan_cl_smem_bytes(a.dm, cw) > 227 * 1024) break;
        cudaError_t e;
        if (a.dm.D == 128)
            e = a.dm.dtype == 1 ? launch_scan_cl_d<128, __nv_bfloat16>(a, ncl, s) : launch_scan_cl_d<128, float>(a, ncl, s);
        else
            e = a.dm.dtype == 1 ? launch_scan_cl_d<64, __nv_bfloat16>(a, ncl, s) : launch_scan_cl_d<64, float>(a, ncl, s);
        if (e != cudaErrorNotSupported) return e;                // launched (or a real error)
    }
    // rows left in global memory: the largest cluster with whole 16-column slices
    // (SRE only; alternative rules take the one-CTA chain when no row pool fits)
    if (a.scorer == 0 && a.dm.lam + a.dm.C <= 32 * kCgKmax) {
        for (int ncl = 8; ncl >= 2; ncl >>= 1) {
            const int cw = a.dm.d / ncl;
            if (cw < 16 || cw > 64 || a.dm.S * ncl > g_num_sms) continue;
            if (scan_cg_smem_bytes(a.dm, cw) > 227 * 1024) continue;
            cudaError_t e;
            if (a.dm.D == 128)
                e = a.dm.dtype == 1 ? launch_scan_cg_d<128, __nv_bfloat16>(a, ncl, s) : launch_scan_cg_d<128, float>(a, ncl, s);
            else
                e = a.dm.dtype == 1 ? launch_scan_cg_d<64, __nv_bfloat16>(a, ncl, s) : launch_scan_cg_d<64, float>(a, ncl, s);
            if (e != cudaErrorNotSupported) return e;
        }
    }
    return a.dm.dtype == 1 ? launch_scan_d<__nv_bfloat16>(a, s) : launch_scan_d<float>(a, s);
}

}  // namespace lola

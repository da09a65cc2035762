// Device pieces shared by the memory-update chain kernels (scan.cu, scan_tc.cu):
// where the slot positions entering a launch come from, the static score of a
// candidate under an alternative scoring rule, and the one-warp top-lambda
// selection with its slot bookkeeping (LoLA notes §2.4, Eqs. 11-13).
#pragma once
#include <type_traits>

#include "device_common.cuh"

namespace lola {

// Slot positions entering chunk a.c_begin: the cache at the start of the call, or
// the snapshot a previous launch of the same call published for that chunk.
__device__ __forceinline__ const int* entering_slots(const PrefillArgs& a, int st) {
    const Dims& dm = a.dm;
    return a.c_begin == 0 ? a.sp.cache_pos + (size_t)st * dm.lam
                          : a.snap_pos + ((size_t)st * (dm.nc_max + 1) + a.c_begin) * dm.lam;
}

// Score of candidate position p (held in cache slot `slot` if it was cached before
// the call) under an alternative rule: its window score, computed for this call's
// positions and the window entering it, else the frozen score kept with its slot.
__device__ __forceinline__ float static_score(const PrefillArgs& a, int st, int p, int slot) {
    const Dims& dm = a.dm;
    if (p >= a.t_start - dm.eta)
        return a.key_sc[(size_t)st * (dm.eta + dm.max_tokens) + (size_t)(p - a.t_start + dm.eta)];
    return a.sp.cache_sc[(size_t)st * dm.lam + slot];
}

// Selection and slot bookkeeping of one scored block, by one full warp (the same
// in every CTA of a cluster).  Candidate e (members e < n_g in slot order, then
// the n_l newcomers in position order) is held by lane e % 32 as bit e / 32 of
// its registers.  Top-lambda by (score, -position): MSB radix passes of 8 bits
// over the fp32 score bits (scores are >= 0, so the bit pattern orders like the
// value) narrow the threshold to a bucket of candidates sharing a bit prefix;
// once the bucket is small (or the bits are exhausted) its members are ranked
// exactly by (bits descending, position ascending).  Then: kept newcomers take,
// in position order, the freed slots (evicted members and never-used slots) in
// slot order; the folded set is listed by pool row and its rows return to the
// free stack (ROWS), or listed by candidate index (no pool).  Returns the number
// of folded pairs.
template <int KMAX, bool ROWS>
__device__ int select_and_place(const float* score, const int* cand_pos, const int* cand_row, int n, int n_g,
                                int n_l, int lam, int l_lo, const int* new_row, int* slot_row, int* slot_pos,
                                int* fold_row, int* free_rows, int nfree, int P, int* free_slots, unsigned* hist,
                                int* eq_list, int* eq_keep) {
    using Mask = std::conditional_t<(KMAX > 32), unsigned long long, unsigned>;
    static_assert(KMAX <= 64, "one mask bit per register row");
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    unsigned u[KMAX];
    int crow[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        const int e = 32 * k + lane;
        u[k] = e < n ? __float_as_uint(score[e]) : 0u;
        crow[k] = ROWS ? (e < n ? cand_row[e] : 0) : e;
    }
    Mask keepm = 0u;
    if (lam > 0) {
        // digits: exponent (bits 30..23), then mantissa bytes; bit 31 is 0 for scores >= 0
        unsigned prefix = 0u, mask = 0x80000000u;
        int kk = lam, cnt = n;             // still to keep from the bucket; bucket size
#pragma unroll 1
        for (int pass = 0; pass < 4 && cnt > 32 && cnt > kk; ++pass) {
            const int shift = pass == 3 ? 0 : 23 - 8 * pass;
            const unsigned dmask = pass == 3 ? 127u : 255u;
            for (int i = lane; i < 256; i += 32) hist[i] = 0u;
            __syncwarp();
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (32 * k >= n) break;
                if (32 * k + lane < n && (u[k] & mask) == prefix) atomicAdd(&hist[(u[k] >> shift) & dmask], 1u);
            }
            __syncwarp();
            unsigned c[8], lsum = 0u;
#pragma unroll
            for (int t = 0; t < 8; ++t) { c[t] = hist[lane * 8 + t]; lsum += c[t]; }
            unsigned suf = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            unsigned above = suf - lsum;   // candidates in higher digits (higher lanes)
            int hit = -1;
            unsigned h_above = 0u, h_cnt = 0u;
#pragma unroll
            for (int t = 7; t >= 0; --t) {
                if (above < (unsigned)kk && (unsigned)kk <= above + c[t]) { hit = t; h_above = above; h_cnt = c[t]; }
                above += c[t];
            }
            const int src = __ffs(__ballot_sync(0xffffffffu, hit >= 0)) - 1;
            const int digit = __shfl_sync(0xffffffffu, lane * 8 + hit, src);
            kk -= (int)__shfl_sync(0xffffffffu, h_above, src);
            cnt = (int)__shfl_sync(0xffffffffu, h_cnt, src);
            prefix |= (unsigned)digit << shift;
            mask |= dmask << shift;
            __syncwarp();
        }
        // above the bucket: kept; the bucket is listed in candidate order
        Mask inbm = 0u;
        unsigned qbase[KMAX];
        int base = 0;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            const bool valid = 32 * k + lane < n;
            const unsigned m = u[k] & mask;
            if (valid && m > prefix) keepm |= Mask(1) << k;
            const bool inb = valid && m == prefix;
            if (inb) inbm |= Mask(1) << k;
            const unsigned b = __ballot_sync(0xffffffffu, inb);
            qbase[k] = (unsigned)base + __popc(b & lt);          // bucket index of this lane's member k
            if (inb) eq_list[base + __popc(b & lt)] = 32 * k + lane;
            base += __popc(b);
        }
        if (cnt == kk) {
            keepm |= inbm;
        } else if (cnt <= 32) {            // one member per lane; rank through shuffles
            __syncwarp();
            const int i = lane < cnt ? eq_list[lane] : 0;
            const unsigned ui = __float_as_uint(score[i]);
            const int pi = cand_pos[i];
            int r = 0;
#pragma unroll
            for (int z = 0; z < 32; ++z) {
                const unsigned w = __shfl_sync(0xffffffffu, ui, z);
                const int pz = __shfl_sync(0xffffffffu, pi, z);
                r += (z < cnt && (w > ui || (w == ui && pz < pi))) ? 1 : 0;
            }
            const unsigned kb = __ballot_sync(0xffffffffu, lane < cnt && r < kk);   // bit q: member q kept
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (((inbm >> k) & 1u) && ((kb >> qbase[k]) & 1u)) keepm |= Mask(1) << k;
        } else {                           // exact ties over many candidates
            __syncwarp();
            for (int q = lane; q < cnt; q += 32) {
                const int i = eq_list[q];
                const unsigned ui = __float_as_uint(score[i]);
                const int pi = cand_pos[i];
                int r = 0;
                for (int z = 0; z < cnt; ++z) {
                    const int j = eq_list[z];
                    const unsigned w = __float_as_uint(score[j]);
                    r += (w > ui || (w == ui && cand_pos[j] < pi)) ? 1 : 0;
                }
                eq_keep[q] = r < kk ? 1 : 0;
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (((inbm >> k) & 1u) && eq_keep[qbase[k]]) keepm |= Mask(1) << k;
        }
    }
    // freed slots, in slot order (member e sits in slot e)
    int base = 0;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        if (32 * k >= lam) break;
        const int j = 32 * k + lane;
        const bool f = j < lam && (j >= n_g || ((keepm >> k) & 1u) == 0u);
        const unsigned b = __ballot_sync(0xffffffffu, f);
        if (f) free_slots[base + __popc(b & lt)] = j;
        base += __popc(b);
    }
    const int n_free_slots = base;
    __syncwarp();
    // kept newcomers, in position order, take them in order
    base = 0;
    for (int i0 = 0; i0 < n_l; i0 += 32) {
        const int i = i0 + lane;
        const int e = min(n_g + i, n - 1);
        const Mask km = __shfl_sync(0xffffffffu, keepm, e & 31);
        const bool kept = i < n_l && ((km >> (e >> 5)) & 1u);
        const unsigned b = __ballot_sync(0xffffffffu, kept);
        const int fs = base + __popc(b & lt);
        if (kept && fs < n_free_slots) {             // always true when exactly lam are kept
            const int sl = free_slots[fs];
            if (ROWS) slot_row[sl] = new_row[i];
            slot_pos[sl] = l_lo + i;
        }
        base += __popc(b);
    }
    // the folded set S = E \ G_new, by pool row; the rows return to the free stack
    base = 0;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        if (32 * k >= n) break;
        const bool f = 32 * k + lane < n && ((keepm >> k) & 1u) == 0u;
        const unsigned b = __ballot_sync(0xffffffffu, f);
        const int q = base + __popc(b & lt);
        if (f && nfree + q < P) {                    // always true when exactly lam are kept
            fold_row[q] = crow[k];
            if (ROWS) free_rows[nfree + q] = crow[k];
        }
        base += __popc(b);
    }
    return min(base, P - nfree);
}

// The same selection and slot bookkeeping as select_and_place (ROWS = false), by
// the whole thread block: keep the lam candidates with the largest (score,
// -position), MSB radix passes over the fp32 score bits narrowing the threshold
// to a bucket, the bucket ranked exactly; freed slots (evicted members and
// never-used slots) in slot order go to the kept newcomers in position order;
// the folded candidates are listed in candidate order in fold_e.  Returns the
// number of folded candidates.  Scratch: keep [n], free_slots [lam + 1], hist
// [256], tmp [>= 32], eq_list [n], flags and ranks [max(n, lam)] each.
__device__ inline int select_place_cta(const float* score, const int* cand_pos, int n, int n_g, int n_l, int lam,
                                       int l_lo, int* slot_pos, int* fold_e, int* keep, int* free_slots,
                                       unsigned* hist, int* tmp, int* eq_list, int* flags, int* ranks) {
    const int tid = threadIdx.x, NT = blockDim.x, lane = tid & 31;
    if (lam > 0) {
        unsigned prefix = 0u, mask = 0x80000000u;            // bit 31 is 0 for scores >= 0
        int kk = lam, cnt = n;
#pragma unroll 1
        for (int pass = 0; pass < 4 && cnt > 32 && cnt > kk; ++pass) {
            const int shift = pass == 3 ? 0 : 23 - 8 * pass;
            const unsigned dmask = pass == 3 ? 127u : 255u;
            for (int i = tid; i < 256; i += NT) hist[i] = 0u;
            __syncthreads();
            for (int e = tid; e < n; e += NT) {
                const unsigned u = __float_as_uint(score[e]);
                if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
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
                unsigned above = suf - lsum;                 // candidates in higher digits (higher lanes)
#pragma unroll
                for (int t = 7; t >= 0; --t) {
                    if (above < (unsigned)kk && (unsigned)kk <= above + c[t]) {
                        tmp[0] = lane * 8 + t;
                        tmp[1] = kk - (int)above;
                        tmp[2] = (int)c[t];
                    }
                    above += c[t];
                }
            }
            __syncthreads();
            prefix |= (unsigned)tmp[0] << shift;
            mask |= dmask << shift;
            kk = tmp[1];
            cnt = tmp[2];
        }
        // above the bucket: kept; the bucket's members are ranked by (bits desc, position asc)
        if (tid == 0) tmp[3] = 0;
        __syncthreads();
        for (int e = tid; e < n; e += NT) {
            const unsigned m = __float_as_uint(score[e]) & mask;
            keep[e] = m > prefix ? 1 : 0;
            if (m == prefix) {
                if (cnt == kk) keep[e] = 1;
                else eq_list[atomicAdd(&tmp[3], 1)] = e;
            }
        }
        __syncthreads();
        if (cnt != kk) {
            const int neq = tmp[3];
            for (int q = tid; q < neq; q += NT) {
                const int i = eq_list[q];
                const unsigned ui = __float_as_uint(score[i]);
                const int pi = cand_pos[i];
                int r = 0;
                for (int z = 0; z < neq; ++z) {
                    const int j = eq_list[z];
                    const unsigned w = __float_as_uint(score[j]);
                    r += (w > ui || (w == ui && cand_pos[j] < pi)) ? 1 : 0;
                }
                keep[i] = r < kk ? 1 : 0;
            }
            __syncthreads();
        }
    } else {
        for (int e = tid; e < n; e += NT) keep[e] = 0;
        __syncthreads();
    }
    int nf = 0;
    // One block-wide exclusive scan of three packed counts (21 bits each) over x in
    // [0, max(lam, n)): freed slots in slot order (member e sits in slot e), kept newcomers
    // in position order, folded candidates in candidate order.  hist (free after the radix
    // passes) holds the per-warp sums.
    {
        auto fa = [&](int x) -> unsigned long long { return (x < lam && (x >= n_g || keep[x] == 0)) ? 1ull : 0ull; };
        auto fb = [&](int x) -> unsigned long long { return (x < n_l && keep[n_g + x]) ? 1ull : 0ull; };
        auto fc = [&](int x) -> unsigned long long { return (x < n && keep[x] == 0) ? 1ull : 0ull; };
        auto fl = [&](int x) { return fa(x) | (fb(x) << 21) | (fc(x) << 42); };
        constexpr unsigned long long F = (1ull << 21) - 1;
        unsigned long long* wsum = reinterpret_cast<unsigned long long*>(hist);
        const int X = max(lam, n), per = (X + NT - 1) / NT;
        const int lo = min(X, tid * per), hi = min(X, lo + per);
        const int warp = tid >> 5, NW = NT / 32;
        unsigned long long sum = 0ull;
        for (int x = lo; x < hi; ++x) sum += fl(x);
        unsigned long long incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            unsigned long long w = lane < NW ? wsum[lane] : 0ull;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            if (lane < NW) wsum[lane] = w;
        }
        __syncthreads();
        unsigned long long base = (warp ? wsum[warp - 1] : 0ull) + incl - sum;
        for (int x = lo; x < hi; ++x) {
            const unsigned long long f = fl(x);
            if (f & F) free_slots[(int)(base & F)] = x;
            if ((f >> 21) & F) ranks[x] = (int)((base >> 21) & F);
            if (f >> 42) fold_e[(int)(base >> 42)] = x;
            base += f;
        }
        nf = (int)(wsum[NW - 1] >> 42);
        __syncthreads();
        // kept newcomers take the freed slots in order
        for (int i = tid; i < n_l; i += NT) if (keep[n_g + i]) slot_pos[free_slots[ranks[i]]] = l_lo + i;
        __syncthreads();
    }
    return nf;
}

}  // namespace lola

// Per-token LoLA decode step (notes §2.4, Fig. 1; the one-token block of §2.6).
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
//
// SRE without recomputing H^T phi for every candidate: each cache slot keeps
// its residual R_e = H^T phi_e - den_e v_e and den_e = phi_e . s, so that
// SRE_e = ||R_e||^2 / den_e^2 (and ||v_e||^2 while den_e = 0, the empty
// memory recalling zero).  A decode step folds exactly one pair f, a rank-1
// change of (H, s), after which R_e += k_e (v_f - v_e), den_e += k_e with
// k_e = phi_e . phi_f: O(lambda (D + d)) work per step instead of
// O(lambda D d), and no cancellation (the residual itself is stored).
// residual_init_kernel computes them exactly from (H, s) after a prefill.  The
// pass that updates R_e also stores each member's SRE against the new state,
// so the next step's scoring reads one float per member instead of R.
//
// Layout: one CTA of 256 threads per stream, 64 registers and about 44 KB of
// shared memory, so that four CTAs share an SM and every stream of a decode
// batch of 512 streams is resident at once.  H stays in global memory: one
// streaming pass reads it for phi(q)^T H and H^T phi_l, and the fold updates it
// in place while it is still in L2.  Under the SRE rule with the read first the
// step runs: the products over the entering (H, s), the selection and fold, the
// read, the residual update right after P V (the members' value rows still in
// L2), and last the writes of l's slot and of the ring slot.
#include "device_common.cuh"
#include "umma.cuh"

namespace lola {

constexpr int kDecThreads = 256;
constexpr int kDecSlotBatch = 8;  // value rows per warp in flight in P V

struct DecOffsets {
    int ss, L, hp, Ws, qs, phq, kn, vn, phk, phl, Pl, vf, phf, red, kp, sc, R, part, total;
};

__host__ __device__ inline DecOffsets dec_offsets(int DIM, int DH, int Gq, int lam, int eta, int esize) {
    const int D = 2 * DH, NK = lam + eta + 1, NW = kDecThreads / 32;
    DecOffsets o;
    int p = 0;
    auto take = [&](int n) { int r = p; p += (n + 3) & ~3; return r; };
    o.ss = take(D);
    o.L = take(Gq * DIM);                  // phi(q)^T H per head
    o.hp = take(kDecThreads / DIM * (Gq + 1) * DIM);   // the H pass's partial sums
    o.Ws = 0;                             // set below: W (raw, <= 4 B per element) aliases R/part
    o.qs = take(Gq * DIM);
    o.phq = take(Gq * D);
    o.kn = take(DIM);
    o.vn = take(DIM);
    o.phk = take(D);
    o.phl = take(D);
    o.Pl = take(DIM);
    o.vf = take(DIM);
    o.phf = take(D);
    o.red = take(128);
    o.kp = take(4 * NK);                   // key and value row pointers (64-bit each)
    o.sc = take(max(Gq * NK, lam + 1));    // slot scores (update phase)
    // the read-phase partial sums [NW][Gq][DIM] alias the z scratch and the staged W
    o.R = take(max(NW * Gq * DIM, (DIM * DH * esize + 3) / 4 + (Gq + 1) * DH));
    o.part = o.R;
    o.Ws = o.R + (Gq + 1) * DH;           // after the z scratch rows
    o.total = p;
    return o;
}

// A quad of 4 lanes handles one row.  The row is cut into 4-element chunks and
// lane q of the quad takes chunks q, q + 4, q + 8, ...: element u of lane q is
// row[qidx(q, u)].  Lanes of a quad then read shared-memory operands in
// different banks, and each chunk is one 16-byte (f32) or 8-byte (bf16) load.
__device__ __forceinline__ int qidx(int q, int u) { return ((u >> 2) * 4 + q) * 4 + (u & 3); }
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}
// Rows kept as raw 32-bit words until their values are used (a bf16 word holds
// two elements, the lower address in the low half).
template <int NWD>
__device__ __forceinline__ void load_words(const void* p, unsigned* w) {
    if constexpr (NWD == 4) { const uint4 v = *reinterpret_cast<const uint4*>(p); w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w; }
    else if constexpr (NWD == 2) { const uint2 v = *reinterpret_cast<const uint2*>(p); w[0] = v.x; w[1] = v.y; }
    else { static_assert(NWD == 1, "1, 2 or 4 words"); w[0] = *reinterpret_cast<const unsigned*>(p); }
}
template <typename T> __device__ __forceinline__ float word_elem(unsigned w, int h);
template <> __device__ __forceinline__ float word_elem<float>(unsigned w, int) { return __uint_as_float(w); }
template <> __device__ __forceinline__ float word_elem<__nv_bfloat16>(unsigned w, int h) {
    return __uint_as_float(h ? (w & 0xffff0000u) : (w << 16));
}

// An octet of 8 lanes handles one row in the residual update: lane o takes the
// 4-element chunks o, o + 8, o + 16, ..., so element u of lane o is row[oidx(o, u)].
__device__ __forceinline__ int oidx(int o, int u) { return ((u >> 2) * 8 + o) * 4 + (u & 3); }
__device__ __forceinline__ float oct_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    return x;
}
template <int N, typename T>
__device__ __forceinline__ void load_oct(const T* row, int o, float (&out)[N / 8]) {
#pragma unroll
    for (int i = 0; i < N / 32; ++i) {
        const float4 f = load4(row + (8 * i + o) * 4);
        out[4 * i] = f.x; out[4 * i + 1] = f.y; out[4 * i + 2] = f.z; out[4 * i + 3] = f.w;
    }
}
template <int N>
__device__ __forceinline__ void load_quarter(const float* row, int q, float (&out)[N / 4]) {
#pragma unroll
    for (int i = 0; i < N / 16; ++i) {
        const float4 f = *reinterpret_cast<const float4*>(row + (4 * i + q) * 4);
        out[4 * i] = f.x; out[4 * i + 1] = f.y; out[4 * i + 2] = f.z; out[4 * i + 3] = f.w;
    }
}
template <int N>
__device__ __forceinline__ void load_quarter(const __nv_bfloat16* row, int q, float (&out)[N / 4]) {
#pragma unroll
    for (int i = 0; i < N / 16; ++i) {
        const float4 f = load4(row + (4 * i + q) * 4);
        out[4 * i] = f.x; out[4 * i + 1] = f.y; out[4 * i + 2] = f.z; out[4 * i + 3] = f.w;
    }
}

// GQM bounds the query heads per kv head (Gq <= GQM): per-head registers are sized by it.
template <int DIM, int DH, int GQM, typename TIn>
__global__ void __launch_bounds__(kDecThreads, 4) decode_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int D = 2 * DH, NT = kDecThreads, NW = NT / 32, CPL = DIM / 32;
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int Gq = dm.Gq, lam = dm.lam, eta = dm.eta, t = a.t;
    const int st = blockIdx.x, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const DecOffsets o = dec_offsets(DIM, DH, Gq, lam, eta, (int)sizeof(TIn));
    float* ss = smem + o.ss;
    float* Lq = smem + o.L;
    float* qs = smem + o.qs;
    float* phq = smem + o.phq;
    float* kn = smem + o.kn;
    float* vn = smem + o.vn;
    float* phk = smem + o.phk;
    float* phl = smem + o.phl;
    float* Pl = smem + o.Pl;
    float* vf = smem + o.vf;
    float* phf = smem + o.phf;
    float* red = smem + o.red;
    const TIn** kp = reinterpret_cast<const TIn**>(smem + o.kp);
    float* sc = smem + o.sc;
    float* Ws = smem + o.Ws;
    float* part = smem + o.part;

    float* Hg = a.sp.H + (size_t)st * D * DIM;
    float* sg = a.sp.s + (size_t)st * D;
    const TIn* Wg = (const TIn*)a.sp.W + (size_t)g * DIM * DH;
    // s and W with asynchronous copies (H stays in global memory: one pass reads
    // it for the products below, the fold updates it in place)
    TIn* Wsm = reinterpret_cast<TIn*>(Ws);
    for (int i = tid; i < D / 4; i += NT) umma::cp_async16(ss + 4 * i, sg + 4 * i);
    constexpr int WCH = DIM * DH * (int)sizeof(TIn) / 16;
    for (int i = tid; i < WCH; i += NT)
        umma::cp_async16(reinterpret_cast<char*>(Wsm) + 16 * i, reinterpret_cast<const char*>(Wg) + 16 * i);
    umma::cp_async_commit();
    const TIn* qg = (const TIn*)a.q + ((size_t)b * dm.Hq + (size_t)g * Gq) * DIM;
    for (int i = tid; i < Gq * DIM; i += NT) qs[i] = to_f32(qg[i]);
    const TIn* kg = (const TIn*)a.k + ((size_t)b * dm.Hkv + g) * DIM;
    const TIn* vg = (const TIn*)a.v + ((size_t)b * dm.Hkv + g) * DIM;
    for (int i = tid; i < DIM; i += NT) { kn[i] = to_f32(kg[i]); vn[i] = to_f32(vg[i]); }
    const int n_g = min(lam, max(0, t - eta));
    const size_t cbase = (size_t)st * lam, wbase = (size_t)st * eta;
    const bool hide_state = (a.read_mask & 1) != 0, hide_sparse = (a.read_mask & 2) != 0;
    // key row pointers of the read: cache slots [0, rg), window positions [rlo, t)
    // (ring slot p % eta), then the token itself; returns the key count
    auto fill_kp = [&](int rg, int rlo) -> int {
        const int rw = t - rlo, nk = rg + rw + 1;
        for (int i = tid; i < nk; i += NT) {
            const TIn* p;
            const TIn* pv;        // the value row sits at the same offset of the matching value array
            if (i < rg) {
                p = (const TIn*)a.sp.cache_k + (cbase + i) * DIM;
                pv = (const TIn*)a.sp.cache_v + (cbase + i) * DIM;
            } else if (i < rg + rw) {
                const size_t ws = wbase + (size_t)((rlo + i - rg) % eta);
                p = (const TIn*)a.sp.win_k + ws * DIM;
                pv = (const TIn*)a.sp.win_v + ws * DIM;
            } else {
                p = kg;
                pv = vg;
            }
            kp[2 * i] = p;
            kp[2 * i + 1] = pv;
        }
        return nk;
    };
    // read first: the memories entering the step (the window holds [t - eta, t));
    // update first reads after the update (see the end of the kernel)
    const int rg0 = hide_sparse ? 0 : n_g, rlo0 = max(0, t - eta);
    const int NK = a.update_first ? 0 : fill_kp(rg0, rlo0);
    umma::cp_async_wait<0>();
    __syncthreads();

    // feature map of the queries and the new key: z = x W (thread per (row, column)), then
    // softmax(z) and softmax(-z) per row (one warp per row)
    const int lpos = t - eta, rs = lpos >= 0 ? lpos % eta : 0;
    const bool leaving = t >= eta;
    if (leaving)
        for (int i = tid; i < D; i += NT) phl[i] = a.sp.win_phik[(wbase + rs) * D + i];
    __syncthreads();
    float* zs = smem + o.R;                                           // scratch [Gq + 1][DH]
    for (int idx = tid; idx < (Gq + 1) * DH; idx += NT) {
        const int r = idx / DH, col = idx % DH;
        const float* x = r < Gq ? qs + r * DIM : kn;
        float z = 0.f;
#pragma unroll 8
        for (int j = 0; j < DIM; ++j) z = fmaf(x[j], to_f32(Wsm[j * DH + col]), z);
        zs[idx] = z;
    }
    __syncthreads();
    for (int r = warp; r <= Gq; r += NW) {
        float z[DH / 32];
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) z[u] = zs[r * DH + lane + 32 * u];
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

    // ---- one pass over H ([D][DIM] in global memory): Lq[hh][cc] = phi(q_hh)^T H[:, cc]
    // for the read and Pl[cc] = H[:, cc] . phi_l for the update; NT / DIM threads per
    // column, each over a contiguous share of the rows, then their sums in share order ----
    auto h_pass = [&](const bool wantL, const bool wantP) {
        constexpr int NSP = NT / DIM, RPS = D / NSP, HB = 8;
        const int cc = tid % DIM, sp = tid / DIM;
        float acc[GQM + 1];
#pragma unroll
        for (int k = 0; k <= GQM; ++k) acc[k] = 0.f;
        const float* hcol = Hg + (size_t)sp * RPS * DIM + cc;
        for (int j0 = 0; j0 < RPS; j0 += HB) {
            float h[HB];
#pragma unroll
            for (int u = 0; u < HB; ++u) h[u] = hcol[(size_t)(j0 + u) * DIM];   // the batch's loads first
#pragma unroll
            for (int u = 0; u < HB; ++u) {
                const int j = sp * RPS + j0 + u;
                if (wantL) {
#pragma unroll
                    for (int hh = 0; hh < GQM; ++hh)
                        if (hh < Gq) acc[hh] = fmaf(phq[hh * D + j], h[u], acc[hh]);
                }
                if (wantP) acc[GQM] = fmaf(phl[j], h[u], acc[GQM]);
            }
        }
        float* hp = smem + o.hp;                                    // [NSP][Gq + 1][DIM]
#pragma unroll
        for (int hh = 0; hh < GQM; ++hh)
            if (hh < Gq) hp[(sp * (Gq + 1) + hh) * DIM + cc] = acc[hh];
        hp[(sp * (Gq + 1) + Gq) * DIM + cc] = acc[GQM];
        __syncthreads();
        for (int idx = tid; idx < (Gq + 1) * DIM; idx += NT) {
            float x = 0.f;
            for (int k = 0; k < NSP; ++k) x += hp[k * (Gq + 1) * DIM + idx];
            const int hh = idx / DIM;
            if (hh < Gq) { if (wantL) Lq[idx] = x; }
            else if (wantP) Pl[idx - Gq * DIM] = x;
        }
        __syncthreads();
    };

    // ---- read: scores (a quad per key), softmax per head, P V (lane owns columns) ----
    // Eq. 14 over the NK keys of kp and, unless hidden, the state (H, s): phi(q)^T H from
    // the H pass (Lq), phi(q) . s from s in shared memory
    // hL / hP: run the H pass after P V for phi(q)^T H / H^T phi_l; dlReady: phi(q) . s
    // is already in red[16 + hh] (taken before a fold that precedes the read)
    auto read_phase = [&](const int NK, const int rg, const int rlo, const bool hL, const bool hP, const bool dlReady) {
        // a quad of lanes per key, KPQ keys per quad; lane q4 takes the 16-byte chunks
        // q4, q4 + 4, ... of the row, kept as raw words
        constexpr int CH = 16 / (int)sizeof(TIn), NCH = DIM / CH / 4, KW = NCH * 4, EPW = 4 / (int)sizeof(TIn);
        constexpr int KPQ = sizeof(TIn) == 2 ? 2 : 1;
        const int q4 = lane & 3, rq = lane >> 2;                     // lane in quad, quad in warp
        const float scale = 1.0f / sqrtf((float)DIM);
        for (int i0 = warp * 8 * KPQ; i0 < NK; i0 += NW * 8 * KPQ) {
            unsigned kw[KPQ][KW];
#pragma unroll
            for (int kq = 0; kq < KPQ; ++kq) {
                const int i = i0 + kq * 8 + rq;
                if (i < NK)
#pragma unroll
                    for (int c = 0; c < NCH; ++c) load_words<4>(kp[2 * i] + (c * 4 + q4) * CH, &kw[kq][4 * c]);
            }
#pragma unroll
            for (int hh = 0; hh < GQM; ++hh) {
                if (hh < Gq) {
                    float sd[KPQ];
#pragma unroll
                    for (int kq = 0; kq < KPQ; ++kq) sd[kq] = 0.f;
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
#pragma unroll
                        for (int w = 0; w < 4; ++w)
#pragma unroll
                            for (int h = 0; h < EPW; ++h) {
                                const float qv = qs[hh * DIM + (c * 4 + q4) * CH + w * EPW + h];
#pragma unroll
                                for (int kq = 0; kq < KPQ; ++kq) sd[kq] = fmaf(qv, word_elem<TIn>(kw[kq][4 * c + w], h), sd[kq]);
                            }
#pragma unroll
                    for (int kq = 0; kq < KPQ; ++kq) {
                        const float x = quad_sum(sd[kq]);
                        const int i = i0 + kq * 8 + rq;
                        if (i < NK && q4 == 0) sc[hh * NK + i] = x * scale;
                    }
                }
            }
        }
        __syncthreads();
        if (a.scorer) {
            // alternative rules: the query credits every window key it reads, and itself
            for (int i = rg + warp; i < NK; i += NW) {
                const bool self = i == NK - 1;
                const size_t ws = wbase + (size_t)((self ? t : rlo + i - rg) % eta);
                const float* pk = self ? phk : a.sp.win_phik + ws * D;
                float term = 0.f;
                for (int hh = 0; hh < Gq; ++hh) {
                    float f = 0.f;
                    for (int j = lane; j < D; j += 32) f = fmaf(phq[hh * D + j], pk[j], f);
                    f = warp_sum(f);
                    term += window_term(a.scorer, expf(sc[hh * NK + i]), f);
                }
                if (lane == 0) {
                    if (!self) a.sp.win_sc[ws] += term;
                    else if (a.update_first) a.sp.win_sc[ws] = term;   // the ring slot is already the token's
                    else red[48] = term;                                 // stored with the token after the update
                }
            }
            __syncthreads();
        }
        for (int hh = warp; hh < Gq; hh += NW) {
            float mx = -INFINITY;
            for (int i = lane; i < NK; i += 32) mx = fmaxf(mx, sc[hh * NK + i]);
            mx = warp_max(mx);
            float sum = 0.f;
            for (int i = lane; i < NK; i += 32) { const float e = expf(sc[hh * NK + i] - mx); sc[hh * NK + i] = e; sum += e; }
            sum = warp_sum(sum);
            if (!dlReady) {
                float dl = 0.f;
                if (!hide_state)
                    for (int j = lane; j < D; j += 32) dl = fmaf(phq[hh * D + j], ss[j], dl);
                dl = warp_sum(dl);
                if (lane == 0) red[16 + hh] = dl;
            }
            if (lane == 0) { red[hh] = mx; red[8 + hh] = sum; }
        }
        __syncthreads();
        float accp[GQM][CPL];
#pragma unroll
        for (int hh = 0; hh < GQM; ++hh)
#pragma unroll
            for (int u = 0; u < CPL; ++u) accp[hh][u] = 0.f;
        constexpr int PVW = CPL * (int)sizeof(TIn) / 4;              // words of a lane's columns
        for (int i0 = warp; i0 < NK; i0 += NW * kDecSlotBatch) {
            unsigned vw[kDecSlotBatch][PVW];
#pragma unroll
            for (int bb = 0; bb < kDecSlotBatch; ++bb) {             // issue the batch's loads first
                const int i = i0 + bb * NW;
                if (i < NK) load_words<PVW>(kp[2 * i + 1] + lane * CPL, vw[bb]);
            }
#pragma unroll
            for (int bb = 0; bb < kDecSlotBatch; ++bb) {
                const int i = i0 + bb * NW;
                if (i >= NK) break;
#pragma unroll
                for (int hh = 0; hh < GQM; ++hh) {
                    if (hh < Gq) {
                        const float p = sc[hh * NK + i];
#pragma unroll
                        for (int u = 0; u < CPL; ++u)
                            accp[hh][u] = fmaf(p, word_elem<TIn>(vw[bb][u / EPW], u % EPW), accp[hh][u]);
                    }
                }
            }
        }
#pragma unroll
        for (int hh = 0; hh < GQM; ++hh)
            if (hh < Gq)
#pragma unroll
                for (int u = 0; u < CPL; ++u) part[(warp * Gq + hh) * DIM + lane * CPL + u] = accp[hh][u];
        __syncthreads();
        // phi(q)^T H for the output and, read first, H^T phi_l for the update: H is read
        // here, close to the fold, so that the fold finds it in L2
        if (hL || hP) h_pass(hL, hP);
        for (int idx = tid; idx < Gq * DIM; idx += NT) {
            const int hh = idx / DIM, cc = idx % DIM;
            float A = 0.f;
            for (int w = 0; w < NW; ++w) A += part[(w * Gq + hh) * DIM + cc];
            const float L = hide_state ? 0.f : Lq[idx];
            const float em = expf(-red[hh]);
            a.y[((size_t)b * dm.Hq + (size_t)g * Gq + hh) * DIM + cc] = (A + em * L) / (red[8 + hh] + em * red[16 + hh]);
        }
        __syncthreads();
    };

    int f_fold = lam;                                             // the folded candidate
    float den_fold = 0.f;                                         // phi_l . s before the fold
    // the remaining members' residuals follow the rank-1 fold of f (SRE only), then l
    // takes the folded member's slot
    auto members_and_slot = [&](const int f, const float den_l) {
        const size_t wsl = wbase + rs;
        const TIn* vl = (const TIn*)a.sp.win_v + wsl * DIM;
        float* Rg = a.sp.cache_R + cbase * DIM;
        float* deng = a.sp.cache_den + cbase;
        // an octet per member: k_e = phi_e . phi_f, R_e += k_e (v_f - v_e), den_e += k_e
        if (!a.scorer) {
            constexpr int PO = D / 8, RO = DIM / 8;
            const int o8 = lane & 7, ro = lane >> 3;
            for (int e0 = warp * 4; e0 <= lam; e0 += NW * 4) {
                const int e = e0 + ro;
                const bool act = e <= lam && e != f;
                float pv[PO], vv[RO], r0[RO];
                float d0 = 0.f;
                if (act) {
                    load_oct<D>(e < lam ? a.sp.cache_phik + (cbase + e) * D : phl, o8, pv);
                    load_oct<DIM>(e < lam ? (const TIn*)a.sp.cache_v + (cbase + e) * DIM : vl, o8, vv);
                    if (e < lam) {
                        load_oct<DIM>(Rg + (size_t)e * DIM, o8, r0);
                        d0 = deng[e];
                    } else {
#pragma unroll
                        for (int u = 0; u < RO; ++u) r0[u] = Pl[oidx(o8, u)] - den_l * vv[u];
                        d0 = den_l;
                    }
                }
                float kap = 0.f;
                if (act) {
#pragma unroll
                    for (int u = 0; u < PO; ++u) kap = fmaf(pv[u], phf[oidx(o8, u)], kap);
                }
                kap = oct_sum(kap);
                float q = 0.f, vq = 0.f;
                const int dst = e < lam ? e : f;   // its own slot, or f's slot for the newcomer l
                if (act) {
                    float* rw = Rg + (size_t)dst * DIM;
#pragma unroll
                    for (int u = 0; u < RO; u += 4) {
                        const int c0 = oidx(o8, u);                       // 4 consecutive columns
                        const float4 r4 = make_float4(
                            fmaf(kap, vf[c0] - vv[u], r0[u]), fmaf(kap, vf[c0 + 1] - vv[u + 1], r0[u + 1]),
                            fmaf(kap, vf[c0 + 2] - vv[u + 2], r0[u + 2]), fmaf(kap, vf[c0 + 3] - vv[u + 3], r0[u + 3]));
                        *reinterpret_cast<float4*>(rw + c0) = r4;
                        q = fmaf(r4.x, r4.x, q); q = fmaf(r4.y, r4.y, q);
                        q = fmaf(r4.z, r4.z, q); q = fmaf(r4.w, r4.w, q);
                    }
#pragma unroll
                    for (int u = 0; u < RO; ++u) vq = fmaf(vv[u], vv[u], vq);
                }
                q = oct_sum(q);
                vq = oct_sum(vq);
                if (act && o8 == 0) {
                    const float dn = d0 + kap;
                    deng[dst] = dn;
                    a.sp.cache_sc[cbase + dst] = dn > 0.f ? q / (dn * dn) : vq;   // SRE against the new state
                }
            }
        }
        if (f < lam) {                                            // l takes the folded member's slot
            const size_t cs = cbase + f;
            for (int i = tid; i < DIM; i += NT) {
                ((TIn*)a.sp.cache_k)[cs * DIM + i] = ((const TIn*)a.sp.win_k)[wsl * DIM + i];
                ((TIn*)a.sp.cache_v)[cs * DIM + i] = vl[i];
            }
            for (int i = tid; i < D; i += NT) a.sp.cache_phik[cs * D + i] = phl[i];
            if (tid == 0) {
                a.sp.cache_pos[cs] = lpos;
                if (a.scorer) a.sp.cache_sc[cs] = sc[lam];
            }
        }
    };
    // the new token enters the window ring (after every read of the leaving slot)
    auto ring_write = [&]() {
        __syncthreads();
        const size_t ws = wbase + (size_t)(t % eta);
        for (int i = tid; i < DIM; i += NT) {
            ((TIn*)a.sp.win_k)[ws * DIM + i] = kg[i];
            ((TIn*)a.sp.win_v)[ws * DIM + i] = vg[i];
        }
        for (int i = tid; i < D; i += NT) a.sp.win_phik[ws * D + i] = phk[i];
        if (a.scorer && !a.update_first && tid == 0) a.sp.win_sc[ws] = red[48];
    };

    // ---- update (Eqs. 11-13 with one leaving pair l = t - eta) ----
    auto update_phase = [&](const bool tail) {
        if (leaving) {
            const size_t wsl = wbase + rs;
            const TIn* vl = (const TIn*)a.sp.win_v + wsl * DIM;
            // P_l = H^T phi_l (the H pass), den_l = phi_l . s, R_l = P_l - den_l v_l
            // (pre-fold state; SRE only)
            if (!a.scorer) {
                if (warp == 0) {
                    float x = 0.f;
                    for (int j = lane; j < D; j += 32) x = fmaf(phl[j], ss[j], x);
                    x = warp_sum(x);
                    if (lane == 0) red[32] = x;
                }
            }
            __syncthreads();
            const float den_l = a.scorer ? 0.f : red[32];
            float* Rg = a.sp.cache_R + cbase * DIM;
            float* deng = a.sp.cache_den + cbase;
            if (n_g < lam) {
                // l joins the next free slot (fewer than lambda candidates: keep all)
                const size_t cs = cbase + n_g;
                for (int i = tid; i < DIM; i += NT) {
                    ((TIn*)a.sp.cache_k)[cs * DIM + i] = ((const TIn*)a.sp.win_k)[wsl * DIM + i];
                    ((TIn*)a.sp.cache_v)[cs * DIM + i] = vl[i];
                    if (!a.scorer) Rg[(size_t)n_g * DIM + i] = Pl[i] - den_l * to_f32(vl[i]);
                }
                for (int i = tid; i < D; i += NT) a.sp.cache_phik[cs * D + i] = phl[i];
                if (tid == 0) {
                    a.sp.cache_pos[cs] = lpos;
                    if (a.scorer) a.sp.cache_sc[cs] = a.sp.win_sc[wsl];        // its frozen window score
                    else deng[n_g] = den_l;
                }
                if (!a.scorer && warp == 0) {                             // its SRE against the state
                    float q = 0.f, vq = 0.f;
                    for (int cc = lane; cc < DIM; cc += 32) {
                        const float v = to_f32(vl[cc]);
                        const float r = Pl[cc] - den_l * v;
                        q = fmaf(r, r, q);
                        vq = fmaf(v, v, vq);
                    }
                    q = warp_sum(q);
                    vq = warp_sum(vq);
                    if (lane == 0) a.sp.cache_sc[cs] = den_l > 0.f ? q / (den_l * den_l) : vq;
                }
            } else {
                // scores: members from the cache (stored when their residuals last changed), l from R_l
                float* scs = red + 64;                                    // reuse as scratch for the argmin
                for (int e = tid; e < lam; e += NT) sc[e] = a.sp.cache_sc[cbase + e];
                if (a.scorer) {
                    if (tid == 0) sc[lam] = a.sp.win_sc[wsl];             // l's window score is complete
                } else if (warp == 0) {
                    float q = 0.f, vq = 0.f;
                    for (int cc = lane; cc < DIM; cc += 32) {
                        const float v = to_f32(vl[cc]);
                        const float r = Pl[cc] - den_l * v;
                        q = fmaf(r, r, q);
                        vq = fmaf(v, v, vq);
                    }
                    q = warp_sum(q);
                    vq = warp_sum(vq);
                    if (lane == 0) sc[lam] = den_l > 0.f ? q / (den_l * den_l) : vq;
                }
                __syncthreads();
                // the folded pair: lowest SRE, the newer position on exact ties (keys are unique)
                auto cand_key = [&](int e) -> unsigned long long {
                    const int p = e < lam ? a.sp.cache_pos[cbase + e] : lpos;
                    return ((unsigned long long)__float_as_uint(sc[e]) << 32) | (unsigned long long)(~(unsigned)p);
                };
                unsigned long long best = ~0ull;
                for (int e = tid; e <= lam; e += NT) { const unsigned long long kk = cand_key(e); best = kk < best ? kk : best; }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const unsigned long long o2 = __shfl_xor_sync(0xffffffffu, best, off);
                    best = o2 < best ? o2 : best;
                }
                unsigned long long* keys = reinterpret_cast<unsigned long long*>(scs);
                if (lane == 0) keys[warp] = best;
                __syncthreads();
                unsigned long long bb = keys[0];
                for (int w = 1; w < NW; ++w) bb = keys[w] < bb ? keys[w] : bb;
                int* fsel = reinterpret_cast<int*>(red + 40);
                for (int e = tid; e <= lam; e += NT)
                    if (cand_key(e) == bb) *fsel = e;
                __syncthreads();
                const int f = *fsel;
                f_fold = f;
                den_fold = den_l;
                // stage the folded pair
                for (int i = tid; i < D; i += NT) phf[i] = f < lam ? a.sp.cache_phik[(cbase + f) * D + i] : phl[i];
                for (int i = tid; i < DIM; i += NT) vf[i] = to_f32(f < lam ? ((const TIn*)a.sp.cache_v)[(cbase + f) * DIM + i] : vl[i]);
                __syncthreads();
                // fold (Eqs. 12-13): H += phi_f v_f^T in place (8 float4 loads in flight
                // per thread), s += phi_f
                {
                    constexpr int NV = D * DIM / 4 / NT, FB = NV < 8 ? NV : 8;
                    static_assert(NV * NT * 4 == D * DIM, "whole float4 rounds");
                    float4* H4 = reinterpret_cast<float4*>(Hg);
#pragma unroll 1
                    for (int v0 = 0; v0 < NV; v0 += FB) {
                        float4 h[FB];
#pragma unroll
                        for (int u = 0; u < FB; ++u) h[u] = H4[(v0 + u) * NT + tid];
#pragma unroll
                        for (int u = 0; u < FB; ++u) {
                            const int i = 4 * ((v0 + u) * NT + tid), j = i / DIM, c = i % DIM;
                            const float p = phf[j];
                            h[u].x = fmaf(p, vf[c], h[u].x);
                            h[u].y = fmaf(p, vf[c + 1], h[u].y);
                            h[u].z = fmaf(p, vf[c + 2], h[u].z);
                            h[u].w = fmaf(p, vf[c + 3], h[u].w);
                            H4[(v0 + u) * NT + tid] = h[u];
                        }
                    }
                }
                for (int i = tid; i < D; i += NT) ss[i] += phf[i];
                // residuals of every remaining member follow the rank-1 change (SRE only)
                __syncthreads();
                for (int i = tid; i < D; i += NT) sg[i] = ss[i];
                if (tail) members_and_slot(f, den_l);
            }
        }
        if (tail) ring_write();
    };

    const bool needP = leaving && !a.scorer;                      // H^T phi_l for the update
    if (!a.update_first && !a.scorer) {
        // SRE rule, read first.  The read sees the memories entering the step, so its
        // products over (H, s) are taken first; then the fold, the read itself, and the
        // members' residuals right after P V, while their value rows are still in L2.
        // l's slot and the ring slot are written last, after every read of them.
        if (!hide_state || needP) h_pass(!hide_state, needP);
        for (int hh = warp; hh < Gq; hh += NW) {
            float dl = 0.f;
            if (!hide_state)
                for (int j = lane; j < D; j += 32) dl = fmaf(phq[hh * D + j], ss[j], dl);
            dl = warp_sum(dl);
            if (lane == 0) red[16 + hh] = dl;
        }
        __syncthreads();
        update_phase(false);
        read_phase(NK, rg0, rlo0, false, false, true);
        if (leaving && n_g == lam) members_and_slot(f_fold, den_fold);
        ring_write();
    } else if (!a.update_first) {
        read_phase(NK, rg0, rlo0, !hide_state, needP, false);
        update_phase(true);
    } else {
        if (needP) h_pass(false, true);
        // the token equations read literally: update, then read the new memories
        // (cache slots [0, min(lambda, t + 1 - eta)), window [t + 1 - eta, t), the token)
        update_phase(true);
        __syncthreads();
        const int rg1 = hide_sparse ? 0 : min(lam, max(0, t + 1 - eta)), rlo1 = max(0, t + 1 - eta);
        const int nk = fill_kp(rg1, rlo1);
        __syncthreads();
        read_phase(nk, rg1, rlo1, !hide_state, false, false);     // over the folded state
    }
}

// R_e = H^T phi_e - (phi_e . s) v_e and den_e = phi_e . s for every occupied
// cache slot, from the current state (run before the first decode step that
// follows a prefill).  Grid (streams, slot blocks of 32); H staged in smem.
template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(256) residual_init_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int D = 2 * DH, SB = 32;
    extern __shared__ __align__(16) float smem[];
    const Dims& dm = a.dm;
    const int st = blockIdx.x, lam = dm.lam;
    const int n_g = min(lam, max(0, a.t - dm.eta));
    const int e0 = blockIdx.y * SB;
    if (e0 >= n_g) return;
    const int ne = min(SB, n_g - e0);
    float* Hs = smem;                  // [D][DIM]
    float* ph = Hs + D * DIM;          // [SB][D]
    float* ss = ph + SB * D;           // [D]
    float* den = ss + D;               // [SB]
    const size_t cbase = (size_t)st * lam;
    for (int i = threadIdx.x; i < D * DIM / 4; i += 256)
        reinterpret_cast<float4*>(Hs)[i] = reinterpret_cast<const float4*>(a.sp.H + (size_t)st * D * DIM)[i];
    for (int i = threadIdx.x; i < D; i += 256) ss[i] = a.sp.s[(size_t)st * D + i];
    for (int i = threadIdx.x; i < ne * D; i += 256) ph[i] = a.sp.cache_phik[(cbase + e0) * D + i];
    __syncthreads();
    for (int e = threadIdx.x >> 5; e < ne; e += 8) {
        float x = 0.f;
        for (int j = threadIdx.x & 31; j < D; j += 32) x = fmaf(ph[e * D + j], ss[j], x);
        x = warp_sum(x);
        if ((threadIdx.x & 31) == 0) { den[e] = x; a.sp.cache_den[cbase + e0 + e] = x; }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < ne * DIM; idx += 256) {
        const int e = idx / DIM, cc = idx % DIM;
        float x = 0.f;
        for (int j = 0; j < D; ++j) x = fmaf(ph[e * D + j], Hs[j * DIM + cc], x);
        const float v = to_f32(((const TIn*)a.sp.cache_v)[(cbase + e0 + e) * DIM + cc]);
        a.sp.cache_R[(cbase + e0 + e) * DIM + cc] = x - den[e] * v;
    }
    __syncthreads();
    // each member's SRE against the state (warp per member), from the rows just written
    for (int e = threadIdx.x >> 5; e < ne; e += 8) {
        float q = 0.f, vq = 0.f;
        for (int cc = threadIdx.x & 31; cc < DIM; cc += 32) {
            const float r = a.sp.cache_R[(cbase + e0 + e) * DIM + cc];
            const float v = to_f32(((const TIn*)a.sp.cache_v)[(cbase + e0 + e) * DIM + cc]);
            q = fmaf(r, r, q);
            vq = fmaf(v, v, vq);
        }
        q = warp_sum(q);
        vq = warp_sum(vq);
        if ((threadIdx.x & 31) == 0) a.sp.cache_sc[cbase + e0 + e] = den[e] > 0.f ? q / (den[e] * den[e]) : vq;
    }
}

template <int DIM, int DH, int GQM, typename TIn>
static cudaError_t launch_dec_g(const DecodeArgs& a, cudaStream_t s) {
    const size_t bytes = (size_t)dec_offsets(DIM, DH, a.dm.Gq, a.dm.lam, a.dm.eta, (int)sizeof(TIn)).total * 4;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<DIM, DH, GQM, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    decode_kernel<DIM, DH, GQM, TIn><<<a.dm.S, kDecThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_dec_t(const DecodeArgs& a, cudaStream_t s) {
    if (a.dm.Gq < 1 || a.dm.Gq > 8) return cudaErrorInvalidValue;
    return a.dm.Gq <= 4 ? launch_dec_g<DIM, DH, 4, TIn>(a, s) : launch_dec_g<DIM, DH, 8, TIn>(a, s);
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_rinit_t(const DecodeArgs& a, cudaStream_t s) {
    constexpr int D = 2 * DH;
    const size_t bytes = (size_t)(D * DIM + 32 * D + D + 32) * 4;
    cudaError_t e = cudaFuncSetAttribute(residual_init_kernel<DIM, DH, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(a.dm.S, (a.dm.lam + 31) / 32);
    residual_init_kernel<DIM, DH, TIn><<<grid, 256, bytes, s>>>(a);
    return cudaGetLastError();
}

#define LOLA_DISPATCH_DIM(FN, a, s)                                              \
    do {                                                                         \
        const int d_ = (a).dm.d, Dh_ = (a).dm.Dh;                                \
        if (d_ == 64 && Dh_ == 32) return FN<64, 32, TIn>(a, s);                \
        if (d_ == 64 && Dh_ == 64) return FN<64, 64, TIn>(a, s);                \
        if (d_ == 128 && Dh_ == 32) return FN<128, 32, TIn>(a, s);              \
        if (d_ == 128 && Dh_ == 64) return FN<128, 64, TIn>(a, s);              \
        return cudaErrorInvalidValue;                                            \
    } while (0)

template <typename TIn>
static cudaError_t launch_dec_d(const DecodeArgs& a, cudaStream_t s) { LOLA_DISPATCH_DIM(launch_dec_t, a, s); }
template <typename TIn>
static cudaError_t launch_rinit_d(const DecodeArgs& a, cudaStream_t s) { LOLA_DISPATCH_DIM(launch_rinit_t, a, s); }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_dec_d<__nv_bfloat16>(a, s) : launch_dec_d<float>(a, s);
}

cudaError_t launch_residual_init(const DecodeArgs& a, cudaStream_t s) {
    if (a.dm.lam == 0) return cudaSuccess;
    return a.dm.dtype == 1 ? launch_rinit_d<__nv_bfloat16>(a, s) : launch_rinit_d<float>(a, s);
}

size_t decode_smem_bytes(const Dims& dm) {   // the smaller layout (residuals re-read from global)
    return (size_t)dec_offsets(dm.d, dm.Dh, dm.Gq, dm.lam, dm.eta, dm.esize).total * 4;
}

}  // namespace lola

// Stored-pair SRE map of the last prefill call (LoLA notes §4.4: Fig. 3, and
// Fig. 10 / Eq. 26 for the relative form).  For every state time c of the call
// (the state entering chunk c; c = nc is the state after the call) and every
// position i of the sequence:
//   sre[c][i] = || H_c^T phi(k_i) / (phi(k_i)^T s_c) - v_i ||^2   if pair i is
//               folded into (H_c, s_c), else 0,
//   rel[c][i] = sre[c][i] - sre[c_i][i], c_i = the first state time of the map
//               that holds pair i (0 where pair i is not folded).
// Pair i is folded at time c exactly when it has left the window
// (i < t_c - eta, t_c = first position of chunk c) and is not one of the
// cache members published for chunk c.  The prefill's snapshots (H_c^T, s_c
// and the member positions of each chunk) are the input; nothing is changed.
//
// One CTA per (stream, 64 positions), looping over the state times in order so
// that phi(k) and v of its positions are formed once and the first-write SRE
// stays in shared memory.  Per state time: H_c staged transposed into shared
// memory (row stride d + 4), den_i = phi_i . s_c in quarter sums, then an fp32
// register-tiled product (4 positions x d/16 columns per thread, paired FMAs)
// whose epilogue forms the squared residual and reduces it across the 16
// column groups of a half warp.  Chunks where no position of the tile has left
// the window yet only write zeros.
#include "device_common.cuh"

namespace lola {

constexpr int kMapTile = 64;
constexpr int kMapThreads = 256;

template <int DIM, int DH>
struct MapShape {
    static constexpr int D = 2 * DH;
    static constexpr int HLD = DIM + 4;              // row stride of the staged H_c (floats)
    static constexpr int H = 0;                       // [D][HLD]; W and key staging in the prologue
    static constexpr int PHI = H + D * HLD;           // [D][kMapTile] phi(k)^T of the tile
    static constexpr int S = PHI + D * kMapTile;      // [D] s_c
    static constexpr int DEN = S + D;                 // [4][kMapTile] partial phi_i . s_c, then phi_i . s_c
    static constexpr int FIRST = DEN + 4 * kMapTile;  // [kMapTile] SRE at first write
    static constexpr int FLAGS = FIRST + kMapTile;    // [kMapTile] bit 0: cache member at c; bit 1: seen
    static constexpr int total = FLAGS + kMapTile;    // floats
    static_assert(DIM * DH + 8 * DIM <= D * HLD, "prologue staging must fit the H_c buffer");
};

template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(kMapThreads, 2) sre_map_kernel(const __grid_constant__ SreMapArgs a) {
    using Sh = MapShape<DIM, DH>;
    constexpr int D = Sh::D, TILE = kMapTile, HLD = Sh::HLD, CPL = DH / 32;
    constexpr int NQ = DIM / 64;                      // column quads per thread: 64 u + 4 cg .. + 3
    constexpr int CPT = 4 * NQ;
    extern __shared__ __align__(16) float smem[];
    float* Hs = smem + Sh::H;
    float* Ph = smem + Sh::PHI;
    float* sc = smem + Sh::S;
    float* den = smem + Sh::DEN;
    float* first = smem + Sh::FIRST;
    int* flags = reinterpret_cast<int*>(smem + Sh::FLAGS);
    const Dims& dm = a.dm;
    const int st = blockIdx.y, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lo = blockIdx.x * TILE;
    const int nvalid = min(TILE, a.T - lo);
    const size_t snaps = (size_t)dm.nc_max + 1;
    float* sre_st = a.sre + (size_t)st * (a.nc + 1) * a.T;
    float* rel_st = a.rel ? a.rel + (size_t)st * (a.nc + 1) * a.T : nullptr;

    // ---- phi(k) of the tile's keys: the prefill's feature map, same arithmetic ----
    float* Ws = Hs;                                   // [DIM][DH]
    float* xs = Hs + DIM * DH;                        // [8][DIM]
    const TIn* Wg = (const TIn*)a.W + (size_t)g * DIM * DH;
    for (int i = tid; i < DIM * DH; i += kMapThreads) Ws[i] = to_f32(Wg[i]);
    if (tid < TILE) { flags[tid] = 0; first[tid] = 0.f; }
    __syncthreads();
    for (int r = 0; r < TILE / 8; ++r) {
        const int p = warp * (TILE / 8) + r;          // warp-uniform
        if (p < nvalid) {
            const TIn* x = (const TIn*)a.k + (((size_t)b * a.T + lo + p) * dm.Hkv + g) * DIM;
            for (int j = lane; j < DIM; j += 32) xs[warp * DIM + j] = to_f32(x[j]);
            __syncwarp();
            float z[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) z[c] = 0.f;
            for (int j = 0; j < DIM; ++j) {
                const float xj = xs[warp * DIM + j];
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
                Ph[(lane + 32 * c) * TILE + p] = ep[c] / sp;
                Ph[(DH + lane + 32 * c) * TILE + p] = en[c] / sn;
            }
            __syncwarp();
        } else {
            for (int j = lane; j < D; j += 32) Ph[j * TILE + p] = 0.f;
        }
    }
    // ---- the thread's values: positions 4 pg .. 4 pg + 3, columns 64 u + 4 cg .. + 3 ----
    const int pg = warp * 2 + (lane >> 4), cg = lane & 15;
    float vr[4][CPT];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int p = 4 * pg + q;
        const TIn* vrow = (const TIn*)a.v + (((size_t)b * a.T + lo + min(p, nvalid - 1)) * dm.Hkv + g) * DIM;
#pragma unroll
        for (int u = 0; u < NQ; ++u) {
            const float4 f = p < nvalid ? load4(vrow + 64 * u + 4 * cg) : make_float4(0.f, 0.f, 0.f, 0.f);
            vr[q][4 * u] = f.x; vr[q][4 * u + 1] = f.y; vr[q][4 * u + 2] = f.z; vr[q][4 * u + 3] = f.w;
        }
    }
    __syncthreads();                                  // W and key staging are dead from here

    for (int c = 0; c <= a.nc; ++c) {
        const int lim = a.t0 + c * dm.C - dm.eta;     // positions below lim have left the window
        float* srow = sre_st + (size_t)c * a.T + lo;
        float* rrow = rel_st ? rel_st + (size_t)c * a.T + lo : nullptr;
        if (lim <= lo) {                              // no pair of the tile is in the state yet
            for (int p = tid; p < nvalid; p += kMapThreads) {
                srow[p] = 0.f;
                if (rrow) rrow[p] = 0.f;
            }
            continue;
        }
        // cache members at time c among the tile's positions (positions are unique)
        const int ng = min(dm.lam, lim);
        const int* gpos = a.snap_pos + ((size_t)st * snaps + c) * dm.lam;
        if (tid < TILE) flags[tid] &= ~1;
        __syncthreads();
        for (int e = tid; e < ng; e += kMapThreads) {
            const int p = gpos[e] - lo;
            if (p >= 0 && p < TILE) flags[p] |= 1;
        }
        // H_c (rows j) from the snapshot H_c^T [DIM][D]; s_c
        const float* Hc = a.snap_H + ((size_t)st * snaps + c) * D * DIM;
        for (int it = tid; it < DIM * (D / 4); it += kMapThreads) {
            const int cc = it % DIM, j4 = it / DIM;
            const float4 h = *reinterpret_cast<const float4*>(Hc + (size_t)cc * D + 4 * j4);
            Hs[(4 * j4) * HLD + cc] = h.x;
            Hs[(4 * j4 + 1) * HLD + cc] = h.y;
            Hs[(4 * j4 + 2) * HLD + cc] = h.z;
            Hs[(4 * j4 + 3) * HLD + cc] = h.w;
        }
        for (int j = tid; j < D; j += kMapThreads) sc[j] = a.snap_s[((size_t)st * snaps + c) * D + j];
        __syncthreads();
        {                                             // den_i = phi_i . s_c: four quarter sums per position
            const int p = tid % TILE, part = tid / TILE;
            float x = 0.f;
#pragma unroll 8
            for (int j = part * (D / 4); j < (part + 1) * (D / 4); ++j) x = fmaf(Ph[j * TILE + p], sc[j], x);
            den[part * TILE + p] = x;
        }
        __syncthreads();
        if (tid < TILE) den[tid] = (den[tid] + den[TILE + tid]) + (den[2 * TILE + tid] + den[3 * TILE + tid]);
        __syncthreads();
        // numerators H_c^T phi_i of the thread's 4 positions x CPT columns
        unsigned long long acc[4][CPT / 2];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int m = 0; m < CPT / 2; ++m) acc[q][m] = 0ull;
#pragma unroll 4
        for (int j = 0; j < D; ++j) {
            const float4 ph = *reinterpret_cast<const float4*>(Ph + j * TILE + 4 * pg);
            unsigned long long hh[CPT / 2];
#pragma unroll
            for (int u = 0; u < NQ; ++u) {
                const float4 h = *reinterpret_cast<const float4*>(Hs + j * HLD + 64 * u + 4 * cg);
                hh[2 * u] = f2pack(h.x, h.y);
                hh[2 * u + 1] = f2pack(h.z, h.w);
            }
            const float pv[4] = {ph.x, ph.y, ph.z, ph.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const unsigned long long pp = f2pack(pv[q], pv[q]);
#pragma unroll
                for (int m = 0; m < CPT / 2; ++m) acc[q][m] = f2fma(pp, hh[m], acc[q][m]);
            }
        }
        // squared residual per position, summed over the 16 column groups of the half warp
        float sq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float dn = den[4 * pg + q];
            const float inv = dn > 0.f ? 1.f / dn : 0.f;
            float s2 = 0.f;
#pragma unroll
            for (int m = 0; m < CPT / 2; ++m) {
                float x, y;
                f2unpack(acc[q][m], x, y);
                const float rx = x * inv - vr[q][2 * m];
                const float ry = y * inv - vr[q][2 * m + 1];
                s2 = fmaf(rx, rx, s2);
                s2 = fmaf(ry, ry, s2);
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, off);
            sq[q] = s2;
        }
        if (cg == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int p = 4 * pg + q;
                if (p >= nvalid) continue;
                const int fl = flags[p];
                const bool member = lo + p < lim && !(fl & 1);
                float out = 0.f, r = 0.f;
                if (member) {
                    out = sq[q];
                    if (!(fl & 2)) { first[p] = out; flags[p] = fl | 2; }
                    r = out - first[p];
                }
                srow[p] = out;
                if (rrow) rrow[p] = r;
            }
        }
        __syncthreads();                              // H_c, s_c, den and flags are reused
    }
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_map_t(const SreMapArgs& a, cudaStream_t s) {
    const size_t bytes = (size_t)MapShape<DIM, DH>::total * 4;
    cudaError_t e = cudaFuncSetAttribute(sre_map_kernel<DIM, DH, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((a.T + kMapTile - 1) / kMapTile, a.dm.S);
    sre_map_kernel<DIM, DH, TIn><<<grid, kMapThreads, bytes, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_map_d(const SreMapArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (d == 64 && Dh == 32) return launch_map_t<64, 32, TIn>(a, s);
    if (d == 64 && Dh == 64) return launch_map_t<64, 64, TIn>(a, s);
    if (d == 128 && Dh == 32) return launch_map_t<128, 32, TIn>(a, s);
    if (d == 128 && Dh == 64) return launch_map_t<128, 64, TIn>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_sre_map(const SreMapArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_map_d<__nv_bfloat16>(a, s) : launch_map_d<float>(a, s);
}

}  // namespace lola

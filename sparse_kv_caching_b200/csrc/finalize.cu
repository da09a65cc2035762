// End of a prefill call: make the state self-contained for the next call.
//
// During the call, cache members and window pairs are read where they
// already are (input arrays, window ring, or their old cache slot; see
// lola_internal.h).  Afterwards two kernels copy (k, v, phi(k)) of every
// cache member that joined during the call into its slot, then write the
// call's last min(eta, T) tokens into the window ring (slot p % eta), so that
// the next call (prefill or decode) finds the memories of notes §2.4 (Fig. 1)
// in the state.  The cache copies read the old ring; the kernel boundary
// orders them before the ring is overwritten.
#include "device_common.cuh"

namespace lola {

constexpr int kSlotsPerBlock = 32;

// A row of the state is copied as 16-byte pieces: k and v (d elements each) then
// phi(k) (D floats); all rows start on 16-byte boundaries.
struct RowPieces {
    int kp, fp, per;                  // pieces of k (= of v), of phi, of a whole row
    __device__ RowPieces(const Dims& dm) : kp(dm.d * dm.esize / 16), fp(dm.D / 4), per(2 * kp + fp) {}
};

template <typename TIn>
__global__ void __launch_bounds__(256) finalize_cache_kernel(const __grid_constant__ PrefillArgs a) {
    const Dims& dm = a.dm;
    const int st = blockIdx.x, b = st / dm.Hkv, g = st % dm.Hkv;
    const int d = dm.d, D = dm.D, lam = dm.lam, eta = dm.eta;
    const int j0 = blockIdx.y * kSlotsPerBlock, nj = min(kSlotsPerBlock, lam - j0);
    const size_t snaps = (size_t)dm.nc_max + 1;
    const int* fin = a.snap_pos + ((size_t)st * snaps + a.nc) * lam;
    const RowPieces rp(dm);
    for (int idx = threadIdx.x; idx < nj * rp.per; idx += 256) {
        const int j = j0 + idx / rp.per, x = idx % rp.per;
        const int p = fin[j];
        const size_t cs = (size_t)st * lam + j;
        if (x == 0) a.sp.cache_pos[cs] = p;
        if (p < 0 || p < a.t_start - eta) continue;      // empty, or cached before this call
        const PairRef<TIn> r = pair_ref<TIn>(a, st, b, g, p, j);
        if (x < rp.kp)
            reinterpret_cast<uint4*>((TIn*)a.sp.cache_k + cs * d)[x] = reinterpret_cast<const uint4*>(r.k)[x];
        else if (x < 2 * rp.kp)
            reinterpret_cast<uint4*>((TIn*)a.sp.cache_v + cs * d)[x - rp.kp] =
                reinterpret_cast<const uint4*>(r.v)[x - rp.kp];
        else
            reinterpret_cast<float4*>(a.sp.cache_phik + cs * D)[x - 2 * rp.kp] =
                reinterpret_cast<const float4*>(r.phik)[x - 2 * rp.kp];
    }
}

template <typename TIn>
__global__ void __launch_bounds__(256) finalize_window_kernel(const __grid_constant__ PrefillArgs a) {
    const Dims& dm = a.dm;
    const int st = blockIdx.x, b = st / dm.Hkv, g = st % dm.Hkv;
    const int d = dm.d, D = dm.D, eta = dm.eta;
    const int t_end = a.t_start + a.T;
    const int p_lo = max(a.t_start, t_end - eta);
    const int p0 = p_lo + blockIdx.y * kSlotsPerBlock;
    const int np = min(kSlotsPerBlock, t_end - p0);
    const RowPieces rp(dm);
    for (int idx = threadIdx.x; idx < np * rp.per; idx += 256) {
        const int p = p0 + idx / rp.per, x = idx % rp.per;
        const size_t i = (size_t)(p - a.t_start);
        const size_t off = (((size_t)b * a.T + i) * dm.Hkv + g) * d;
        const size_t ws = (size_t)st * eta + (size_t)(p % eta);
        if (x < rp.kp)
            reinterpret_cast<uint4*>((TIn*)a.sp.win_k + ws * d)[x] = reinterpret_cast<const uint4*>((const TIn*)a.k + off)[x];
        else if (x < 2 * rp.kp)
            reinterpret_cast<uint4*>((TIn*)a.sp.win_v + ws * d)[x - rp.kp] =
                reinterpret_cast<const uint4*>((const TIn*)a.v + off)[x - rp.kp];
        else
            reinterpret_cast<float4*>(a.sp.win_phik + ws * D)[x - 2 * rp.kp] =
                reinterpret_cast<const float4*>(a.phik_new + ((size_t)st * dm.max_tokens + i) * D)[x - 2 * rp.kp];
    }
}

template <typename TIn>
static cudaError_t launch_fin_t(const PrefillArgs& a, cudaStream_t s) {
    if (a.dm.lam > 0) {
        dim3 g1(a.dm.S, (a.dm.lam + kSlotsPerBlock - 1) / kSlotsPerBlock);
        finalize_cache_kernel<TIn><<<g1, 256, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int nw = min(a.dm.eta, a.T);
    dim3 g2(a.dm.S, (nw + kSlotsPerBlock - 1) / kSlotsPerBlock);
    finalize_window_kernel<TIn><<<g2, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const PrefillArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_fin_t<__nv_bfloat16>(a, s) : launch_fin_t<float>(a, s);
}

}  // namespace lola

// Feature map of the new keys of a prefill call:
//   phi(k) = [softmax(k W_g), softmax(-k W_g)]   (Hedgehog form; D = 2 Dh)
// The pages only call phi "learned" (LoLA notes §2.1 notation table, §2.2);
// this library fixes the Hedgehog form with per-kv-head W.  fp32 FFMA with
// W staged in shared memory, exact softmax via expf.  Output layout
// phik_new [S][max_tokens][D] (row i = token t_start + i of stream st).
// A launch covers the tokens of chunks [c_begin, c_end) of the call.
#include "device_common.cuh"

namespace lola {

template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(256) phi_keys_kernel(PrefillArgs a) {
    constexpr int ROWS_PER_WARP = 16;            // 128 rows per block share one staging of W
    constexpr int CPL = DH / 32;                 // feature columns per lane (1 or 2)
    __shared__ float Ws[DIM * DH];
    __shared__ float xs[8][DIM];
    const Dims& dm = a.dm;
    const int st = blockIdx.y, b = st / dm.Hkv, g = st % dm.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const TIn* Wg = (const TIn*)a.sp.W + (size_t)g * DIM * DH;
    for (int i = threadIdx.x; i < DIM * DH; i += 256) Ws[i] = to_f32(Wg[i]);
    __syncthreads();
    const int i_end = a.c_end * dm.C;
    for (int r = 0; r < ROWS_PER_WARP; ++r) {
        const int i = a.c_begin * dm.C + (blockIdx.x * 8 + warp) * ROWS_PER_WARP + r;
        if (i >= i_end) break;
        const TIn* x = (const TIn*)a.k + (((size_t)b * a.T + i) * dm.Hkv + g) * DIM;
        for (int j = lane; j < DIM; j += 32) xs[warp][j] = to_f32(x[j]);
        __syncwarp();
        float z[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) z[c] = 0.f;
        for (int j = 0; j < DIM; ++j) {
            const float xj = xs[warp][j];
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
        float* out = a.phik_new + ((size_t)st * dm.max_tokens + i) * (2 * DH);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            out[lane + 32 * c] = ep[c] / sp;
            out[DH + lane + 32 * c] = en[c] / sn;
        }
        __syncwarp();
    }
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_phi_t(const PrefillArgs& a, cudaStream_t s) {
    const int rows_per_block = 8 * 16;
    const int rows = (a.c_end - a.c_begin) * a.dm.C;
    dim3 grid((rows + rows_per_block - 1) / rows_per_block, a.dm.S);
    phi_keys_kernel<DIM, DH, TIn><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_phi_d(const PrefillArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (d == 64 && Dh == 32) return launch_phi_t<64, 32, TIn>(a, s);
    if (d == 64 && Dh == 64) return launch_phi_t<64, 64, TIn>(a, s);
    if (d == 128 && Dh == 32) return launch_phi_t<128, 32, TIn>(a, s);
    if (d == 128 && Dh == 64) return launch_phi_t<128, 64, TIn>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_phi_keys(const PrefillArgs& a, cudaStream_t s) {
    return a.dm.dtype == 1 ? launch_phi_d<__nv_bfloat16>(a, s) : launch_phi_d<float>(a, s);
}

}  // namespace lola

// Feature map of the new keys of a prefill call:
//   phi(k) = [softmax(k W_g), softmax(-k W_g)]   (Hedgehog form; D = 2 Dh)
// The pages only call phi "learned" (LoLA notes §2.1 notation table, §2.2);
// this library fixes the Hedgehog form with per-kv-head W.  fp32 FFMA with
// W staged in shared memory (each W value read feeds 8 rows held in
// registers), exact softmax via expf.  Output layout
// phik_new [S][max_tokens][D] (row i = token t_start + i of stream st).
// A launch covers the tokens of chunks [c_begin, c_end) of the call.
#include "device_common.cuh"

namespace lola {

template <int DIM, int DH, typename TIn>
__global__ void __launch_bounds__(256) phi_keys_kernel(PrefillArgs a) {
    constexpr int RG = 8;                        // rows per warp and pass: one W read feeds RG rows
    constexpr int PASSES = 2;                    // 8 warps x 8 rows x 2 passes = 128 rows per block
    constexpr int CPL = DH / 32;                 // feature columns per lane (1 or 2)
    extern __shared__ __align__(16) float phi_smem[];
    float* Ws = phi_smem;                                           // [DIM][DH]
    float (*xs)[RG][DIM] = reinterpret_cast<float (*)[RG][DIM]>(phi_smem + DIM * DH);   // [8 warps]
    const Dims& dm = a.dm;
    const int st = blockIdx.y, b = st / dm.Hkv, g = st % dm.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const TIn* Wg = (const TIn*)a.sp.W + (size_t)g * DIM * DH;
    for (int i = threadIdx.x; i < DIM * DH; i += 256) Ws[i] = to_f32(Wg[i]);
    __syncthreads();
    const int i_end = a.c_end * dm.C;
    for (int pass = 0; pass < PASSES; ++pass) {
        const int i0 = a.c_begin * dm.C + ((blockIdx.x * PASSES + pass) * 8 + warp) * RG;
        if (i0 >= i_end) break;
        // the warp's RG rows of k (rows past the end repeat the last valid row, not stored)
        for (int idx = lane; idx < RG * DIM; idx += 32) {
            const int r = idx / DIM, j = idx % DIM, i = min(i0 + r, i_end - 1);
            xs[warp][r][j] = to_f32(((const TIn*)a.k)[(((size_t)b * a.T + i) * dm.Hkv + g) * DIM + j]);
        }
        __syncwarp();
        float z[RG][CPL];
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int c = 0; c < CPL; ++c) z[r][c] = 0.f;
#pragma unroll 2
        for (int j = 0; j < DIM; j += 4) {
            float w[4][CPL];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int c = 0; c < CPL; ++c) w[u][c] = Ws[(j + u) * DH + lane + 32 * c];
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                const float4 x = *reinterpret_cast<const float4*>(&xs[warp][r][j]);
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    z[r][c] = fmaf(x.x, w[0][c], z[r][c]);
                    z[r][c] = fmaf(x.y, w[1][c], z[r][c]);
                    z[r][c] = fmaf(x.z, w[2][c], z[r][c]);
                    z[r][c] = fmaf(x.w, w[3][c], z[r][c]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            const int i = i0 + r;
            float mx = -INFINITY, mn = INFINITY;
#pragma unroll
            for (int c = 0; c < CPL; ++c) { mx = fmaxf(mx, z[r][c]); mn = fminf(mn, z[r][c]); }
            mx = warp_max(mx);
            mn = -warp_max(-mn);
            float ep[CPL], en[CPL], sp = 0.f, sn = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                ep[c] = expf(z[r][c] - mx);
                en[c] = expf(mn - z[r][c]);
                sp += ep[c];
                sn += en[c];
            }
            sp = warp_sum(sp);
            sn = warp_sum(sn);
            if (i < i_end) {
                float* out = a.phik_new + ((size_t)st * dm.max_tokens + i) * (2 * DH);
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    out[lane + 32 * c] = ep[c] / sp;
                    out[DH + lane + 32 * c] = en[c] / sn;
                }
            }
        }
        __syncwarp();
    }
}

template <int DIM, int DH, typename TIn>
static cudaError_t launch_phi_t(const PrefillArgs& a, cudaStream_t s) {
    const int rows_per_block = 8 * 8 * 2;
    const int rows = (a.c_end - a.c_begin) * a.dm.C;
    dim3 grid((rows + rows_per_block - 1) / rows_per_block, a.dm.S);
    const int bytes = (DIM * DH + 8 * 8 * DIM) * 4;
    cudaError_t e = cudaFuncSetAttribute(phi_keys_kernel<DIM, DH, TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    phi_keys_kernel<DIM, DH, TIn><<<grid, 256, bytes, s>>>(a);
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

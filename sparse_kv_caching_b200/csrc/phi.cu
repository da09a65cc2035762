// Feature map of the new keys of a prefill call:
//   phi(k) = [softmax(k W_g), softmax(-k W_g)]   (Hedgehog form; D = 2 Dh)
// The pages only call phi "learned" (LoLA notes §2.1 notation table, §2.2);
// this library fixes the Hedgehog form with per-kv-head W.  fp32 FFMA with
// W staged in shared memory (each W value read feeds 8 rows held in
// registers), exact softmax via expf.  Output layout
// phik_new [S][max_tokens][D] (row i = token t_start + i of stream st).
// A launch covers the tokens of chunks [c_begin, c_end) of the call.
#include "device_common.cuh"
#include "umma.cuh"

namespace lola {

// The same map for bf16 inputs with z = k W on the tensor cores: one CTA takes 128
// key rows (thread r owns row r), the rows are copied into a 128-byte swizzled
// K-major operand, W into a chunk-major MN-major one, and z [128 x DH] f32 lands
// in tensor memory (bf16 products are exact, the accumulation f32); each thread
// then reads its row of z and writes its row of phi with expf as above.
template <int DIM, int DH>
__global__ void __launch_bounds__(128) phi_keys_tc_kernel(const __grid_constant__ PrefillArgs a) {
    using bf16 = __nv_bfloat16;
    constexpr int ROWS = 128, KB = DIM / 64;
    constexpr int KBYTES = ROWS * DIM * 2, WBYTES = DIM * DH * 2;
    extern __shared__ __align__(1024) uint8_t phi_tc_raw[];
    uint8_t* smem = phi_tc_raw + ((1024u - (umma::smem_addr(phi_tc_raw) & 1023u)) & 1023u);
    uint8_t* sK = smem;
    uint8_t* sW = smem + KBYTES;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + KBYTES + WBYTES);
    uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + KBYTES + WBYTES + 8);
    const Dims& dm = a.dm;
    const int st = blockIdx.y, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int i_begin = a.c_begin * dm.C, i_end = a.c_end * dm.C;
    const int i0 = i_begin + blockIdx.x * ROWS;
    if (warp == 0) umma::tmem_alloc(tptr, 64);
    if (tid == 0) { umma::mbar_init(mbar, 1); umma::fence_mbar_init(); }
    // rows i0 .. i0 + 127 (past the end: zero), eight threads per 128-byte piece
    const bf16* kbase = (const bf16*)a.k + ((size_t)b * a.T * dm.Hkv + g) * DIM;
    for (int idx = tid; idx < ROWS * DIM / 8; idx += ROWS) {
        const int c = idx & 7, kb = (idx >> 3) % KB, r = (idx >> 3) / KB, i = i0 + r;
        const bool valid = i < i_end;
        umma::cp_async16_zfill(sK + kb * (ROWS * 128) + umma::sw128_off(r, c),
                               kbase + (size_t)(valid ? i : i_begin) * dm.Hkv * DIM + 64 * kb + 8 * c, valid);
    }
    const bf16* Wg = (const bf16*)a.sp.W + (size_t)g * DIM * DH;   // [DIM][DH]
    for (int idx = tid; idx < DIM * (DH / 8); idx += ROWS) {
        const int k = idx % DIM, n8 = idx / DIM;
        umma::cp_async16(sW + n8 * DIM * 16 + k * 16, Wg + (size_t)k * DH + 8 * n8);
    }
    umma::cp_async_commit();
    umma::cp_async_wait<0>();
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tptr;
    if (tid == 0) {
        const uint32_t id = umma::idesc(umma::kBF16, ROWS, DH, false, true);
#pragma unroll
        for (int ks = 0; ks < DIM / 16; ++ks)
            umma::mma_bf16(tmem, umma::sdesc_sw128(umma::smem_addr(sK) + (ks >> 2) * ROWS * 128 + (ks & 3) * 32, 16, 1024),
                           umma::sdesc(umma::smem_addr(sW) + ks * 16 * 16, 128, DIM * 16), id, ks > 0 ? 1u : 0u);
        umma::commit(mbar);
    }
    const bool ok = umma::mbar_wait(mbar, 0);
    umma::fence_after_sync();
    float z[DH];
#pragma unroll
    for (int c0 = 0; c0 < DH; c0 += 16)
        umma::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + c0, *reinterpret_cast<float(*)[16]>(z + c0));
    umma::tmem_wait_ld();
    const int i = i0 + tid;
    if (ok && i < i_end) {
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int c = 0; c < DH; ++c) { mx = fmaxf(mx, z[c]); mn = fminf(mn, z[c]); }
        float sp = 0.f, sn = 0.f;
#pragma unroll
        for (int c = 0; c < DH; ++c) { sp += expf(z[c] - mx); sn += expf(mn - z[c]); }
        const float isp = 1.f / sp, isn = 1.f / sn;
        float4* out = reinterpret_cast<float4*>(a.phik_new + ((size_t)st * dm.max_tokens + i) * (2 * DH));
#pragma unroll
        for (int c = 0; c < DH; c += 4)
            out[c / 4] = make_float4(expf(z[c] - mx) * isp, expf(z[c + 1] - mx) * isp, expf(z[c + 2] - mx) * isp,
                                     expf(z[c + 3] - mx) * isp);
#pragma unroll
        for (int c = 0; c < DH; c += 4)
            out[(DH + c) / 4] = make_float4(expf(mn - z[c]) * isn, expf(mn - z[c + 1]) * isn, expf(mn - z[c + 2]) * isn,
                                            expf(mn - z[c + 3]) * isn);
    }
    if (!ok && tid == 0 && a.err) atomicOr(a.err, 1);
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, 64);
}

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

template <int DIM, int DH>
static cudaError_t launch_phi_tc_t(const PrefillArgs& a, cudaStream_t s) {
    const int rows = (a.c_end - a.c_begin) * a.dm.C;
    dim3 grid((rows + 127) / 128, a.dm.S);
    const int bytes = 128 * DIM * 2 + DIM * DH * 2 + 16 + 1024;   // K, W, barrier + tmem slot, alignment slack
    cudaError_t e = cudaFuncSetAttribute(phi_keys_tc_kernel<DIM, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    phi_keys_tc_kernel<DIM, DH><<<grid, 128, bytes, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_phi_keys(const PrefillArgs& a, cudaStream_t s) {
    if (a.dm.dtype == 1) {
        const int d = a.dm.d, Dh = a.dm.Dh;
        if (d == 128 && Dh == 64) return launch_phi_tc_t<128, 64>(a, s);
        if (d == 128 && Dh == 32) return launch_phi_tc_t<128, 32>(a, s);
        if (d == 64 && Dh == 64) return launch_phi_tc_t<64, 64>(a, s);
        if (d == 64 && Dh == 32) return launch_phi_tc_t<64, 32>(a, s);
        return launch_phi_d<__nv_bfloat16>(a, s);
    }
    return launch_phi_d<float>(a, s);
}

}  // namespace lola

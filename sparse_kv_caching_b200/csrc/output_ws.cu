// Hybrid output of chunkwise LoLA prefill on the fifth-generation tensor
// cores, warp-specialised (bf16 inputs).  Same computation as output.cu and
// the notes' Eq. 14 (§2.5, §2.6):
//   y_t = (H_c^T phi(q_t) + sum_i e^{a_ti} v_i) / (phi(q_t)^T s_c + sum_i e^{a_ti})
// over i in G_c u W_c u {block keys <= t}, one shared normaliser.
//
// One CTA serves 256 query rows (row = (head of the kv group, query of block
// c)) as two 128-row tiles A and B that read the same gathered keys, so every
// K/V tile fetched from L2 feeds twice the tensor-core work (d = 128; d = 64
// runs one 128-row tile per CTA).  Roles:
//   warps 0-3 / 4-7  softmax and epilogue of tile A / B (thread r owns row r)
//   warps 8-9        gather K and V rows of each 64-key tile with cp.async
//                    into a 5-stage ring (row addresses looked up once per key
//                    and shared by shuffles, each key's cache position read
//                    one tile ahead); tile A's softmax warps turn V into f16
//                    in place once their weights are stored
// K and V tiles sit in the 128-byte swizzled layout: each 128-byte half of a
// key row is one contiguous shared-memory row (its 16-byte chunks permuted), so
// the eight lanes that copy it touch one global line and one shared row, and
// the same bytes serve as the K-major B operand of Q K^T and the MN-major B
// operand of P V.
//   warp 10, lane 0  issues every MMA
// Tensor memory: O_A, O_B [128 x d] f32 and two S buffers per tile [128 x 64].
// Per key tile j the MMA thread issues S_t(j+1) = Q_t K^T (bf16) while the
// softmax warps turn S_t(j) into P_t (f16, exp2 in the log2 domain with a
// lazily raised reference maximum) and store it over S_t(j) in tensor memory
// (two f16 per column); then O_t += P_t V (f16, A = P_t read from tensor
// memory, B = V from shared memory).
// Prologue (all warps, before the roles split): z = Q W (bf16 MMA), phi(q)
// in registers, O_t = phi(q)^T H_c (tf32 MMA over 32-column chunks), l =
// phi(q) . s_c: the linear branch enters the online softmax as logit 0.
// Every wait is bounded; a wait that gives up raises an abort flag that
// releases all other waits of the CTA, and sets the state's error word.
#include "device_common.cuh"
#include "umma.cuh"

namespace lola {

template <int DIM, int DH>
struct WsShape {
    static constexpr int ROWS = 128, KT = 64, D = 2 * DH, NCH = DIM / 8, NST = 5;
    static constexpr int NT = 352;                              // 11 warps
    // query tiles per CTA: two 128-row tiles share every gathered key tile for d = 128;
    // one for d = 64 (with two tiles at d = 64 the second tile's scores came out wrong
    // on the B200s here, a fault not explained by the operand layouts; see the tests)
    static constexpr int NTILE = DIM == 128 ? 2 : 1;
    static constexpr int QB = ROWS * DIM * 2;                   // one query tile (bf16)
    static constexpr int KVB = KT * DIM * 2;                    // one K or V tile
    static constexpr int Q = 0;                                 // [2 tiles]
    static constexpr int KV = Q + NTILE * QB;                   // [NST][K, V]
    static constexpr int MBAR = KV + NST * 2 * KVB;             // 19 barriers
    static constexpr int FLAG = MBAR + 24 * 8;                  // abort flag, tmem pointer
    static constexpr int END = FLAG + 16;
    static constexpr int KPOS = MBAR;                           // (end of the prologue aliases)
    // prologue aliases (the KV and P regions are free until the roles start)
    static constexpr int HT = KV;                               // H_c^T, [D/32][DIM x 32] f32
    static constexpr int HTC = DIM * 32 * 4;
    static constexpr int W = HT + (D / 32) * HTC;               // W [DIM][DH] bf16, MN-major B
    static constexpr int PHIS = NTILE * ROWS * 32 * 4;          // one 32-column piece of phi(q), both tiles
    static constexpr int PHI = W + DIM * DH * 2;                // [2 pieces][2 tiles][128 x 32] f32
    static constexpr int SC = PHI + 2 * PHIS;                   // s_c [D] f32
    static_assert(SC + D * 4 <= KPOS, "prologue buffers must fit in the KV and P regions");
    // tensor-memory columns
    // O of tile t at column t * OT (each output tile on a 128-column boundary), the four
    // S buffers from column TS
    static constexpr uint32_t TO = 0, OT = 128, TS = 256, TMEM_COLS = 512;
    static_assert(DIM <= (int)OT && TS + 4 * KT <= 512, "tensor memory");
};

// barrier indices (five ring stages): K and V landed, stage free; S ready (two buffers
// per query tile), P ready (for tile A: V in f16 too), P V done (per query tile); prologue
enum : int { kKvFull = 0, kKvFree = 5, kSFull = 10, kPFull = 14, kPvDone = 16, kPro = 18 };

// Bounded mbarrier wait that also gives up once another thread of the CTA has
// raised the abort flag; returns false if it gave up (and raises the flag).
__device__ __forceinline__ bool ws_wait(uint64_t* mbar, uint32_t parity, volatile int* abort) {
    if (umma::mbar_try_wait(mbar, parity)) return true;
    const uint64_t t0 = umma::globaltimer_ns();
    while (!umma::mbar_try_wait(mbar, parity)) {
        if (*abort) return false;
        if (umma::globaltimer_ns() - t0 > 4000000000ull) { *abort = 1; return false; }
    }
    return true;
}


__device__ __forceinline__ float ws_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t ws_pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t ws_bf2_to_h2(uint32_t u) {
    return ws_pack_f16(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ void ws_st4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" :: "r"(umma::smem_addr(p)), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// N columns (a multiple of 16) of this warp's lanes from tensor memory, one wait.
template <int N>
__device__ __forceinline__ void ws_tmem_ld(uint32_t taddr, float (&r)[N]) {
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 16) umma::tmem_ld16(taddr + c0, *reinterpret_cast<float(*)[16]>(r + c0));
    umma::tmem_wait_ld();
}

template <int DIM, int DH>
__global__ void __launch_bounds__(352, 1) output_ws_kernel(const __grid_constant__ PrefillArgs a) {
    using Sh = WsShape<DIM, DH>;
    using bf16 = __nv_bfloat16;
    constexpr int ROWS = Sh::ROWS, KT = Sh::KT, D = Sh::D, NCH = Sh::NCH, NST = Sh::NST, NT = Sh::NT;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzle atoms want 1024-byte aligned tiles (the launch adds the slack)
    uint8_t* smem = smem_raw + ((1024u - (umma::smem_addr(smem_raw) & 1023u)) & 1023u);
    const Dims& dm = a.dm;
    const int rows_total = dm.Gq * dm.C;
    constexpr int NTILE = Sh::NTILE;
    const int nrp = (rows_total + NTILE * ROWS - 1) / (NTILE * ROWS);
    const int c = a.c_begin + (int)blockIdx.x / nrp, rp = blockIdx.x % nrp;
    const int g = blockIdx.y, b = blockIdx.z, st = b * dm.Hkv + g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = a.t_start + c * dm.C;
    const int rfirst = rp * NTILE * ROWS, rlast = min(rows_total, rfirst + NTILE * ROWS) - 1;
    const bool twoB = NTILE == 2 && rlast >= rfirst + ROWS;    // tile B holds rows
    const int qi_max = (rlast / dm.C != rfirst / dm.C) ? dm.C - 1 : rlast % dm.C;
    const size_t snaps = (size_t)dm.nc_max + 1;
    const bool has_lin = (t0 - dm.eta) > dm.lam && !(a.read_mask & 1);
    const int n_g = (a.read_mask & 2) ? 0 : min(dm.lam, max(0, t0 - dm.eta));
    const int w_lo = max(0, t0 - dm.eta), n_w = t0 - w_lo;
    const int N = n_g + n_w + qi_max + 1;
    const int ntiles = (N + KT - 1) / KT;

    uint8_t* sQ = smem + Sh::Q;
    uint8_t* sKV = smem + Sh::KV;
    static_assert(NST == 5, "barrier indices assume five stages");
    const int* cpos = a.snap_pos + ((size_t)st * snaps + c) * dm.lam;   // cache positions of the block
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + Sh::MBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Sh::FLAG);
    uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + Sh::FLAG + 8);

    if (warp == 0) umma::tmem_alloc(tptr, Sh::TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            umma::mbar_init(&mbar[kKvFull + i], 64);
            umma::mbar_init(&mbar[kKvFree + i], 1);
        }
        for (int i = 0; i < 4; ++i) umma::mbar_init(&mbar[kSFull + i], 1);
        for (int t = 0; t < 2; ++t) { umma::mbar_init(&mbar[kPFull + t], ROWS); umma::mbar_init(&mbar[kPvDone + t], 1); }
        umma::mbar_init(&mbar[kPro], 1);
        *abort_flag = 0;
        umma::fence_mbar_init();
    }

    // ---- prologue: queries of both tiles, 128-byte swizzled (block kb holds dims
    // 64 kb .. 64 kb + 63 of every row; eight lanes copy one 128-byte piece) ----
    for (int idx = tid; idx < NTILE * ROWS * NCH; idx += NT) {
        const int c = idx & 7, kb = (idx >> 3) % (DIM / 64), rt = (idx >> 3) / (DIM / 64);
        const int r = rt % ROWS, t = rt / ROWS;
        uint8_t* dst = sQ + t * Sh::QB + kb * (ROWS * 128) + umma::sw128_off(r, c);
        const int R = rfirst + t * ROWS + r;
        if (R < rows_total) {
            const int hr = g * dm.Gq + R / dm.C, ir = R % dm.C;
            umma::cp_async16(dst, (const bf16*)a.q + (((size_t)b * a.T + (t0 + ir - a.t_start)) * dm.Hq + hr) * DIM +
                                      64 * kb + 8 * c);
        } else {
            ws_st4(dst, 0u, 0u, 0u, 0u);
        }
    }
    const float* Hc = a.snap_H + ((size_t)st * snaps + c) * D * DIM;     // H_c^T [DIM][D]
    const float* sc_g = a.snap_s + ((size_t)st * snaps + c) * D;
    float* s_c = reinterpret_cast<float*>(smem + Sh::SC);
    if (has_lin) {
        const bf16* Wg = (const bf16*)a.sp.W + (size_t)g * DIM * DH;   // [DIM][DH]; MN-major B
        for (int idx = tid; idx < DIM * (DH / 8); idx += NT) {
            const int k = idx % DIM, n8 = idx / DIM;
            umma::cp_async16(smem + Sh::W + n8 * DIM * 16 + k * 16, Wg + (size_t)k * DH + 8 * n8);
        }
        for (int idx = tid; idx < D / 4; idx += NT) umma::cp_async16(s_c + 4 * idx, sc_g + 4 * idx);
    }
    umma::cp_async_commit();                                   // group: Q, W, s_c
    if (has_lin) {
        // H_c^T piece ch (its columns 32 ch .. 32 ch + 31) as a K-major tf32 operand, 128-byte
        // swizzled: row cc of the piece is 128 contiguous bytes of H_c^T row cc
        for (int idx = tid; idx < (D / 32) * DIM * 8; idx += NT) {
            const int c = idx & 7, cc = (idx >> 3) % DIM, ch = (idx >> 3) / DIM;
            umma::cp_async16(smem + Sh::HT + ch * Sh::HTC + umma::sw128_off(cc, c), Hc + (size_t)cc * D + 32 * ch + 4 * c);
        }
    }
    umma::cp_async_commit();                                   // group: H_c^T (needed after phi(q))
    umma::cp_async_wait<1>();
    umma::fence_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tptr;
    const int wg = warp < 4 ? 0 : (warp < 8 ? 1 : 2);          // 0, 1: softmax tiles A, B; 2: loader / MMA
    const int r = tid & (ROWS - 1);                            // row within the tile (softmax warps)
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int R = rfirst + wg * ROWS + r;
    const bool row_ok = wg < 2 && R < rows_total;
    const int qpos = t0 + (row_ok ? R % dm.C : 0);
    const bool mma_thread = warp == 10 && lane == 0;
    bool dead = false;
    float l = 0.f;
    uint32_t pro_phase = 0;

    // ---- prologue: the linear branch (phi(q)^T H_c, phi(q) . s_c) of both tiles ----
    if (has_lin) {
        if (mma_thread) {
            const uint32_t id = umma::idesc(umma::kBF16, ROWS, DH, false, true);
            for (int t = 0; t < (twoB ? 2 : 1); ++t)
                for (int ks = 0; ks < DIM / 16; ++ks)
                    umma::mma_bf16(tmem + Sh::TS + 2 * t * KT,
                                   umma::sdesc_sw128(umma::smem_addr(sQ + t * Sh::QB) + (ks >> 2) * ROWS * 128 + (ks & 3) * 32,
                                                     16, 1024),
                                   umma::sdesc(umma::smem_addr(smem + Sh::W) + ks * 16 * 16, 128, DIM * 16), id, ks > 0);
            umma::commit(&mbar[kPro]);
        }
        dead |= !ws_wait(&mbar[kPro], pro_phase, abort_flag);
        pro_phase ^= 1;
        umma::fence_after_sync();
        // phi(q) = [softmax(z), softmax(-z)] with z in the log2 domain (exp2 on the XU; the
        // feature map of the queries reaches y only, within its tolerance)
        constexpr float kLog2e = 1.4426950408889634f;
        float z[DH];
        float mx = -INFINITY, mn = INFINITY, isp = 0.f, isn = 0.f;
        if (wg < (twoB ? 2 : 1)) {
            ws_tmem_ld<DH>(tmem + lane_off + Sh::TS + 2 * wg * KT, z);
#pragma unroll
            for (int i = 0; i < DH; ++i) { z[i] *= kLog2e; mx = fmaxf(mx, z[i]); mn = fminf(mn, z[i]); }
            float sp = 0.f, sn = 0.f;
#pragma unroll
            for (int i = 0; i < DH; ++i) { sp += ws_ex2(z[i] - mx); sn += ws_ex2(mn - z[i]); }
            isp = 1.f / sp;
            isn = 1.f / sn;
        }
        umma::cp_async_wait<0>();                              // H_c^T
        umma::fence_async_smem();
        // two 32-column pieces of phi(q) per round: store them, then their products
#pragma unroll
        for (int j0 = 0; j0 < D; j0 += 64) {
            if (wg < (twoB ? 2 : 1)) {
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint8_t* sPhi = smem + Sh::PHI + q * Sh::PHIS + wg * ROWS * 32 * 4;
#pragma unroll
                    for (int jq = 0; jq < 8; ++jq) {
                        float f[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int j = j0 + 32 * q + 4 * jq + u;
                            f[u] = j < DH ? ws_ex2(z[j] - mx) * isp : ws_ex2(mn - z[j - DH]) * isn;
                            l = fmaf(f[u], s_c[j], l);
                        }
                        ws_st4(sPhi + jq * ROWS * 16 + r * 16, __float_as_uint(f[0]), __float_as_uint(f[1]),
                               __float_as_uint(f[2]), __float_as_uint(f[3]));
                    }
                }
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncthreads();
            umma::fence_after_sync();
            if (mma_thread && !dead) {
                const uint32_t id = umma::idesc(umma::kTF32, ROWS, DIM, false, false);
                for (int q = 0; q < 2; ++q) {
                    const int jc = j0 + 32 * q;
                    const uint8_t* sHt = smem + Sh::HT + (jc / 32) * Sh::HTC;
                    for (int t = 0; t < (twoB ? 2 : 1); ++t)
                        for (int ks = 0; ks < 4; ++ks)
                            umma::mma_tf32(tmem + Sh::TO + t * Sh::OT,
                                           umma::sdesc(umma::smem_addr(smem + Sh::PHI + q * Sh::PHIS + t * ROWS * 32 * 4) +
                                                           ks * 2 * ROWS * 16,
                                                       ROWS * 16, 128),
                                           umma::sdesc_sw128(umma::smem_addr(sHt) + ks * 32, 16, 1024), id,
                                           (jc > 0 || ks > 0) ? 1u : 0u);
                }
                umma::commit(&mbar[kPro]);
            }
            dead |= !ws_wait(&mbar[kPro], pro_phase, abort_flag);
            pro_phase ^= 1;
            umma::fence_after_sync();
        }
        if (!row_ok) l = 0.f;
    }
    umma::fence_before_sync();
    __syncthreads();                                           // prologue buffers are free again
    umma::fence_after_sync();

    if (wg == 2 && warp < 10) {
        // ---- loaders: warp 8 takes keys 0-31 of every tile, warp 9 keys 32-63 ----
        constexpr int NH = DIM / 64;                           // 128-byte halves of a key row
        constexpr int HB = KT * 128;                           // one half of a K or V tile
        const int kb = (warp - 8) * 32;
        auto landed = [&](int s) {                             // this warp's copies of stage s are in
            umma::fence_async_smem();
            umma::mbar_arrive(&mbar[kKvFull + s]);
        };
        // the cache position of this lane's key, loaded one tile ahead
        int pos_c = kb + lane < n_g ? cpos[kb + lane] : 0;
        for (int j = 0; j < ntiles; ++j) {
            const int s = j % NST;
            const int gk_next = (j + 1) * KT + kb + lane;
            const int pos_n = gk_next < n_g ? cpos[gk_next] : 0;
            if (j >= NST) {
                bool ok = true;
                if (lane == 0 && !dead) ok = ws_wait(&mbar[kKvFree + s], ((j / NST) - 1) & 1, abort_flag);
                dead |= !__shfl_sync(0xffffffffu, ok ? 1 : 0, 0);
            }
            // where my key lives (cache slot, window, or block key up to the last query); keys
            // past the last one are zero-filled (their source address is only a placeholder)
            unsigned long long kr = reinterpret_cast<unsigned long long>(a.k), dv = 0;
            bool valid = false;
            {
                const int gk = j * KT + kb + lane;
                if (gk < N && !dead) {
                    const int pos = gk < n_g ? pos_c : (gk < n_g + n_w ? w_lo + (gk - n_g) : t0 + (gk - n_g - n_w));
                    const PairRef<bf16> pr = pair_ref<bf16>(a, st, b, g, pos, gk < n_g ? gk : 0);
                    kr = reinterpret_cast<unsigned long long>(pr.k);
                    dv = reinterpret_cast<unsigned long long>(pr.v) - kr;
                    valid = true;
                }
            }
            pos_c = pos_n;
            uint8_t* sK = sKV + s * 2 * Sh::KVB;
            uint8_t* sV = sK + Sh::KVB;
            // one 16-byte chunk of K and of V per lane and pass: eight lanes per half row,
            // four half rows per pass
#pragma unroll
            for (int it = 0; it < NH * 8; ++it) {
                const int q = it * 32 + lane, c = q & 7, kh = q >> 3;
                const int kl = NH == 2 ? kh >> 1 : kh, hf = NH == 2 ? (kh & 1) : 0;
                const unsigned long long kq = __shfl_sync(0xffffffffu, kr, kl);
                const unsigned long long dq = __shfl_sync(0xffffffffu, dv, kl);
                const bool vq = __shfl_sync(0xffffffffu, valid ? 1 : 0, kl) != 0;
                const uint32_t off = hf * HB + umma::sw128_off(kb + kl, c);
                const bf16* ks = reinterpret_cast<const bf16*>(kq) + 64 * hf + 8 * c;
                umma::cp_async16_zfill(sK + off, ks, vq);
                umma::cp_async16_zfill(sV + off, vq ? reinterpret_cast<const bf16*>(kq + dq) + 64 * hf + 8 * c : ks, vq);
            }
            umma::cp_async_commit();
            if (j >= 1) {
                umma::cp_async_wait<1>();
                __syncwarp();
                landed((j - 1) % NST);
            }
        }
        if (ntiles > 0) {
            umma::cp_async_wait<0>();
            __syncwarp();
            landed((ntiles - 1) % NST);
        }
    } else if (wg == 2) {
        // ---- MMA issuer ----
        if (mma_thread) {
            const uint32_t idS = umma::idesc(umma::kBF16, ROWS, KT, false, false);
            const uint32_t idO = umma::idesc(umma::kF16, ROWS, DIM, false, true);   // A = P in tensor memory
            const int ntl = twoB ? 2 : 1;
            // operand descriptors built once (the address field counts 16-byte units).  Q and K
            // (swizzled, K-major): a K step moves the start by 32 bytes inside a 128-byte half
            // row, the next half ROWS (KT) rows further.  V (swizzled, MN-major): 16 key rows of 128 bytes.  P (tensor
            // memory, two f16 per column): 8 columns.
            const uint64_t dQ0 = umma::sdesc_sw128(umma::smem_addr(sQ), 16, 1024);
            const uint64_t dQ1 = umma::sdesc_sw128(umma::smem_addr(sQ + (NTILE - 1) * Sh::QB), 16, 1024);
            // stage s sits 2 KVB bytes after stage s - 1
            const uint64_t dK0 = umma::sdesc_sw128(umma::smem_addr(sKV), 16, 1024);
            const uint64_t dV0 = umma::sdesc_sw128(umma::smem_addr(sKV + Sh::KVB), KT * 128, 1024);
            auto issue_s = [&](int j) {
                const int s = j % NST;
                const uint64_t bk = dK0 + (uint64_t)(s * (2 * Sh::KVB / 16));
                const uint32_t d0 = tmem + Sh::TS + (j & 1) * KT;
#pragma unroll
                for (int ks = 0; ks < DIM / 16; ++ks)
                    umma::mma_bf16(d0, dQ0 + (uint64_t)((ks >> 2) * ROWS * 8 + (ks & 3) * 2),
                                   bk + (uint64_t)((ks >> 2) * KT * 8 + (ks & 3) * 2), idS, ks > 0 ? 1u : 0u);
                umma::commit(&mbar[kSFull + (j & 1)]);
                if (ntl > 1) {
#pragma unroll
                    for (int ks = 0; ks < DIM / 16; ++ks)
                        umma::mma_bf16(d0 + 2 * KT, dQ1 + (uint64_t)((ks >> 2) * ROWS * 8 + (ks & 3) * 2),
                                       bk + (uint64_t)((ks >> 2) * KT * 8 + (ks & 3) * 2), idS, ks > 0 ? 1u : 0u);
                    umma::commit(&mbar[kSFull + 2 + (j & 1)]);
                }
            };
            // Non-blocking schedule: tile j's P V products are issued as soon as its softmax
            // is done, the next tile's scores as soon as its keys have landed and an S buffer
            // is free (S(j) reuses the buffer of S(j - 2) and P(j - 2): the issue of P V (j - 2)
            // has waited for that softmax, and the tensor cores run P V (j - 2) before S(j)).
            int js = 0, jp = 0, tp = 0;                       // next S tile; next P V tile and query tile
            uint64_t idle_since = umma::globaltimer_ns();
            while (jp < ntiles && !dead) {
                bool progress = false;
                // test_wait, not try_wait: a try_wait on a barrier that is not ready may
                // suspend this thread while the other one completes
                if (js < ntiles && js <= jp + 1 &&
                    umma::mbar_test_wait(&mbar[kKvFull + js % NST], (js / NST) & 1)) {
                    umma::fence_after_sync();
                    issue_s(js);
                    ++js;
                    progress = true;
                }
                // (tile B's P V follows tile A's, whose P barrier also covers V in f16)
                if (jp < js && umma::mbar_test_wait(&mbar[kPFull + tp], jp & 1)) {
                    umma::fence_after_sync();
                    const int sj = jp % NST;
                    const uint64_t bv = dV0 + (uint64_t)(sj * (2 * Sh::KVB / 16));
                    const uint32_t first = (has_lin || jp > 0) ? 1u : 0u;
                    const uint32_t aP = tmem + Sh::TS + (2 * tp + (jp & 1)) * KT;
                    const uint32_t dO = tmem + Sh::TO + tp * Sh::OT;
#pragma unroll
                    for (int ks = 0; ks < KT / 16; ++ks)
                        umma::mma_f16_ts(dO, aP + 8 * ks, bv + (uint64_t)(ks * 128), idO, ks > 0 ? 1u : first);
                    umma::commit(&mbar[kPvDone + tp]);
                    if (++tp == ntl) {                        // both query tiles done with this key tile
                        umma::commit(&mbar[kKvFree + jp % NST]);
                        tp = 0;
                        ++jp;
                    }
                    progress = true;
                }
                if (progress) {
                    idle_since = umma::globaltimer_ns();
                } else if (*abort_flag) {
                    dead = true;
                } else if (umma::globaltimer_ns() - idle_since > 4000000000ull) {
                    *abort_flag = 1;
                    dead = true;
                }
            }
        }
    } else if (wg == 0 || twoB) {
        // ---- softmax of tile wg: thread r owns row r ----
        const int t = wg;
        const float c2 = 1.4426950408889634f / sqrtf((float)DIM);    // log2(e) / sqrt(d)
        float m_ref = 0.f;
        for (int j = 0; j < ntiles; ++j) {
            bool ok = !dead;
            if (ok) ok = ws_wait(&mbar[kSFull + 2 * t + (j & 1)], (j >> 1) & 1, abort_flag);
            dead |= !__all_sync(0xffffffffu, ok);
            if (dead) break;
            umma::fence_after_sync();
            float sv[KT];
            ws_tmem_ld<KT>(tmem + lane_off + Sh::TS + (2 * t + (j & 1)) * KT, sv);
            // cache and window keys precede the block; block key m is visible to query qi iff
            // m <= qi: key i of tile j is visible iff j KT + i < lim
            const int lim = row_ok ? min(N, n_g + n_w + (qpos - t0) + 1) - j * KT : 0;
            float mx = -INFINITY;
            if (lim >= KT) {
#pragma unroll
                for (int i = 0; i < KT; ++i) mx = fmaxf(mx, sv[i]);
            } else {
#pragma unroll
                for (int i = 0; i < KT; ++i) {
                    sv[i] = i < lim ? sv[i] : -INFINITY;
                    mx = fmaxf(mx, sv[i]);
                }
            }
            mx *= c2;                                             // scores in the log2 domain (c2 > 0)
            float factor = 1.f;
            bool rescale = false;
            if (mx != -INFINITY) {
                if (l == 0.f) m_ref = mx;                         // nothing accumulated yet
                else if (mx > m_ref + 8.f) { factor = ws_ex2(m_ref - mx); rescale = true; m_ref = mx; }
            }
            // weights P (f16) for the product; the normaliser sums them before rounding
            uint32_t pw[KT / 2];
            float rs = 0.f;
#pragma unroll
            for (int u = 0; u < KT / 2; ++u) {
                const float e0 = ws_ex2(fmaf(sv[2 * u], c2, -m_ref)), e1 = ws_ex2(fmaf(sv[2 * u + 1], c2, -m_ref));
                pw[u] = ws_pack_f16(e0, e1);
                rs += e0 + e1;
            }
            // P(j) over S(j): the tensor cores finished P V (j - 2), which read this buffer,
            // before S(j), whose scores were just read
            {
                const uint32_t pcol = tmem + lane_off + Sh::TS + (2 * t + (j & 1)) * KT;
#pragma unroll
                for (int c0 = 0; c0 < KT / 2; c0 += 16)
                    umma::tmem_st16(pcol + c0, *reinterpret_cast<const float(*)[16]>(pw + c0));
            }
            // P V (j - 1) complete: O may be rescaled, and the MMA thread has taken the previous
            // phase of this tile's P barrier (arriving again before that would alias its parity)
            ok = true;
            if (j >= 1) ok = ws_wait(&mbar[kPvDone + t], (j - 1) & 1, abort_flag);
            dead |= !__all_sync(0xffffffffu, ok);
            if (dead) break;
            umma::fence_after_sync();
            if (__any_sync(0xffffffffu, rescale)) {               // warp-collective TMEM access
                l *= factor;
#pragma unroll
                for (int c0 = 0; c0 < DIM; c0 += 64) {
                    float r64[64];
                    ws_tmem_ld<64>(tmem + lane_off + Sh::TO + t * Sh::OT + c0, r64);
#pragma unroll
                    for (int i = 0; i < 64; ++i) r64[i] *= factor;
#pragma unroll
                    for (int i = 0; i < 64; i += 16)
                        umma::tmem_st16(tmem + lane_off + Sh::TO + t * Sh::OT + c0 + i, *reinterpret_cast<float(*)[16]>(r64 + i));
                }
                umma::tmem_wait_st();
            }
            if (t == 0) {
                // V of this stage (bf16; landed before S(j) was issued, the wait only makes that
                // visible to these threads) to f16 in place, 16-byte chunks spread over the
                // tile's threads; P V (j) waits for this barrier
                ok = ws_wait(&mbar[kKvFull + j % NST], (j / NST) & 1, abort_flag);
                dead |= !__all_sync(0xffffffffu, ok);
                if (dead) break;
                constexpr int NCV = KT * DIM / 8;                 // 16-byte chunks of the V tile
                uint8_t* sV = sKV + (j % NST) * 2 * Sh::KVB + Sh::KVB;
#pragma unroll
                for (int u = 0; u < NCV / ROWS; ++u) {
                    uint4* pv = reinterpret_cast<uint4*>(sV + (u * ROWS + r) * 16);
                    const uint4 x = *pv;
                    *pv = make_uint4(ws_bf2_to_h2(x.x), ws_bf2_to_h2(x.y), ws_bf2_to_h2(x.z), ws_bf2_to_h2(x.w));
                }
                umma::fence_async_smem();
            }
            umma::tmem_wait_st();
            l += rs;
            umma::fence_before_sync();
            umma::mbar_arrive(&mbar[kPFull + t]);
        }
        // ---- epilogue: y = O / l, staged in the (now free) K/V ring so that whole rows of y
        // go out in single store instructions ----
        bool ok = !dead && ntiles > 0;
        if (ok) ok = ws_wait(&mbar[kPvDone + t], (ntiles - 1) & 1, abort_flag);
        if (ok && twoB) ok = ws_wait(&mbar[kPvDone + 1 - t], (ntiles - 1) & 1, abort_flag);   // ring unread
        dead |= !__all_sync(0xffffffffu, ok);
        umma::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        constexpr int RS = DIM * 4 + 16;                          // padded row: conflict-free staging
        static_assert(2 * ROWS * RS <= NST * 2 * Sh::KVB, "staging fits in the ring");
        uint8_t* srow = sKV + (t * ROWS + r) * RS;
#pragma unroll
        for (int c0 = 0; c0 < DIM; c0 += 64) {
            float r64[64];
            ws_tmem_ld<64>(tmem + lane_off + Sh::TO + t * Sh::OT + c0, r64);
#pragma unroll
            for (int i = 0; i < 64; i += 4)
                ws_st4(srow + (c0 + i) * 4, __float_as_uint(r64[i] * inv), __float_as_uint(r64[i + 1] * inv),
                       __float_as_uint(r64[i + 2] * inv), __float_as_uint(r64[i + 3] * inv));
        }
        const int NR = (twoB ? 2 : 1) * ROWS;                     // rows of this CTA's epilogue threads
        umma::named_sync(1, NR);
        constexpr int F4 = DIM / 4;                               // 16-byte pieces of a row
        for (int idx = tid; idx < NR * F4; idx += NR) {
            const int row = idx / F4, c4 = idx % F4, Rr = rfirst + row;
            if (Rr < rows_total && !dead) {
                const int hr = Rr / dm.C, ir = Rr % dm.C;
                float* dst = a.y + (((size_t)b * a.T + (t0 + ir - a.t_start)) * dm.Hq + g * dm.Gq + hr) * DIM + 4 * c4;
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(sKV + row * RS + 16 * c4);
            }
        }
    }
    umma::cp_async_wait<0>();
    umma::fence_before_sync();
    __syncthreads();
    if (tid == 0 && *abort_flag && a.err) atomicOr(a.err, 1);
    if (warp == 0) umma::tmem_dealloc(tmem, Sh::TMEM_COLS);
}

template <int DIM, int DH>
static cudaError_t launch_ws_t(const PrefillArgs& a, cudaStream_t s) {
    using Sh = WsShape<DIM, DH>;
    const int bytes = Sh::END + 1024;                                  // + alignment slack
    if (bytes > 227 * 1024) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(output_ws_kernel<DIM, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    const int nrp = (a.dm.Gq * a.dm.C + Sh::NTILE * Sh::ROWS - 1) / (Sh::NTILE * Sh::ROWS);
    dim3 grid((a.c_end - a.c_begin) * nrp, a.dm.Hkv, a.dm.B);
    output_ws_kernel<DIM, DH><<<grid, Sh::NT, bytes, s>>>(a);
    return cudaGetLastError();
}

// bf16 inputs on the warp-specialised kernel; cudaErrorNotSupported for other shapes.
cudaError_t launch_output_ws(const PrefillArgs& a, cudaStream_t s) {
    const int d = a.dm.d, Dh = a.dm.Dh;
    if (a.dm.dtype != 1) return cudaErrorNotSupported;
    if (d == 128 && Dh == 64) return launch_ws_t<128, 64>(a, s);
    if (d == 128 && Dh == 32) return launch_ws_t<128, 32>(a, s);
    if (d == 64 && Dh == 32) return launch_ws_t<64, 32>(a, s);
    if (d == 64 && Dh == 64) return launch_ws_t<64, 64>(a, s);
    return cudaErrorNotSupported;
}

}  // namespace lola

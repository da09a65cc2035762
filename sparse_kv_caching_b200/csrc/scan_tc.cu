// The per-stream memory-update chain of chunkwise LoLA prefill on the
// fifth-generation tensor cores.
//
// LoLA notes §2.6 (Eq. 15, Fig. 2): after each block the pairs leaving the
// window and the cache members are scored by Self-Recall Error against the
// state (§2.3, Eq. 10), the lambda highest stay in the cache and the rest are
// folded into (H, s) (§2.4, Eqs. 11-13).  Blocks of one stream run in order;
// streams are independent.  Like scan.cu, the chain publishes the memories
// entering every block of the call (cache positions by slot, H_c^T, s_c) for
// the output kernel.
//
// Layout of the work (one stream per CTA, or per cluster of NCL CTAs that
// split the candidates of every block between them):
//   * H^T lives in tensor memory for the whole launch: lane c holds column c
//     of H (rows c >= d are zero), one f32 per TMEM column j < D.  Beside it
//     the launch keeps H_hi = H rounded down to tf32 and H_lo = H - H_hi.
//   * SRE, warp-specialised: a loader warp copies each tile's phi rows (three
//     tiles ahead), the compute warps split them and hand the tile to an
//     issuing warp, then take the scores of the previous tile while its
//     products run (named barriers among the compute warps, mbarriers between
//     the roles).
//     For a tile of 64 candidates, P^T = H^T Phi^T is three tf32 MMAs
//     with A = H_hi / H_lo read from tensor memory and B = Phi_hi / Phi_lo
//     (the candidates' phi rows as loaded, which the tensor cores read to tf32,
//     and their remainders) in shared memory, in the
//     128-byte swizzled layout (each 128-byte piece of a phi row is one
//     shared-memory row, so a warp's copies touch few lines and rows):
//     P = H_hi Phi_hi + H_lo Phi_hi + H_hi Phi_lo, f32-accurate products
//     (the dropped H_lo Phi_lo term is 2^-22 relative) with f32 accumulation.
//     The epilogue reads P^T back (lane c, column e), divides by den_e =
//     phi_e . s (f32 FMAs on the CUDA cores), subtracts v_e[c], squares and
//     sums over c across lanes and warps: score_e = || P_e / den_e - v_e ||^2
//     (the zero prediction while den_e = 0).
//   * Select: the exact radix top-lambda of chain_common.cuh, by the whole CTA.
//   * Fold: H^T += V_S^T Phi_S as bf16 MMAs (kind::f16, f32 accumulation)
//     straight into the tensor-memory H^T: V is split into bf16 parts (one
//     part, exact, for bf16 inputs; three for f32), Phi_S into three bf16
//     parts (8 + 8 + 8 mantissa bits), and the products down to 2^-24
//     relative are issued.  s += sum of Phi_S rows on the CUDA cores.
// Every wait on the tensor cores is bounded; a wait that gives up sets the
// error word, and the launch stops issuing tensor-core work and finishes
// without valid results.
#include <cooperative_groups.h>

#include "chain_common.cuh"
#include "device_common.cuh"
#include "umma.cuh"

namespace lola {

constexpr int kTcCompute = 256;  // warps 0-7: loads, tf32 split, epilogue, selection, fold
constexpr int kTcMmaWarp = 8;    // warp 8: issues the SRE products
constexpr int kTcLoadWarp = 9;   // warp 9: copies the SRE tiles' phi rows
constexpr int kTcThreads = kTcCompute + 64;
constexpr uint32_t kTcComputeBar = 1;   // named barrier of the compute warps
constexpr int kTcTN = 64;        // candidates per SRE tile (N of the SRE product)
constexpr int kTcFK = 64;        // folded pairs per fold product (K), f32 inputs
constexpr int kTcFKB = 128;      // the same for bf16 inputs (one product per block at C <= 128)
constexpr int kTcMinSmem = 170 * 1024;   // one chain CTA per SM: its tensor memory is not shared

struct TcOffsets {               // byte offsets in dynamic shared memory
    int raw, lo, dpart, inv, vptr;   // SRE ring: raw[3] phi tiles, lo[2], den partials[3], 1/den[3], value rows[4]
    int fa, fb, fphi, fv, fpsum, fptr;   // fold operands, staged rows, column partial sums, row addresses
                                         // (alias the SRE ring)
    int score, xsc, cand_pos, keep, eq_list, fold_e, flags, ranks, slot_pos, free_slots, hist, tmp, part, ss, mbar,
        tptr;
    int total;
};

__host__ __device__ inline TcOffsets tc_offsets(int D, int DV, int esize, int lam, int C, int ncl) {
    constexpr int TN = kTcTN, FK = kTcFK;
    TcOffsets o;
    int p = 0;
    auto take = [&](int n, int al) { p = (p + al - 1) / al * al; const int r = p; p += n; return r; };
    o.raw = take(3 * TN * D * 4, 1024);        // 128-byte swizzled tiles: 1024-byte aligned
    o.lo = take(2 * TN * D * 4, 1024);
    const int ring = p;
    // fold: A = value parts [AP][128 / 8 chunks][FK rows][16 B], B = phi parts [3][D / 8][FK][16 B];
    // f32 inputs stage the folded rows as loaded (phi [FK][D] f32, values [FK][DV]); bf16 inputs
    // copy the values straight into A and split phi from global memory, keeping per row range
    // column sums of phi [256 / (D / 8)][D] f32
    p = 0;
    if (esize == 4) {
        o.fa = take(3 * FK * 128 * 2, 128);
        o.fb = take(3 * FK * D * 2, 128);
        o.fphi = take(FK * D * 4, 128);
        o.fv = take(FK * DV * esize, 128);
        o.fpsum = o.fptr = 0;
    } else {
        o.fa = take(kTcFKB * 128 * 2, 1024);          // 128-byte swizzled operands
        o.fb = take(3 * kTcFKB * D * 2, 1024);
        o.fphi = o.fv = 0;
        o.fpsum = take(8 * 256 * 4, 16);
        o.fptr = take(2 * kTcFKB * 8, 16);            // phi and value row addresses of the folded rows
    }
    p = ring > p ? ring : p;
    o.dpart = take(3 * 4 * TN * 4, 16);
    o.inv = take(3 * TN * 4, 16);
    o.vptr = take(4 * TN * 8, 16);
    const int NM = ((lam + C) + 3) & ~3;
    o.score = take(NM * 4, 16);
    o.xsc = take(ncl > 1 ? 2 * NM * 4 : 0, 16);
    o.cand_pos = take(NM * 4, 16);
    o.keep = take(NM * 4, 16);
    o.eq_list = take(NM * 4, 16);
    o.fold_e = take(NM * 4, 16);
    o.flags = take(NM * 4, 16);
    o.ranks = take(NM * 4, 16);
    o.slot_pos = take((lam + 1) * 4, 16);
    o.free_slots = take((lam + 1) * 4, 16);
    o.hist = take(256 * 4, 16);
    o.tmp = take(32 * 4, 16);
    o.part = take(4 * TN * 4, 16);
    o.ss = take(D * 4, 16);
    o.mbar = take(16 * 8, 8);
    o.tptr = take(16, 16);
    o.total = p;
    return o;
}

// x = b0 + b1 + b2 with bf16 parts, each the top 16 bits of what is left (the
// last rounded to nearest): exact to 2^-24 relative for normal x.
__device__ __forceinline__ void split3_bf16(float x, uint16_t& b0, uint16_t& b1, uint16_t& b2) {
    const uint32_t u0 = __float_as_uint(x) & 0xFFFF0000u;
    const float r1 = x - __uint_as_float(u0);
    const uint32_t u1 = __float_as_uint(r1) & 0xFFFF0000u;
    const float r2 = r1 - __uint_as_float(u1);
    b0 = (uint16_t)(u0 >> 16);
    b1 = (uint16_t)(u1 >> 16);
    const __nv_bfloat16 h2 = __float2bfloat16_rn(r2);
    b2 = *reinterpret_cast<const uint16_t*>(&h2);
}

__device__ __forceinline__ void st_shared_zero16(void* p) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" :: "r"(umma::smem_addr(p)), "r"(0u) : "memory");
}

template <int D, int DV, int NCL, typename TIn>
__global__ void __launch_bounds__(kTcThreads, 1) scan_tc_kernel(const __grid_constant__ PrefillArgs a) {
    namespace cg = cooperative_groups;
    constexpr int NT = kTcThreads, TN = kTcTN, FK = kTcFK, M = 128;
    constexpr int ES = (int)sizeof(TIn);
    constexpr bool F32IN = ES == 4;
    constexpr uint32_t TCOLS = 512;
    // tensor-memory columns: H^T (f32 accumulator), H_hi, H_lo, two P^T tiles
    constexpr uint32_t cH = 0, cHhi = D, cHlo = 2 * D, cP = 3 * D;
    static_assert(3 * D + 2 * TN <= (int)TCOLS, "tensor memory");
    static_assert(DV % 32 == 0 && DV <= M && D % 16 == 0, "shape");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzle atoms want 1024-byte aligned tiles (the launch adds the slack)
    uint8_t* smem = smem_raw + ((1024u - (umma::smem_addr(smem_raw) & 1023u)) & 1023u);
    const Dims& dm = a.dm;
    const int lam = dm.lam, C = dm.C, eta = dm.eta;
    int rank = 0;
    if constexpr (NCL > 1) rank = (int)cg::this_cluster().block_rank();
    const int st = blockIdx.x / NCL, b = st / dm.Hkv, g = st % dm.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, half = warp >> 2;          // TMEM lane quarter; column half
    const int crow = 32 * quarter + lane;                    // this thread's H column / TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const TcOffsets o = tc_offsets(D, DV, ES, lam, C, NCL);
    const int NM = ((lam + C) + 3) & ~3;
    float* score = reinterpret_cast<float*>(smem + o.score);
    float* xsc = reinterpret_cast<float*>(smem + o.xsc);
    int* cand_pos = reinterpret_cast<int*>(smem + o.cand_pos);
    int* keep = reinterpret_cast<int*>(smem + o.keep);
    int* eq_list = reinterpret_cast<int*>(smem + o.eq_list);
    int* fold_e = reinterpret_cast<int*>(smem + o.fold_e);
    int* flags = reinterpret_cast<int*>(smem + o.flags);
    int* ranks = reinterpret_cast<int*>(smem + o.ranks);
    int* slot_pos = reinterpret_cast<int*>(smem + o.slot_pos);
    int* free_slots = reinterpret_cast<int*>(smem + o.free_slots);
    unsigned* hist = reinterpret_cast<unsigned*>(smem + o.hist);
    int* tmp = reinterpret_cast<int*>(smem + o.tmp);
    float* part = reinterpret_cast<float*>(smem + o.part);
    float* ss = reinterpret_cast<float*>(smem + o.ss);
    // [0], [1]: SRE products of tiles i % 2 done; [2]: fold products done; [3], [4]: tile i % 2
    // split and ready for its products; [5 + i % 3]: tile i's phi rows and value pointers in;
    // [8 + i % 3]: tile i's products done (its raw buffer free again)
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + o.mbar);
    uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + o.tptr);

    if (warp == 0) umma::tmem_alloc(tptr, TCOLS);
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) umma::mbar_init(&mbar[i], 1);
        for (int i = 5; i < 8; ++i) umma::mbar_init(&mbar[i], 33);   // 32 copy arrivals + the pointers
        for (int i = 8; i < 11; ++i) umma::mbar_init(&mbar[i], 1);
        umma::fence_mbar_init();
    }
    const size_t snaps = (size_t)dm.nc_max + 1;
    {
        const float* s_in = a.c_begin == 0 ? a.sp.s + (size_t)st * D : a.snap_s + ((size_t)st * snaps + a.c_begin) * D;
        for (int i = tid; i < D; i += NT) ss[i] = s_in[i];
        const int* slots_in = entering_slots(a, st);
        for (int j = tid; j < lam; j += NT) slot_pos[j] = slots_in[j];
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tptr;
    uint32_t phases = 0u;                                     // bit i: parity of mbar[i] (barriers this thread waits on)
    bool failed = false;                                      // uniform across the CTA
    const bool compute = warp < kTcCompute / 32;

    // H^T entering the launch into tensor memory (and its tf32 split); warp half
    // h covers columns j in [h D/2, (h+1) D/2)
    if (compute) {
        const float* Hrow = a.sp.H + (size_t)st * D * DV;                              // [D][DV]
        const float* Hsnap = a.snap_H + ((size_t)st * snaps + a.c_begin) * D * DV;      // [DV][D]
        for (int j0 = half * (D / 2); j0 < (half + 1) * (D / 2); j0 += 16) {
            float x[16], hi[16], lo[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int j = j0 + u;
                x[u] = crow >= DV ? 0.f : (a.c_begin == 0 ? Hrow[(size_t)j * DV + crow] : Hsnap[(size_t)crow * D + j]);
                hi[u] = umma::tf32_hi(x[u]);
                lo[u] = x[u] - hi[u];
            }
            umma::tmem_st16(tmem + lane_off + cH + j0, x);
            umma::tmem_st16(tmem + lane_off + cHhi + j0, hi);
            umma::tmem_st16(tmem + lane_off + cHlo + j0, lo);
        }
        umma::tmem_wait_st();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();

    // H_{c}^T, slot positions and s_c into the snapshots of block c (rows of H^T and
    // slot ranges split over the cluster, s by rank 0)
    // (rows of H_c^T go out whole: staged in the SRE ring, which is free between blocks,
    // with a padded row so that the staging stores do not collide)
    auto publish = [&](int c) {
        float* sH = a.snap_H + ((size_t)st * snaps + c) * D * DV;
        constexpr int RSB = D * 4 + 16;
        uint8_t* stage = smem + o.raw;
        if (compute && crow < DV) {
            float x[D / 2];
#pragma unroll
            for (int j0 = 0; j0 < D / 2; j0 += 16)
                umma::tmem_ld16(tmem + lane_off + cH + half * (D / 2) + j0, *reinterpret_cast<float(*)[16]>(x + j0));
            umma::tmem_wait_ld();
            uint8_t* row = stage + crow * RSB + half * (D / 2) * 4;
#pragma unroll
            for (int u = 0; u < D / 8; ++u)
                *reinterpret_cast<float4*>(row + 16 * u) = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
        }
        __syncthreads();
        {
            // this CTA's share of the rows (split over the cluster), one 16-byte piece per thread
            constexpr int F4 = D / 4, NR = DV / NCL;
            const int r0 = rank * NR;
            for (int idx = tid; idx < NR * F4; idx += NT) {
                const int rr = r0 + idx / F4, c4 = idx % F4;
                *reinterpret_cast<float4*>(sH + (size_t)rr * D + 4 * c4) =
                    *reinterpret_cast<const float4*>(stage + rr * RSB + 16 * c4);
            }
        }
        int* sp_ = a.snap_pos + ((size_t)st * snaps + c) * lam;
        for (int j = rank * NT + tid; j < lam; j += NCL * NT) sp_[j] = slot_pos[j];
        if (rank == 0) {
            float* sS = a.snap_s + ((size_t)st * snaps + c) * D;
            for (int i = tid; i < D; i += NT) sS[i] = ss[i];
        }
    };
    if (a.c_begin == 0) publish(0);

    // bounded wait on a tensor-core completion; the outcome is made uniform across the CTA
    auto wait_mma = [&](int i) {
        bool ok = true;
        if (!failed) ok = umma::mbar_wait(&mbar[i], (phases >> i) & 1u);
        phases ^= 1u << i;
        umma::fence_after_sync();
        if (__syncthreads_or(!ok ? 1 : 0)) {
            if (!failed && a.err && tid == 0) atomicOr(a.err, 1);
            failed = true;
        }
    };

    // the same among the compute warps only (during the SRE, while the issuing warp runs its loop)
    auto wait_mma_c = [&](int i) {
        bool ok = true;
        if (!failed) ok = umma::mbar_wait(&mbar[i], (phases >> i) & 1u);
        phases ^= 1u << i;
        umma::fence_after_sync();
        if (umma::named_sync_or(kTcComputeBar, kTcCompute, !ok)) {
            if (!failed && a.err && tid == 0) atomicOr(a.err, 1);
            failed = true;
        }
    };

    // ---- SRE of the candidates of one block -------------------------------------
    // Ring of three raw phi tiles (the tile's rows, K-major B operand, 128-byte swizzled:
    // the 16-byte chunk jc of row r, jc = 8 kb + c, at kb (TN 128) + 128 r + 16 (c ^ r % 8)),
    // two tf32-low tiles in the same layout, and per tile the partial and final 1/den and
    // the value-row pointers (four slots).  Loads run two tiles ahead.
    float* dpart = reinterpret_cast<float*>(smem + o.dpart);
    float* invd = reinterpret_cast<float*>(smem + o.inv);
    const TIn** vptr = reinterpret_cast<const TIn**>(smem + o.vptr);
    auto raw_tile = [&](int s3) { return smem + o.raw + s3 * (TN * D * 4); };
    auto lo_tile = [&](int lb) { return smem + o.lo + lb * (TN * D * 4); };
    // The loader warp: the phi rows of tile t (slot i of this CTA's tiles) into raw[i % 3]
    // (rows past n zero-filled), the value-row pointers into vptr[i % 4] (rows past n: the
    // value row of candidate 0, a valid address, so that the value loads need no test; those
    // scores are never stored).  Lane l looks up rows l and l + 32; eight lanes copy each
    // 128-byte piece of a row (one global line, one shared row).  Every lane's copies arrive
    // on mbar[5 + i % 3] as they land, lane 0 once more after the pointers.
    auto load_tile = [&](int t, int i, int n) {
        uint8_t* base = raw_tile(i % 3);
        const int e0 = t * TN + lane, e1 = e0 + 32;
        const PairRef<TIn> p0 = pair_ref<TIn>(a, st, b, g, cand_pos[e0 < n ? e0 : 0], e0 < n ? e0 : 0);
        const PairRef<TIn> p1 = pair_ref<TIn>(a, st, b, g, cand_pos[e1 < n ? e1 : 0], e1 < n ? e1 : 0);
        const unsigned long long s0 = e0 < n ? reinterpret_cast<unsigned long long>(p0.phik) : 0ull;
        const unsigned long long s1 = e1 < n ? reinterpret_cast<unsigned long long>(p1.phik) : 0ull;
        vptr[(i % 4) * TN + lane] = p0.v;
        vptr[(i % 4) * TN + 32 + lane] = p1.v;
        const int c = lane & 7;
        const float* dummy = a.sp.H;                          // placeholder source of zero fills
#pragma unroll 4
        for (int rg = 0; rg < TN / 4; ++rg) {
            const int row = 4 * rg + (lane >> 3);
            const unsigned long long p = __shfl_sync(0xffffffffu, rg < 8 ? s0 : s1, row & 31);
#pragma unroll
            for (int kb = 0; kb < D / 32; ++kb) {
                uint8_t* dst = base + kb * (TN * 128) + umma::sw128_off(row, c);
                umma::cp_async16_zfill(dst, p != 0ull ? reinterpret_cast<const float*>(p) + 32 * kb + 4 * c : dummy,
                                       p != 0ull);
            }
        }
        umma::cp_async_arrive_noinc(&mbar[5 + i % 3]);
        __syncwarp();
        if (lane == 0) umma::mbar_arrive(&mbar[5 + i % 3]);
    };
    // the compute warps' wait for tile i's rows (uniform outcome among them)
    auto wait_landed = [&](int i) {
        const int lb = 5 + i % 3;
        bool ok = true;
        if (!failed) ok = umma::mbar_wait(&mbar[lb], (phases >> lb) & 1u);
        phases ^= 1u << lb;
        if (umma::named_sync_or(kTcComputeBar, kTcCompute, !ok)) {
            if (!failed && a.err && tid == 0) atomicOr(a.err, 1);
            failed = true;
        }
    };
    // tf32 split: the raw tile in raw[i % 3] serves as Phi_hi as it is (kind::tf32 reads the
    // top 19 bits of each f32), Phi_lo = phi - hi goes to lo[i % 2]; partial den_e = phi_e . s
    // over a quarter of the chunks (thread (r, q): chunks q, q+4, ...)
    auto prep = [&](int i) {
        float* phi = reinterpret_cast<float*>(raw_tile(i % 3));
        float* plo = reinterpret_cast<float*>(lo_tile(i & 1));
        float* dp = dpart + (i % 3) * 4 * TN;
        const int r = tid % TN, q = tid / TN;
        float d0 = 0.f, d1 = 0.f;
        for (int jc = q; jc < D / 4; jc += kTcCompute / TN) {
            const int off = ((jc >> 3) * (TN * 128) + (int)umma::sw128_off(r, jc & 7)) / 4;
            const float4 x = *reinterpret_cast<const float4*>(phi + off);
            const float4 s4 = *reinterpret_cast<const float4*>(ss + 4 * jc);
            d0 = fmaf(x.x, s4.x, d0); d1 = fmaf(x.y, s4.y, d1);
            d0 = fmaf(x.z, s4.z, d0); d1 = fmaf(x.w, s4.w, d1);
            const float4 h = make_float4(umma::tf32_hi(x.x), umma::tf32_hi(x.y), umma::tf32_hi(x.z), umma::tf32_hi(x.w));
            *reinterpret_cast<float4*>(plo + off) = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
        }
        dp[q * TN + r] = d0 + d1;
    };
    // 1 / den_e of slot i (0 while den_e = 0: the empty memory recalls zero)
    auto den_final = [&](int i) {
        const float* dp = dpart + (i % 3) * 4 * TN;
        if (tid < TN) {
            const float dn = (dp[tid] + dp[TN + tid]) + (dp[2 * TN + tid] + dp[3 * TN + tid]);
            invd[(i % 3) * TN + tid] = dn > 0.f ? 1.f / dn : 0.f;
        }
    };
    auto issue_sre_mma = [&](int i) {                        // lane 0 of the issuing warp
        const int pb = i & 1;
        const uint32_t id = umma::idesc(umma::kTF32, M, TN, false, false);
        const uint64_t bh0 = umma::sdesc_sw128(umma::smem_addr(raw_tile(i % 3)), 16, 1024);
        const uint64_t bl0 = umma::sdesc_sw128(umma::smem_addr(lo_tile(i & 1)), 16, 1024);
        const uint32_t dP = tmem + cP + pb * TN;
        // a K step of 8 moves the operand start by 32 bytes inside a 128-byte row piece, the
        // next piece TN rows further (the descriptor's address field counts 16-byte units)
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks) {
            const uint64_t step = (uint64_t)((ks >> 2) * (TN * 8) + (ks & 3) * 2);
            umma::mma_tf32_ts(dP, tmem + cHhi + ks * 8, bh0 + step, id, ks > 0 ? 1u : 0u);
            umma::mma_tf32_ts(dP, tmem + cHlo + ks * 8, bh0 + step, id, 1u);
            umma::mma_tf32_ts(dP, tmem + cHhi + ks * 8, bl0 + step, id, 1u);
        }
        umma::commit(&mbar[pb]);
        umma::commit(&mbar[8 + i % 3]);
    };
    // score_e of tile t (slot i) -> out[e]: squared residual over this quarter's 32
    // columns (values v from registers, loaded before the MMA wait), summed across the
    // lanes (each lane ends with one candidate) and across the quarters
    auto epilogue = [&](int t, int i, int n, float* out, const TIn (&v)[32]) {
        const float* inv = invd + (i % 3) * TN;
        if (32 * quarter < DV) {
            float x[32];
            const uint32_t col = tmem + lane_off + cP + (i & 1) * TN + 32 * half;
            umma::tmem_ld16(col, *reinterpret_cast<float(*)[16]>(x));
            umma::tmem_ld16(col + 16, *reinterpret_cast<float(*)[16]>(x + 16));
            umma::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float r = x[k] * inv[32 * half + k] - to_f32(v[k]);
                x[k] = r * r;
            }
            // transpose-reduce: after the step with offset o every lane keeps half of its
            // values (the half selected by its lane bit o) plus its partner's
#pragma unroll
            for (int off = 16, w = 16; off >= 1; off >>= 1, w >>= 1) {
                const bool up = (lane & off) != 0;
#pragma unroll
                for (int k = 0; k < w; ++k) {
                    const float send = up ? x[k] : x[k + w];
                    const float keepv = up ? x[k + w] : x[k];
                    x[k] = keepv + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            part[quarter * TN + 32 * half + lane] = x[0];
        }
        umma::named_sync(kTcComputeBar, kTcCompute);
        if (tid < TN) {
            const int e = t * TN + tid;
            if (e < n) {
                float sc = part[tid];
#pragma unroll
                for (int q = 1; q < DV / 32; ++q) sc += part[q * TN + tid];
                out[e] = sc;
            }
        }
    };
    int xb = 0;                                               // exchange buffer parity (clusters)
    auto sre_block = [&](int n) {
        const int nt = (n + TN - 1) / TN;
        const int mt = nt > rank ? (nt - rank + NCL - 1) / NCL : 0;    // tiles rank, rank + NCL, ...
        float* out = NCL > 1 ? xsc + xb * NM : score;
        auto tile_of = [&](int i) { return i < mt ? rank + i * NCL : -1; };
        if (mt > 0 && compute) {
            wait_landed(0);
            // split tile i and hand it to the issuing warp (mbar[3 + i % 2])
            auto prep_and_pass = [&](int i) {
                prep(i);
                umma::fence_async_smem();
                umma::fence_before_sync();
                umma::named_sync(kTcComputeBar, kTcCompute);
                if (tid == 0) umma::mbar_arrive(&mbar[3 + (i & 1)]);
            };
            prep_and_pass(0);
            den_final(0);
            // this thread's values (column crow of its 32 candidates) of a tile, loaded one
            // tile ahead of the epilogue that needs them
            auto load_values = [&](int i, TIn (&v)[32]) {
                const TIn* const* vp = vptr + (i % 4) * TN + 32 * half;
                if (32 * quarter < DV) {                      // warp-uniform
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = vp[k][crow];
                }
            };
            TIn vcur[32], vnext[32];
            load_values(0, vcur);
            for (int i = 0; i < mt; ++i) {
                const int t = tile_of(i);
                if (i + 1 < mt) {
                    wait_landed(i + 1);
                    // lo[(i + 1) % 2] was last read by the products of tile i - 1, waited for
                    prep_and_pass(i + 1);
                    den_final(i + 1);
                    load_values(i + 1, vnext);
                }
                wait_mma_c(i & 1);                            // tile i's products
                epilogue(t, i, n, out, vcur);
                umma::fence_before_sync();
#pragma unroll
                for (int k = 0; k < 32; ++k) vcur[k] = vnext[k];
            }
            umma::named_sync(kTcComputeBar, kTcCompute);
        } else if (mt > 0 && warp == kTcMmaWarp) {
            // the issuing warp: tile i's products once the compute warps have split it; the
            // ready barriers alternate, so a compute warp signalling tile i + 2 has already
            // waited for the products of tile i, issued after this warp saw tile i ready
            for (int i = 0; i < mt; ++i) {
                const int rb = 3 + (i & 1);
                bool ok = true;
                if (lane == 0 && !failed) ok = umma::mbar_wait(&mbar[rb], (phases >> rb) & 1u);
                phases ^= 1u << rb;
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) failed = true;                       // made uniform after the block
                umma::fence_after_sync();
                if (lane == 0 && !failed) issue_sre_mma(i);
                __syncwarp();
            }
        } else if (mt > 0 && warp == kTcLoadWarp) {
            // tile i's rows once the products of tile i - 3 (same raw buffer) are done; every
            // tile's completion is waited for once, the last three after the last copy
            for (int i = 0; i < mt + 3; ++i) {
                if (i >= 3) {
                    const int fb = 8 + (i - 3) % 3;
                    bool ok = true;
                    if (lane == 0 && !failed) ok = umma::mbar_wait(&mbar[fb], (phases >> fb) & 1u);
                    phases ^= 1u << fb;
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) failed = true;                   // made uniform after the block
                }
                if (i < mt) load_tile(tile_of(i), i, n);
            }
        }
        if (__syncthreads_or(failed ? 1 : 0)) {
            if (!failed && a.err && tid == 0) atomicOr(a.err, 1);
            failed = true;
        }
        if constexpr (NCL > 1) {
            cg::cluster_group cluster = cg::this_cluster();
            cluster.sync();                                   // every CTA's tile scores are written
            for (int e = tid; e < n; e += NT) {
                const int owner = (e / TN) % NCL;
                score[e] = *cluster.map_shared_rank(xsc + xb * NM + e, owner);
            }
            xb ^= 1;
        }
        umma::cp_async_wait<0>();
        __syncthreads();
    };

    // ---- fold: H^T += V_S^T Phi_S, s += sum Phi_S ---------------------------------
    // The folded rows are staged with cp.async (phi [FK][D] f32, values [FK][DV]), then
    // split into MN-major bf16 operand parts: A part p = value row k, columns c, at
    // (c/8)(FK 16) + 16 k; B part p = phi row k, columns j, at (j/8)(FK 16) + 16 k.
    // bf16 inputs: up to kTcFKB folded pairs per product.  The value rows go straight into
    // the A operand (bf16 is exact: one part); thread (j8, rr) of the compute warps reads
    // columns 8 j8 .. 8 j8 + 7 of rows rr RPT .. rr RPT + RPT - 1 of phi from global memory,
    // splits them into the three B parts and keeps the column sums of its rows; s then adds
    // the row ranges' sums in range order.  Both operands are MN-major and 128-byte swizzled:
    // folded row k of block mb holds its columns 64 mb .. 64 mb + 63 as one 128-byte row.
    auto fold_b16 = [&](int nf) {
        constexpr int FKB = kTcFKB, J8 = D / 8, RR = kTcCompute / J8, RPT = FKB / RR;
        static_assert(RR * J8 == kTcCompute && RPT * RR == FKB, "fold tiling");
        uint8_t* fa = smem + o.fa;
        uint8_t* fb = smem + o.fb;
        float* psum = reinterpret_cast<float*>(smem + o.fpsum);
        // each folded row's phi and value addresses, looked up once
        const float** prow = reinterpret_cast<const float**>(smem + o.fptr);
        const TIn** vrow = reinterpret_cast<const TIn**>(smem + o.fptr + FKB * 8);
        for (int f0 = 0; f0 < nf; f0 += FKB) {
            const int nff = min(FKB, nf - f0), nk = (nff + 15) & ~15;
            for (int k = tid; k < nff; k += NT) {
                const int e = fold_e[f0 + k];
                const PairRef<TIn> pr = pair_ref<TIn>(a, st, b, g, cand_pos[e], e);
                prow[k] = pr.phik;
                vrow[k] = pr.v;
            }
            __syncthreads();
            for (int idx = tid; idx < nk * (M / 8); idx += NT) {
                const int k = idx / (M / 8), c8 = idx % (M / 8);
                uint8_t* dst = fa + (c8 >> 3) * (FKB * 128) + umma::sw128_off(k, c8 & 7);
                if (k < nff && 8 * c8 < DV) {
                    umma::cp_async16(dst, vrow[k] + 8 * c8);
                } else {
                    st_shared_zero16(dst);
                }
            }
            umma::cp_async_commit();
            if (compute) {
                const int j8 = tid % J8, rr = tid / J8;
                // every row's loads in flight before the first split
                float xs[RPT][8];
#pragma unroll
                for (int u = 0; u < RPT; ++u) {
                    const int k = rr * RPT + u;
                    if (k < nff) {
                        const float* src = prow[k] + 8 * j8;
                        const float4 xa = *reinterpret_cast<const float4*>(src);
                        const float4 xb4 = *reinterpret_cast<const float4*>(src + 4);
                        xs[u][0] = xa.x; xs[u][1] = xa.y; xs[u][2] = xa.z; xs[u][3] = xa.w;
                        xs[u][4] = xb4.x; xs[u][5] = xb4.y; xs[u][6] = xb4.z; xs[u][7] = xb4.w;
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) xs[u][i] = 0.f;
                    }
                }
                float cs[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) cs[i] = 0.f;
#pragma unroll
                for (int u = 0; u < RPT; ++u) {
                    const int k = rr * RPT + u;
                    if (k >= nk) break;
                    // zero rows (k >= nff) split into zero parts
                    uint32_t w0[4], w1[4], w2[4];
#pragma unroll
                    for (int i = 0; i < 8; ++i) cs[i] += xs[u][i];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint16_t p0, p1, p2, q0, q1, q2;
                        split3_bf16(xs[u][2 * q], p0, p1, p2);
                        split3_bf16(xs[u][2 * q + 1], q0, q1, q2);
                        w0[q] = (uint32_t)p0 | ((uint32_t)q0 << 16);
                        w1[q] = (uint32_t)p1 | ((uint32_t)q1 << 16);
                        w2[q] = (uint32_t)p2 | ((uint32_t)q2 << 16);
                    }
                    const int off = (j8 >> 3) * (FKB * 128) + (int)umma::sw128_off(k, j8 & 7);
                    *reinterpret_cast<uint4*>(fb + off) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                    *reinterpret_cast<uint4*>(fb + FKB * D * 2 + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                    *reinterpret_cast<uint4*>(fb + 2 * FKB * D * 2 + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) psum[rr * D + 8 * j8 + i] = cs[i];
            }
            umma::cp_async_wait<0>();
            __syncthreads();
            for (int j = tid; j < D; j += NT) {
                float acc = 0.f;
                for (int q = 0; q < RR; ++q) acc += psum[q * D + j];
                ss[j] += acc;
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncthreads();
            umma::fence_after_sync();
            if (tid == 0 && !failed) {
                const uint32_t id = umma::idesc(umma::kBF16, M, D, true, true);
                const uint32_t A0 = umma::smem_addr(fa), B0 = umma::smem_addr(fb);
                constexpr uint32_t PB = FKB * D * 2;                      // bytes between phi parts
                // MN-major swizzled: lbo = the stride between 64-column blocks, sbo = 8 rows
                const uint64_t a0 = umma::sdesc_sw128(A0, FKB * 128, 1024), b0 = umma::sdesc_sw128(B0, FKB * 128, 1024);
#pragma unroll
                for (int ks = 0; ks < FKB / 16; ++ks) {
                    if (ks * 16 >= nk) break;
                    // a K step of 16 rows moves the start by 2048 bytes; the phi parts are PB bytes apart
                    const uint64_t da = a0 + (uint64_t)((ks * 2048) >> 4);
                    umma::mma_bf16(tmem + cH, da, b0 + (uint64_t)((ks * 2048) >> 4), id, 1u);
                    umma::mma_bf16(tmem + cH, da, b0 + (uint64_t)((PB + ks * 2048) >> 4), id, 1u);
                    umma::mma_bf16(tmem + cH, da, b0 + (uint64_t)((2 * PB + ks * 2048) >> 4), id, 1u);
                }
                umma::commit(&mbar[2]);
            }
            wait_mma(2);                                      // the operands may be overwritten now
        }
    };

    auto fold_f32 = [&](int nf) {
        uint8_t* fa = smem + o.fa;
        uint8_t* fb = smem + o.fb;
        const float* fphi = reinterpret_cast<const float*>(smem + o.fphi);
        const TIn* fv = reinterpret_cast<const TIn*>(smem + o.fv);
        constexpr int AP = F32IN ? 3 : 1;                     // value parts
        constexpr int VP = DV * ES / 16;                      // 16-byte pieces of a value row
        for (int f0 = 0; f0 < nf; f0 += FK) {
            const int nff = min(FK, nf - f0), nk = (nff + 15) & ~15;
            for (int idx = tid; idx < nff * (D / 4); idx += NT) {
                const int k = idx / (D / 4), q = idx % (D / 4), e = fold_e[f0 + k];
                umma::cp_async16(smem + o.fphi + k * (D * 4) + 16 * q, pair_ref<TIn>(a, st, b, g, cand_pos[e], e).phik + 4 * q);
            }
            for (int idx = tid; idx < nff * VP; idx += NT) {
                const int k = idx / VP, q = idx % VP, e = fold_e[f0 + k];
                umma::cp_async16(smem + o.fv + k * (DV * ES) + 16 * q,
                                 reinterpret_cast<const char*>(pair_ref<TIn>(a, st, b, g, cand_pos[e], e).v) + 16 * q);
            }
            umma::cp_async_commit();
            umma::cp_async_wait<0>();
            __syncthreads();
            // phi parts (rows past nff are zero)
            for (int idx = tid; idx < nk * (D / 8); idx += NT) {
                const int k = idx / (D / 8), j8 = idx % (D / 8);
                uint32_t w0[4] = {0u, 0u, 0u, 0u}, w1[4] = {0u, 0u, 0u, 0u}, w2[4] = {0u, 0u, 0u, 0u};
                if (k < nff) {
                    const float4 xa = *reinterpret_cast<const float4*>(fphi + k * D + 8 * j8);
                    const float4 xb4 = *reinterpret_cast<const float4*>(fphi + k * D + 8 * j8 + 4);
                    const float xs[8] = {xa.x, xa.y, xa.z, xa.w, xb4.x, xb4.y, xb4.z, xb4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint16_t p0, p1, p2, q0, q1, q2;
                        split3_bf16(xs[2 * u], p0, p1, p2);
                        split3_bf16(xs[2 * u + 1], q0, q1, q2);
                        w0[u] = (uint32_t)p0 | ((uint32_t)q0 << 16);
                        w1[u] = (uint32_t)p1 | ((uint32_t)q1 << 16);
                        w2[u] = (uint32_t)p2 | ((uint32_t)q2 << 16);
                    }
                }
                const int off = j8 * (FK * 16) + k * 16;
                *reinterpret_cast<uint4*>(fb + off) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                *reinterpret_cast<uint4*>(fb + FK * D * 2 + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                *reinterpret_cast<uint4*>(fb + 2 * FK * D * 2 + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
            }
            // value parts (rows c >= DV and k >= nff stay zero)
            for (int idx = tid; idx < nk * (M / 8); idx += NT) {
                const int k = idx / (M / 8), c8 = idx % (M / 8);
                uint32_t w0[4] = {0u, 0u, 0u, 0u}, w1[4] = {0u, 0u, 0u, 0u}, w2[4] = {0u, 0u, 0u, 0u};
                if (k < nff && 8 * c8 < DV) {
                    const TIn* src = fv + k * DV + 8 * c8;
                    if constexpr (F32IN) {
                        const float4 xa = load4(src), xb4 = load4(src + 4);
                        const float xs[8] = {xa.x, xa.y, xa.z, xa.w, xb4.x, xb4.y, xb4.z, xb4.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            uint16_t p0, p1, p2, q0, q1, q2;
                            split3_bf16(xs[2 * u], p0, p1, p2);
                            split3_bf16(xs[2 * u + 1], q0, q1, q2);
                            w0[u] = (uint32_t)p0 | ((uint32_t)q0 << 16);
                            w1[u] = (uint32_t)p1 | ((uint32_t)q1 << 16);
                            w2[u] = (uint32_t)p2 | ((uint32_t)q2 << 16);
                        }
                    } else {
                        const uint4 raw = *reinterpret_cast<const uint4*>(src);       // 8 bf16: exact
                        w0[0] = raw.x; w0[1] = raw.y; w0[2] = raw.z; w0[3] = raw.w;
                    }
                }
                const int off = c8 * (FK * 16) + k * 16;
                *reinterpret_cast<uint4*>(fa + off) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                if constexpr (F32IN) {
                    *reinterpret_cast<uint4*>(fa + FK * M * 2 + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                    *reinterpret_cast<uint4*>(fa + 2 * FK * M * 2 + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
                }
            }
            // s += sum over the folded rows, column by column in row order (f32 on the CUDA cores)
            for (int j = tid; j < D; j += NT) {
                float acc = 0.f;
                for (int k = 0; k < nff; ++k) acc += fphi[k * D + j];
                ss[j] += acc;
            }
            umma::fence_async_smem();
            umma::fence_before_sync();
            __syncthreads();
            umma::fence_after_sync();
            if (tid == 0 && !failed) {
                const uint32_t id = umma::idesc(umma::kBF16, M, D, true, true);
                const uint32_t A0 = umma::smem_addr(fa), B0 = umma::smem_addr(fb);
                constexpr uint32_t PA = FK * M * 2, PB = FK * D * 2;       // bytes between parts
                const uint64_t a0 = umma::sdesc(A0, 128, FK * 16), b0 = umma::sdesc(B0, 128, FK * 16);
#pragma unroll
                for (int ks = 0; ks < FK / 16; ++ks) {
                    if (ks * 16 >= nk) break;
                    // a K step of 16 moves the start by 256 bytes; parts are PA / PB bytes apart
                    auto da = [&](int p) { return a0 + (uint64_t)((p * PA + ks * 256) >> 4); };
                    auto db = [&](int p) { return b0 + (uint64_t)((p * PB + ks * 256) >> 4); };
                    // products down to 2^-24 relative: a0 b0, a0 b1, a0 b2 (+ a1 b0, a1 b1, a2 b0)
                    umma::mma_bf16(tmem + cH, da(0), db(0), id, 1u);
                    umma::mma_bf16(tmem + cH, da(0), db(1), id, 1u);
                    umma::mma_bf16(tmem + cH, da(0), db(2), id, 1u);
                    if (AP == 3) {
                        umma::mma_bf16(tmem + cH, da(1), db(0), id, 1u);
                        umma::mma_bf16(tmem + cH, da(1), db(1), id, 1u);
                        umma::mma_bf16(tmem + cH, da(2), db(0), id, 1u);
                    }
                }
                umma::commit(&mbar[2]);
            }
            wait_mma(2);                                      // the operands may be overwritten now
        }
    };

    auto fold = [&](int nf) {
        if constexpr (!F32IN) {
            fold_b16(nf);
        } else {
            fold_f32(nf);
        }
        // refresh the tf32 split of H^T
        for (int j0 = half * (D / 2); compute && j0 < (half + 1) * (D / 2); j0 += 16) {
            float x[16], hi[16], lo[16];
            umma::tmem_ld16(tmem + lane_off + cH + j0, x);
            umma::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) { hi[u] = umma::tf32_hi(x[u]); lo[u] = x[u] - hi[u]; }
            umma::tmem_st16(tmem + lane_off + cHhi + j0, hi);
            umma::tmem_st16(tmem + lane_off + cHlo + j0, lo);
        }
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncthreads();
        umma::fence_after_sync();
    };

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
            if (lam > 0 && a.scorer != 0) {
                for (int e = tid; e < n; e += NT) score[e] = static_score(a, st, cand_pos[e], e);
                __syncthreads();
            } else if (lam > 0) {
                sre_block(n);
            }
            const int nf = select_place_cta(score, cand_pos, n, n_g, n_l, lam, l_lo, slot_pos, fold_e, keep,
                                            free_slots, hist, tmp, eq_list, flags, ranks);
            fold(nf);
        }
        __syncthreads();
        publish(c + 1);
        __syncthreads();                                      // the next block may change slot_pos
    }
    // final state: H [D][DV] row-major (coalesced over columns c), s
    {
        float* Ho = a.sp.H + (size_t)st * D * DV;
        const bool mine = crow < DV && (NCL == 1 || crow / (DV / NCL) == rank);
        for (int j0 = half * (D / 2); compute && j0 < (half + 1) * (D / 2); j0 += 16) {
            float x[16];
            umma::tmem_ld16(tmem + lane_off + cH + j0, x);
            umma::tmem_wait_ld();
            if (mine)
#pragma unroll
                for (int u = 0; u < 16; ++u) Ho[(size_t)(j0 + u) * DV + crow] = x[u];
        }
        if (rank == 0)
            for (int i = tid; i < D; i += NT) a.sp.s[(size_t)st * D + i] = ss[i];
    }
    umma::cp_async_wait<0>();
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) umma::tmem_dealloc(tmem, TCOLS);
    if constexpr (NCL > 1) cg::this_cluster().sync();          // peers may still read our scores
}

size_t scan_tc_smem_bytes(const Dims& dm, int ncl) {
    const size_t b = (size_t)tc_offsets(dm.D, dm.d, dm.esize, dm.lam, dm.C, ncl).total + 1024;   // + alignment slack
    return b < (size_t)kTcMinSmem ? (size_t)kTcMinSmem : b;
}

template <int D, int DV, int NCL, typename TIn>
static cudaError_t launch_tc_chain_t(const PrefillArgs& a, cudaStream_t s) {
    const size_t bytes = scan_tc_smem_bytes(a.dm, NCL);
    auto kern = scan_tc_kernel<D, DV, NCL, TIn>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.dm.S * NCL);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NCL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = NCL > 1 ? 1 : 0;
    if (NCL > 1) {
        // every stream's cluster must be resident at once (the CTAs of a cluster wait on each other)
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
        if (e != cudaSuccess || nclusters < a.dm.S) { (void)cudaGetLastError(); return cudaErrorNotSupported; }
    }
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D, int DV, typename TIn>
static cudaError_t launch_tc_chain_n(const PrefillArgs& a, int ncl, cudaStream_t s) {
    switch (ncl) {
        case 1: return launch_tc_chain_t<D, DV, 1, TIn>(a, s);
        case 2: return launch_tc_chain_t<D, DV, 2, TIn>(a, s);
        case 4: return launch_tc_chain_t<D, DV, 4, TIn>(a, s);
    }
    return cudaErrorNotSupported;
}

template <typename TIn>
static cudaError_t launch_tc_chain_d(const PrefillArgs& a, int ncl, cudaStream_t s) {
    const int d = a.dm.d, D = a.dm.D;
    if (d == 128 && D == 128) return launch_tc_chain_n<128, 128, TIn>(a, ncl, s);
    if (d == 128 && D == 64) return launch_tc_chain_n<64, 128, TIn>(a, ncl, s);
    if (d == 64 && D == 128) return launch_tc_chain_n<128, 64, TIn>(a, ncl, s);
    if (d == 64 && D == 64) return launch_tc_chain_n<64, 64, TIn>(a, ncl, s);
    return cudaErrorNotSupported;
}

// Cluster size of the tensor-core chain: the candidates of a block are split
// into tiles of 64 over the cluster; a larger cluster shortens every block but
// takes SMs from the output kernel that runs beside the chain.  Returns 0 when
// the shape is outside what the kernel covers.
int pick_tc_cluster(const Dims& dm, int num_sms) {
    const int tiles = (dm.lam + dm.C + kTcTN - 1) / kTcTN;
    int ncl = 1;
    while (ncl < 4 && 2 * ncl <= tiles && dm.S * 2 * ncl <= num_sms / 2) ncl *= 2;
    for (; ncl >= 1; ncl >>= 1)
        if (scan_tc_smem_bytes(dm, ncl) <= 227 * 1024) return ncl;
    return 0;
}

// The chain on the tensor cores; cudaErrorNotSupported if the shape or the
// cluster residency is outside what it covers (the caller then takes scan.cu's).
cudaError_t launch_scan_tc(const PrefillArgs& a, int num_sms, cudaStream_t s) {
    for (int ncl = pick_tc_cluster(a.dm, num_sms); ncl >= 1; ncl >>= 1) {
        const cudaError_t e = a.dm.dtype == 1 ? launch_tc_chain_d<__nv_bfloat16>(a, ncl, s)
                                              : launch_tc_chain_d<float>(a, ncl, s);
        if (e != cudaErrorNotSupported) return e;
    }
    return cudaErrorNotSupported;
}

}  // namespace lola

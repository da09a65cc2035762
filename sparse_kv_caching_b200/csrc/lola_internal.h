// Internal declarations shared by the LoLA kernels and the C ABI layer.
//
// Memory model of one stream (one sequence b and kv head g, st = b*Hkv + g),
// all inside the caller's device buffer:
//   H [D][d] f32, s [D] f32                        linear state (notes §2.2, Eqs. 3-5)
//   cache slots: k, v [lambda][d] (dtype), phik [lambda][D] f32, pos [lambda] i32
//                                                  sparse global cache G (notes §2.4)
//   window ring: k, v [eta][d] (dtype), phik [eta][D] f32; position p in slot p % eta
//                                                  sliding window W (notes §2.4)
// The window always holds positions [max(0, t - eta), t) and the cache
// occupies slots [0, min(lambda, max(0, t - eta))) at a block boundary t, so
// both are functions of t alone; only the slot contents need storage.
//
// Where a pair of the current prefill call lives (t_start = first position
// of the call): p >= t_start -> the call's input arrays; t_start - eta <= p
// < t_start -> the window ring; p < t_start - eta -> a cache slot that held
// it when the call began (such a member never changes slot while cached).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace lola {

constexpr int kThreads = 512;

struct Layout {            // byte offsets inside dev_buf (all 256-aligned)
    size_t W, H, s, cache_k, cache_v, cache_phik, cache_pos, win_k, win_v, win_phik, cache_R, cache_den, cache_sc,
        win_sc;
    size_t phik_new, key_sc, snap_pos, snap_H, snap_s, io_q, io_k, io_v, io_y, err;
    size_t total;
};

struct Dims {
    int B, Hq, Hkv, Gq, d, Dh, D, eta, lam, C, dtype, S, max_tokens, nc_max;
    int esize;             // bytes per input element
};

// Pointers to the persistent state of all streams.
struct StatePtrs {
    const void* W;
    float* H;
    float* s;
    void* cache_k;
    void* cache_v;
    float* cache_phik;
    int* cache_pos;
    void* win_k;
    void* win_v;
    float* win_phik;
    float* cache_R;        // [S][lambda][d]  H^T phi_e - den_e v_e (kept by decode)
    float* cache_den;      // [S][lambda]     phi_e . s
    float* cache_sc;       // [S][lambda]     each member's score: SRE against the current (H, s),
                           //                 or its frozen window score under an alternative rule
    float* win_sc;         // [S][eta]        window score accumulated so far (alternative rules; ring slot p % eta)
};

struct PrefillArgs {
    Dims dm;
    StatePtrs sp;
    const void* q;         // [B][T][Hq][d]
    const void* k;         // [B][T][Hkv][d]
    const void* v;
    float* y;              // [B][T][Hq][d]
    int T;                 // tokens in this call
    int t_start;           // position of the first token of the call
    int nc;                // chunks in this call
    int c_begin, c_end;    // chunks [c_begin, c_end) of the call served by this launch (scan, output)
    int read_mask;         // bit 0: queries do not read (H, s); bit 1: nor the sparse cache
    int scorer;            // 0 SRE; 1..4 the alternative rules (window scores, see scores.cu)
    float* key_sc;         // [S][eta + max_tokens] window scores of positions t_start - eta + i
    float* phik_new;       // [S][max_tokens][D]
    int* snap_pos;         // [S][nc_max+1][lambda]
    float* snap_H;         // [S][nc_max+1][d][D] (H_c transposed)
    float* snap_s;         // [S][nc_max+1][D]
    int* err;              // device error word (bit 0: a bounded wait gave up)
};

struct DecodeArgs {
    Dims dm;
    StatePtrs sp;
    const void* q;         // [B][Hq][d]
    const void* k;         // [B][Hkv][d]
    const void* v;
    float* y;              // [B][Hq][d]
    int t;                 // position of the new token
    int read_mask;         // as PrefillArgs::read_mask
    int update_first;      // 1: update the memories, then read them (token equations read literally)
    int scorer;            // as PrefillArgs::scorer
    int* err;              // device error word
};

// Stored-pair SRE map of the last prefill call (analysis; reads the snapshots).
struct SreMapArgs {
    Dims dm;
    const void* k;         // [B][T][Hkv][d]  every position of the sequence so far
    const void* v;
    const void* W;         // [Hkv][d][Dh]
    const float* snap_H;   // [S][nc_max+1][d][D] (H_c transposed)
    const float* snap_s;   // [S][nc_max+1][D]
    const int* snap_pos;   // [S][nc_max+1][lambda]
    float* sre;            // [S][nc+1][T]
    float* rel;            // [S][nc+1][T] or null
    int T;                 // positions covered
    int t0;                // first position of the last prefill call
    int nc;                // its chunks
};

// Launchers (each returns cudaGetLastError() of its launch).
cudaError_t launch_phi_keys(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_scan(const PrefillArgs& a, cudaStream_t s);
// The chain on the tensor cores (scan_tc.cu); cudaErrorNotSupported outside its shapes.
cudaError_t launch_scan_tc(const PrefillArgs& a, int num_sms, cudaStream_t s);
int pick_tc_cluster(const Dims& dm, int num_sms);
cudaError_t launch_output(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_output_tc(const PrefillArgs& a, cudaStream_t s);   // bf16 on tcgen05
cudaError_t launch_output_ws(const PrefillArgs& a, cudaStream_t s);   // ... warp-specialised, two query tiles
cudaError_t launch_finalize(const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_sre_map(const SreMapArgs& a, cudaStream_t s);
cudaError_t launch_key_scores(const PrefillArgs& a, cudaStream_t s);       // alternative rules: window scores
cudaError_t launch_finalize_scores(const PrefillArgs& a, cudaStream_t s);  // ... kept for later calls
cudaError_t launch_residual_init(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_clear(const Dims& dm, const StatePtrs& sp, cudaStream_t s);

// Shared-memory bytes a scan CTA needs (0 if the shape is unsupported).
size_t scan_smem_bytes(const Dims& dm);

}  // namespace lola

/*
 * lola.h - C ABI of the B200 (sm_100a) LoLA hybrid-attention layer.
 *
 * The layer is the inference step of "LoLA: Low-Rank Linear Attention With
 * Sparse Caching" (arXiv 2505.23666v3) as its close-reading notes describe
 * it: every query reads a sliding window W of the eta most recent KV pairs,
 * a sparse global cache G of at most lambda raw KV pairs and a linear state
 * (H, s), under one shared softmax normaliser (notes §2.5, Eq. 14).  After
 * each block of tokens the pairs leaving the window and the cache members
 * are scored by Self-Recall Error against the state (notes §2.3, Eq. 10), the
 * lambda highest are kept in G and the rest are folded into (H, s)
 * (notes §2.4, Eqs. 11-13).  Prefill runs this chunk by chunk (notes §2.6,
 * Eq. 15, Fig. 2); decode runs it one token at a time (notes §2.4, Fig. 1).
 *
 * Conventions (all entry points):
 *   - Every pointer named "device" is CUDA device memory on the current
 *     device; "host" pointers are page-locked (pinned) host memory.  q, k, v
 *     and y must be 16-byte aligned (LOLA_ERR_INVALID_ARG otherwise).
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  All work is enqueued asynchronously on it, in stream order.
 *   - The caller owns every buffer.  The library allocates no device memory:
 *     persistent state and per-call scratch live in the caller's `dev_buf`,
 *     sized by lola_state_bytes().  The library owns only the small host
 *     handle returned by lola_state_init() and, per handle, four CUDA
 *     streams and a few events (no device memory), released by
 *     lola_state_free().
 *   - Return value 0 = LOLA_OK; a negative value is one of the LOLA_ERR_*
 *     codes below and lola_last_error_string() describes it (thread-local).
 *     No entry point aborts the process or traps on the device.
 *   - Feature map phi(x) = [softmax(x W_g), softmax(-x W_g)] (Hedgehog form,
 *     fixed by this library; the pages leave phi as "learned"), D = 2 Dh.
 *   - Sequences of a batch advance in lock step: every call processes the
 *     same number of tokens for all B sequences.
 *   - Precision: SRE, selection, fold and the state are f32.  With bf16
 *     inputs the prefill output runs Q K^T in bf16 and P V in f16 on the
 *     tensor cores (f32 accumulation), so values v must satisfy |v| < 65504;
 *     the linear branch phi(q)^T H runs in tf32.  f32 inputs run in f32.
 *
 * Layouts (row-major, contiguous):
 *   q  [B][T][Hq][d], k and v [B][T][Hkv][d]   in `dtype`
 *   y  [B][T][Hq][d]                            float32
 *   W  [Hkv][d][Dh]                             in `dtype`
 *   Query head h reads kv head h / (Hq / Hkv) (grouped-query attention).
 */
#ifndef LOLA_H
#define LOLA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LOLA_OK                 0
#define LOLA_ERR_INVALID_ARG   (-1)  /* null pointer, bad size, T % chunk != 0, ...    */
#define LOLA_ERR_BUF_TOO_SMALL (-2)  /* dev_buf smaller than lola_state_bytes()         */
#define LOLA_ERR_CUDA          (-3)  /* a CUDA call or kernel launch failed             */
#define LOLA_ERR_TIMEOUT       (-4)  /* a bounded device-side wait gave up              */
#define LOLA_ERR_UNSUPPORTED   (-5)  /* shape outside the compiled kernel variants      */

#define LOLA_DTYPE_F32  0
#define LOLA_DTYPE_BF16 1

/* Shape and budget of one layer.  Supported: d in {64, 128}, Dh in {32, 64},
 * 1 <= Hq / Hkv <= 8 and Hq % Hkv == 0, eta >= 1, 0 <= lambda <= 2048,
 * 1 <= chunk <= 256, max_tokens % chunk == 0. */
typedef struct lola_config {
    int B;           /* sequences in the batch                                   */
    int Hq;          /* query heads                                              */
    int Hkv;         /* key/value heads                                          */
    int d;           /* head dimension (d_k = d_v)                               */
    int Dh;          /* feature-map half width; D = 2 Dh                         */
    int eta;         /* sliding-window size: exact pairs preceding a block       */
    int lambda;      /* sparse-cache capacity                                    */
    int chunk;       /* prefill block length C                                   */
    int dtype;       /* LOLA_DTYPE_F32 or LOLA_DTYPE_BF16 (q, k, v, W)           */
    int max_tokens;  /* largest T of one lola_prefill_chunked call (sizes scratch) */
} lola_config;

typedef struct lola_state lola_state;   /* opaque host handle */

/* Device views of the state (for checks and checkpoints).  Slot layouts:
 *   H [B*Hkv][D][d] f32, s [B*Hkv][D] f32,
 *   cache_k / cache_v [B*Hkv][lambda][d] dtype, cache_phik [B*Hkv][lambda][D] f32,
 *   cache_pos [B*Hkv][lambda] int32 (-1 = empty slot),
 *   win_k / win_v [B*Hkv][eta][d] dtype, win_phik [B*Hkv][eta][D] f32; the pair at
 *   position p sits in window slot p % eta.
 *   trace_pos: for stream i, trace_pos + i*trace_stride holds [trace_len][lambda]
 *   int32: the cache positions (by slot) entering each chunk of the last
 *   lola_prefill_chunked call, then the final set (trace_len = chunks + 1);
 *   trace_t0 is the first position of that call. */
typedef struct lola_state_view {
    long long t;            /* tokens processed per sequence                  */
    int n_cache;            /* occupied cache slots (slots 0 .. n_cache-1)   */
    float* H;
    float* s;
    void* cache_k;
    void* cache_v;
    float* cache_phik;
    int* cache_pos;
    void* win_k;
    void* win_v;
    float* win_phik;
    int* trace_pos;
    int trace_len;          /* chunks of the last prefill call + 1 (0 if none)    */
    int trace_stride;       /* ints between the traces of consecutive streams     */
    long long trace_t0;
    int* err_word;          /* device int, nonzero once a bounded device wait gave
                               up (LOLA_ERR_TIMEOUT condition); cleared by reset */
} lola_state_view;

/* Bytes of device memory one layer state needs (persistent state, prefill
 * scratch and host-I/O staging).  Returns LOLA_ERR_INVALID_ARG or
 * LOLA_ERR_UNSUPPORTED for a configuration outside the limits above. */
int lola_state_bytes(const lola_config* cfg, size_t* bytes);

/* Bind a state to `dev_buf` (device, >= lola_state_bytes bytes, 256-byte
 * aligned), copy W (device, [Hkv][d][Dh] in dtype) into it and clear the
 * memories (t = 0, empty window and cache, H = 0, s = 0).  Enqueued on
 * `stream`; *out receives a new host handle.  Memories: notes §2.4, Fig. 1. */
int lola_state_init(const lola_config* cfg, const void* W, void* dev_buf, size_t bytes,
                    void* stream, lola_state** out);

/* Clear the memories again (t = 0) without touching W; the read options and
 * the scoring rule are kept.  Enqueued on stream. */
int lola_state_reset(lola_state* st, void* stream);

/* Release the host handle.  The caller still owns (and frees) dev_buf. */
int lola_state_free(lola_state* st);

/* Chunkwise prefill (notes §2.6, Eq. 15): process T new tokens of every
 * sequence in blocks of `chunk`.  For each block, every query reads the
 * state entering the block (Eq. 14); then the window advances, the leaving
 * pairs and the cache are scored by SRE (Eq. 10; or by the rule chosen with
 * lola_set_scorer), the top lambda stay
 * cached (older position wins exact ties) and the rest are folded (Eqs.
 * 12-13).  q, k, v: device, layouts above; y: device float32 [B][T][Hq][d].
 * T must be a positive multiple of chunk and <= max_tokens.  Calls may split
 * a sequence at any chunk-aligned point; the result equals one call.
 * A call of >= 32 chunks runs the memory-update chain in four chunk segments
 * (sized 2:2:2:1)
 * on an internal high-priority stream and each segment's output on an
 * internal low-priority stream, forked from and joined back into `stream`
 * with events: the call stays stream-ordered on `stream` (and can be captured
 * into a CUDA graph), and its results equal those of one segment. */
int lola_prefill_chunked(lola_state* st, const void* q, const void* k, const void* v,
                         int T, float* y, void* stream);

/* One decode step (notes §2.4, Fig. 1; a block of one token): q [B][Hq][d],
 * k and v [B][Hkv][d] (device, dtype); y [B][Hq][d] float32 (device). */
int lola_decode_step(lola_state* st, const void* q, const void* k, const void* v,
                     float* y, void* stream);

/* Same as lola_prefill_chunked / lola_decode_step, with pinned HOST buffers:
 * the inputs are copied into device staging inside dev_buf, the layer runs,
 * and y is copied back, all ordered on `stream` (synchronise before reading y).
 * A prefill of >= 8 chunks runs as four chunk-aligned calls whose copies in
 * and back run on internal streams, overlapped with the neighbouring
 * segments' compute (double-buffered staging); the result equals one call. */
int lola_prefill_chunked_host(lola_state* st, const void* q, const void* k, const void* v,
                              int T, float* y, void* stream);
int lola_decode_step_host(lola_state* st, const void* q, const void* k, const void* v,
                          float* y, void* stream);

/* Read options.  read_mask hides memory branches from every later read (the
 * module-read ablation of notes §4.8, App. I, Table 12):
 * LOLA_READ_HIDE_STATE drops phi(q)^T H and phi(q)^T s from the numerator
 * and the shared denominator of Eq. 14, LOLA_READ_HIDE_SPARSE drops the
 * cache members' softmax terms; with both, the queries read the window and
 * their block's own causal keys only.  The memories are updated exactly as
 * without a mask.  decode_update_first = 1 makes lola_decode_step take the
 * token equations (notes §2.4, Eqs. 11-14) literally: the new pair enters the
 * window, the pair eta steps back leaves it and is scored with the cache
 * against the state (the lowest SRE is folded), and only then does the
 * query read: the updated cache and state, and the eta most recent pairs,
 * itself included.  The memories evolve identically under both orders; only
 * y differs.  Prefill always reads first (the queries of a block share the
 * state entering it, notes §2.6).  The options persist across
 * lola_state_reset; 0, 0 restores the default.  LOLA_ERR_INVALID_ARG for
 * other bits or values. */
#define LOLA_READ_HIDE_STATE  1
#define LOLA_READ_HIDE_SPARSE 2
int lola_set_read_options(lola_state* st, int read_mask, int decode_update_first);

/* Scoring rule that ranks the leaving pairs and the cache members (notes
 * §4.5, Table 4; App. F, whose Eqs. 22-25 the pages do not print).
 * LOLA_SCORE_SRE (default) is Eq. 10 against the state.  The four
 * alternatives score a key by a sum over every query that reads it exactly
 * through the window or its own block (all heads of its kv group), with
 * a = exp(q.k / sqrt(d)) and f = phi(q)^T phi(k):
 *   LOLA_SCORE_KERNEL_SQ     (a - f)^2      LOLA_SCORE_KERNEL_ABS  |a - f|
 *   LOLA_SCORE_KERNEL_RATIO  f / a          LOLA_SCORE_ATTN        a
 * The sum stops when the key leaves the window and stays frozen while the
 * key is cached; the lambda highest scores are kept (older position on exact
 * ties), the rest folded, as for SRE.  Under decode_update_first a query
 * credits the window it reads after the update.  The rule can change only
 * while no token has been processed (after init or reset; it persists across
 * resets); LOLA_ERR_INVALID_ARG otherwise or for another value.  Prefill
 * with an alternative rule runs unsegmented on `stream`. */
#define LOLA_SCORE_SRE          0
#define LOLA_SCORE_KERNEL_SQ    1
#define LOLA_SCORE_KERNEL_ABS   2
#define LOLA_SCORE_KERNEL_RATIO 3
#define LOLA_SCORE_ATTN         4
int lola_set_scorer(lola_state* st, int scorer);

/* Stored-pair SRE map of the last prefill call (notes §4.4: Fig. 3, and
 * Fig. 10 / Eq. 26 for the relative form).  With n = the chunks of that call
 * (trace_len - 1 of lola_state_export) and t_c = its first position + c *
 * chunk, state time c in [0, n] is the state entering chunk c (c = n: the
 * state after the call).  For every position i < T:
 *   sre[b][g][c][i] = || H_c^T phi(k_i) / (phi(k_i)^T s_c) - v_i ||^2 when
 *                     pair i is folded into the state at time c (it has left
 *                     the window, i < t_c - eta, and is not cached), else 0;
 *   rel[b][g][c][i] = sre[b][g][c][i] - sre[b][g][c_i][i], c_i the first state
 *                     time of the map at which pair i is folded (0 where not
 *                     folded).
 * k, v: device [B][T][Hkv][d] in dtype, every position of the sequences from
 * 0 (the same values the calls received); T must equal the tokens processed.
 * sre, rel: device float32 [B][Hkv][n + 1][T]; rel may be NULL.  The last
 * call on `st` must be a prefill (LOLA_ERR_INVALID_ARG after a decode step,
 * a reset or no prefill).  For a host-buffer prefill of >= 8 chunks "the
 * last call" is the last of its four chunk-aligned calls.  k, v, sre and rel
 * must be 16-byte aligned (LOLA_ERR_INVALID_ARG otherwise); a failed launch
 * returns LOLA_ERR_CUDA.  Reads the state's per-chunk snapshots and changes
 * nothing; fp32 arithmetic, whatever scoring rule chose the cache. */
int lola_sre_map(lola_state* st, const void* k, const void* v, int T, float* sre, float* rel,
                 void* stream);

/* Sync point for device-side failures: waits for `stream` (every call made
 * on it so far) and reads the state's device error word.  Kernels never trap:
 * a bounded wait (an mbarrier the tensor cores should complete, about 4 s of
 * wall time) that gives up sets the word, finishes without that result and
 * returns.  Returns LOLA_ERR_TIMEOUT if any kernel of this state has set it
 * since the last init or reset (the outputs of those calls are not valid;
 * lola_state_reset clears the word), LOLA_ERR_CUDA if the stream reports an
 * error, LOLA_OK otherwise. */
int lola_state_check(lola_state* st, void* stream);

/* Fill *out with device views of the state (no copy, no synchronisation). */
int lola_state_export(const lola_state* st, lola_state_view* out);

/* Tracing aid.  Kernel classes, in this order: 0 feature map, 1 scan (memory
 * update chain), 2 output, 3 finalize, 4 decode, 5 SRE map, 6 window scores of
 * an alternative scoring rule.  While enabled, every kernel
 * launch of `st` is bracketed by CUDA events recorded on its stream.
 * lola_profile_read waits for those events, adds their elapsed times (ms) and
 * launch counts into ms[0..6] and launches[0..6] (n >= 7 entries each) and
 * forgets them.  Enabling does not change what the kernels compute. */
#define LOLA_KERNEL_CLASSES 7
int lola_profile_enable(lola_state* st, int on);
int lola_profile_read(lola_state* st, float* ms, long long* launches, int n);

/* Number of kernels this library has launched in this process. */
long long lola_launch_count(void);

/* Diagnostic self-test of the tensor-core building blocks (no counterpart in
 * the paper): one CTA computes C[128][N] = A[128][K] * B with tcgen05.mma from
 * the shared-memory operand layouts the kernels use, accumulating in tensor
 * memory.  mode bit 0: B given MN-major as [K][N] (else K-major as [N][K]);
 * bit 1: f32 inputs computed as tf32 (else bf16 inputs); bit 2 (with bit 1):
 * 3xTF32 split products; bit 3: A given MN-major as [K][M] (else [M][K]);
 * bit 4 (not with bit 3): A read from tensor memory (K % 32 == 0 for bf16);
 * bit 5: no MMA is issued and the completion wait gives up after about 1 ms
 * (exercises the bounded-wait failure path: *err is set to 1 and C is filled
 * with NaN); bit 6: operands in the 128-byte swizzled layout (128-byte rows
 * in 1024-byte atoms of 8 rows; K % 64 == 0 for bf16, K % 32 == 0 for tf32;
 * with bit 0, N % 64 == 0; tf32 takes it for K-major operands only, not with
 * bits 0 or 3); bit 7 (with bit 2): the hi parts of the shared-memory operands
 * are the raw f32 values, not rounded down to tf32 (the result must equal the
 * bit-2 result bit for bit if kind::tf32 reads only the top 19 bits).  A, B, C, err are device pointers (C f32 row-major, *err set to
 * 1 if the MMA completion wait gave up).  Requires M = 128, 16 <= N <= 256
 * with N % 16 == 0, K a multiple of 16 (bf16, or A in tensor memory) or 8
 * (tf32), operands that fit in shared memory and at most 512 tensor-memory
 * columns (N, plus K, or 2 K for 3xTF32, with A in tensor memory). */
int lola_selftest_umma(int mode, const void* A, const void* B, float* C, int M, int N, int K,
                       int* err, void* stream);

/* One-shot prefill that allocates nothing (this entry point has no
 * counterpart in the paper; it serves callers that cannot call cudaMalloc,
 * such as a plugin that only receives input and output pointers from its
 * host application, or code running where another component owns every
 * device allocation).  It runs lola_prefill_chunked on a fresh state (t = 0)
 * for T tokens of q, k, v and writes y (all device, layouts above; W device
 * [Hkv][d][Dh]).  The state and all scratch live in one array built into the
 * library, LOLA_NOALLOC_SCRATCH_BYTES (64 MiB) of device memory that every
 * GPU which loads the library holds until the process exits.  Configurations
 * whose state and scratch exceed it are rejected with LOLA_ERR_BUF_TOO_SMALL
 * (the need grows with B * Hkv and max_tokens; the 8B-shaped 4K prefill with
 * B = 1 fits).  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call reuses the same array and clears the
 * memories first, so calls whose GPU work overlaps (different streams, or
 * several host threads) race and corrupt each other: serialise them, e.g. on
 * one stream.  The state is not kept after the call. */
#define LOLA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int lola_prefill_once_noalloc(const lola_config* cfg, const void* W, const void* q, const void* k,
                              const void* v, int T, float* y, void* stream);

/* Text of the last error raised on this host thread ("" if none). */
const char* lola_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* LOLA_H */

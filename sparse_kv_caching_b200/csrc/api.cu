// C ABI of the LoLA layer (declared in include/lola.h): argument checks,
// the layout of the caller's device buffer, and the kernel sequence of each
// call.  No device allocation happens here; every byte lives in dev_buf.
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <string>
#include <vector>

#include "lola.h"
#include "lola_internal.h"

namespace lola {
size_t decode_smem_bytes(const Dims& dm);
size_t selftest_smem(int mode, int M, int N, int K);
int selftest_tmem_cols(int mode, int N, int K);
cudaError_t launch_selftest(int mode, const void* A, const void* B, float* C, int M, int N, int K, int* err,
                            cudaStream_t s);
}

struct lola_prof_mark {
    int cls;
    cudaEvent_t a, b;
};

struct lola_state {
    lola_config cfg;
    lola::Dims dm;
    lola::Layout L;
    char* base;
    size_t bytes;
    long long t;
    int last_nc;
    long long last_t0;
    bool prof = false;
    bool resid_ok = true;     // per-slot decode residuals match (H, s)
    int read_mask = 0;        // LOLA_READ_HIDE_* bits applied to every read
    int update_first = 0;     // decode: update the memories before the read
    int scorer = 0;           // LOLA_SCORE_*: how leaving pairs and members are ranked
    std::vector<lola_prof_mark> marks;
    std::vector<cudaEvent_t> pool;
    // Prefill overlap: the chain runs on a high-priority stream in chunk segments,
    // each segment's output on a low-priority stream as soon as its snapshots exist
    // (null when the state was built without them: one stream, one segment).
    cudaStream_t s_chain = nullptr, s_out = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_seg = nullptr, ev_join_chain = nullptr, ev_join_out = nullptr;
    // Host-buffer prefill: copies in and out on their own streams, overlapped with
    // the compute of neighbouring segments (double-buffered staging).
    cudaStream_t s_in = nullptr, s_back = nullptr;
    cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_done[2] = {nullptr, nullptr}, ev_back[2] = {nullptr, nullptr};
};

namespace {

thread_local std::string g_err;
constexpr int kSplitMinChunks = 32;   // calls with fewer chunks run in one segment
// Relative chunk counts of the chain segments.  The output of segment i runs
// beside the chain of segment i+1; only the last segment's output is exposed,
// so the last segment is the shortest.  2:2:2:2:1 measured 1.6 % faster than
// 2:2:2:1 on the 8B-shaped 16384-token prefill (3 % on the 1B-shaped 32768-token
// one, 1.3 % slower on the 4096-token one); 3:3:3:1, 1:2:2:2:2:1, 1:1:2:2:2:1
// and 1:2:3:3:2:1 were slower there.
constexpr int kSegWeights[] = {2, 2, 2, 2, 1};
constexpr int kSplitSegments = sizeof(kSegWeights) / sizeof(kSegWeights[0]);
constexpr int kHostSegments = 4;      // host-buffer prefill: copies overlap compute per segment
std::atomic<long long> g_launches{0};

cudaEvent_t take_event(lola_state* st) {
    if (!st->pool.empty()) { cudaEvent_t e = st->pool.back(); st->pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Run one launcher; count its kernels and, when profiling, bracket it with events.
template <typename F>
cudaError_t traced(lola_state* st, int cls, int kernels, cudaStream_t s, F&& launch) {
    cudaEvent_t a = nullptr, b = nullptr;
    if (st->prof) { a = take_event(st); b = take_event(st); if (a) cudaEventRecord(a, s); }
    cudaError_t e = launch();
    if (e == cudaSuccess) g_launches += kernels;
    if (st->prof && a && b) {
        cudaEventRecord(b, s);
        st->marks.push_back({cls, a, b});
    }
    return e;
}

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(LOLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxSmem = 227 * 1024;

int make_dims(const lola_config* c, lola::Dims* dm) {
    if (!c) return fail(LOLA_ERR_INVALID_ARG, "null config");
    if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv)
        return fail(LOLA_ERR_INVALID_ARG, "bad heads/batch: B=%d Hq=%d Hkv=%d", c->B, c->Hq, c->Hkv);
    if (c->Hq / c->Hkv > 8) return fail(LOLA_ERR_UNSUPPORTED, "Hq/Hkv=%d > 8", c->Hq / c->Hkv);
    if (c->d != 64 && c->d != 128) return fail(LOLA_ERR_UNSUPPORTED, "d=%d (64 or 128)", c->d);
    if (c->Dh != 32 && c->Dh != 64) return fail(LOLA_ERR_UNSUPPORTED, "Dh=%d (32 or 64)", c->Dh);
    if (c->eta < 1) return fail(LOLA_ERR_INVALID_ARG, "eta=%d < 1", c->eta);
    if (c->lambda < 0 || c->lambda > 2048) return fail(LOLA_ERR_UNSUPPORTED, "lambda=%d (0..2048)", c->lambda);
    if (c->chunk < 1 || c->chunk > 256) return fail(LOLA_ERR_UNSUPPORTED, "chunk=%d (1..256)", c->chunk);
    if (c->max_tokens < c->chunk || c->max_tokens % c->chunk)
        return fail(LOLA_ERR_INVALID_ARG, "max_tokens=%d must be a positive multiple of chunk=%d",
                    c->max_tokens, c->chunk);
    if (c->dtype != LOLA_DTYPE_F32 && c->dtype != LOLA_DTYPE_BF16)
        return fail(LOLA_ERR_INVALID_ARG, "dtype=%d", c->dtype);
    dm->B = c->B; dm->Hq = c->Hq; dm->Hkv = c->Hkv; dm->Gq = c->Hq / c->Hkv;
    dm->d = c->d; dm->Dh = c->Dh; dm->D = 2 * c->Dh;
    dm->eta = c->eta; dm->lam = c->lambda; dm->C = c->chunk; dm->dtype = c->dtype;
    dm->S = c->B * c->Hkv; dm->max_tokens = c->max_tokens; dm->nc_max = c->max_tokens / c->chunk;
    dm->esize = c->dtype == LOLA_DTYPE_BF16 ? 2 : 4;
    if (lola::scan_smem_bytes(*dm) > (size_t)kMaxSmem)
        return fail(LOLA_ERR_UNSUPPORTED, "lambda + chunk too large for the scan kernel's shared memory");
    if (lola::decode_smem_bytes(*dm) > (size_t)kMaxSmem)
        return fail(LOLA_ERR_UNSUPPORTED, "lambda + eta too large for the decode kernel's shared memory");
    return LOLA_OK;
}

lola::Layout make_layout(const lola::Dims& dm) {
    lola::Layout L{};
    size_t off = 0;
    auto take = [&](size_t n) { size_t r = off; off = (off + n + 255) & ~(size_t)255; return r; };
    const size_t S = dm.S, e = dm.esize, snaps = (size_t)dm.nc_max + 1, T = dm.max_tokens;
    L.W = take((size_t)dm.Hkv * dm.d * dm.Dh * e);
    L.err = take(256);     // device error word: before the host-I/O staging, which one-shot calls omit
    L.H = take(S * dm.D * dm.d * 4);
    L.s = take(S * dm.D * 4);
    L.cache_k = take(S * dm.lam * dm.d * e);
    L.cache_v = take(S * dm.lam * dm.d * e);
    L.cache_phik = take(S * dm.lam * dm.D * 4);
    L.cache_pos = take(S * dm.lam * 4);
    L.win_k = take(S * dm.eta * dm.d * e);
    L.win_v = take(S * dm.eta * dm.d * e);
    L.win_phik = take(S * dm.eta * dm.D * 4);
    L.cache_R = take(S * dm.lam * dm.d * 4);
    L.cache_den = take(S * dm.lam * 4);
    L.cache_sc = take(S * dm.lam * 4);
    L.win_sc = take(S * dm.eta * 4);
    L.phik_new = take(S * T * dm.D * 4);
    L.key_sc = take(S * (dm.eta + T) * 4);
    L.snap_pos = take(S * snaps * dm.lam * 4);
    L.snap_H = take(S * snaps * dm.D * dm.d * 4);
    L.snap_s = take(S * snaps * dm.D * 4);
    L.io_q = take((size_t)dm.B * T * dm.Hq * dm.d * e);
    L.io_k = take((size_t)dm.B * T * dm.Hkv * dm.d * e);
    L.io_v = take((size_t)dm.B * T * dm.Hkv * dm.d * e);
    L.io_y = take((size_t)dm.B * T * dm.Hq * dm.d * 4);
    L.total = off;
    return L;
}

lola::StatePtrs state_ptrs(const lola_state* st) {
    lola::StatePtrs p;
    char* b = st->base;
    p.W = b + st->L.W;
    p.H = (float*)(b + st->L.H);
    p.s = (float*)(b + st->L.s);
    p.cache_k = b + st->L.cache_k;
    p.cache_v = b + st->L.cache_v;
    p.cache_phik = (float*)(b + st->L.cache_phik);
    p.cache_pos = (int*)(b + st->L.cache_pos);
    p.win_k = b + st->L.win_k;
    p.win_v = b + st->L.win_v;
    p.win_phik = (float*)(b + st->L.win_phik);
    p.cache_R = (float*)(b + st->L.cache_R);
    p.cache_den = (float*)(b + st->L.cache_den);
    p.cache_sc = (float*)(b + st->L.cache_sc);
    p.win_sc = (float*)(b + st->L.win_sc);
    return p;
}

int clear_state(lola_state* st, cudaStream_t s) {
    const lola::Dims& dm = st->dm;
    const lola::Layout& L = st->L;
    // everything from H up to (not including) the prefill scratch
    cudaError_t e = cudaMemsetAsync(st->base + L.H, 0, L.phik_new - L.H, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(st->base + L.err, 0, 256, s);
    if (e == cudaSuccess && dm.lam > 0)
        e = cudaMemsetAsync(st->base + L.cache_pos, 0xFF, (size_t)dm.S * dm.lam * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the state");
    st->t = 0;
    st->last_nc = -1;
    st->last_t0 = 0;
    st->resid_ok = true;
    return LOLA_OK;
}

bool misaligned(const void* p) { return ((uintptr_t)p & 15u) != 0; }

}  // namespace

extern "C" {

const char* lola_last_error_string(void) { return g_err.c_str(); }

int lola_state_bytes(const lola_config* cfg, size_t* bytes) {
    lola::Dims dm;
    int rc = make_dims(cfg, &dm);
    if (rc) return rc;
    if (!bytes) return fail(LOLA_ERR_INVALID_ARG, "null bytes pointer");
    *bytes = make_layout(dm).total;
    return LOLA_OK;
}

int lola_state_init(const lola_config* cfg, const void* W, void* dev_buf, size_t bytes,
                    void* stream, lola_state** out) {
    lola::Dims dm;
    int rc = make_dims(cfg, &dm);
    if (rc) return rc;
    if (!W || !dev_buf || !out) return fail(LOLA_ERR_INVALID_ARG, "null W, dev_buf or out");
    if ((uintptr_t)dev_buf & 255) return fail(LOLA_ERR_INVALID_ARG, "dev_buf is not 256-byte aligned");
    const lola::Layout L = make_layout(dm);
    if (bytes < L.total)
        return fail(LOLA_ERR_BUF_TOO_SMALL, "dev_buf has %zu bytes, needs %zu", bytes, L.total);
    lola_state* st = new lola_state();
    st->cfg = *cfg;
    st->dm = dm;
    st->L = L;
    st->base = (char*)dev_buf;
    st->bytes = bytes;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(st->base + L.W, W, (size_t)dm.Hkv * dm.d * dm.Dh * dm.esize,
                                    cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) { delete st; return cuda_fail(e, "copying W"); }
    rc = clear_state(st, s);
    if (rc) { delete st; return rc; }
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&st->s_chain, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&st->s_out, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_seg, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_join_chain, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_join_out, cudaEventDisableTiming) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st->s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st->s_back, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_in[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_in[1], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_done[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_done[1], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_back[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&st->ev_back[1], cudaEventDisableTiming) != cudaSuccess) {
        e = cudaGetLastError();
        lola_state_free(st);
        return cuda_fail(e, "creating the prefill streams");
    }
    *out = st;
    return LOLA_OK;
}

int lola_state_reset(lola_state* st, void* stream) {
    if (!st) return fail(LOLA_ERR_INVALID_ARG, "null state");
    return clear_state(st, (cudaStream_t)stream);
}

int lola_state_free(lola_state* st) {
    if (st) {
        for (auto& m : st->marks) { cudaEventDestroy(m.a); cudaEventDestroy(m.b); }
        for (auto e : st->pool) cudaEventDestroy(e);
        for (cudaEvent_t e : {st->ev_fork, st->ev_seg, st->ev_join_chain, st->ev_join_out, st->ev_in[0],
                              st->ev_in[1], st->ev_done[0], st->ev_done[1], st->ev_back[0], st->ev_back[1]})
            if (e) cudaEventDestroy(e);
        for (cudaStream_t q : {st->s_chain, st->s_out, st->s_in, st->s_back})
            if (q) cudaStreamDestroy(q);
    }
    delete st;
    return LOLA_OK;
}

int lola_sre_map(lola_state* st, const void* k, const void* v, int T, float* sre, float* rel, void* stream) {
    if (!st || !k || !v || !sre) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    if (misaligned(k) || misaligned(v) || misaligned(sre) || (rel && misaligned(rel)))
        return fail(LOLA_ERR_INVALID_ARG, "k, v, sre and rel must be 16-byte aligned");
    const lola::Dims& dm = st->dm;
    if (st->last_nc < 0) return fail(LOLA_ERR_INVALID_ARG, "no prefill call since the state was initialised or reset");
    if (st->t != st->last_t0 + (long long)st->last_nc * dm.C)
        return fail(LOLA_ERR_INVALID_ARG, "decode steps followed the last prefill call; its snapshots no longer "
                    "describe the state");
    if ((long long)T != st->t)
        return fail(LOLA_ERR_INVALID_ARG, "T=%d must equal the tokens processed (%lld)", T, st->t);
    lola::SreMapArgs a{};
    a.dm = dm;
    a.k = k; a.v = v;
    a.W = st->base + st->L.W;
    a.snap_H = (const float*)(st->base + st->L.snap_H);
    a.snap_s = (const float*)(st->base + st->L.snap_s);
    a.snap_pos = (const int*)(st->base + st->L.snap_pos);
    a.sre = sre; a.rel = rel;
    a.T = T;
    a.t0 = (int)st->last_t0;
    a.nc = st->last_nc;
    cudaStream_t s = (cudaStream_t)stream;
    const cudaError_t e = traced(st, 5, 1, s, [&] { return lola::launch_sre_map(a, s); });
    if (e != cudaSuccess) return cuda_fail(e, "SRE map kernel");
    return LOLA_OK;
}

int lola_set_scorer(lola_state* st, int scorer) {
    if (!st) return fail(LOLA_ERR_INVALID_ARG, "null state");
    if (scorer < LOLA_SCORE_SRE || scorer > LOLA_SCORE_ATTN)
        return fail(LOLA_ERR_INVALID_ARG, "scorer=%d is not one of the LOLA_SCORE_* rules", scorer);
    if (st->t != 0 && scorer != st->scorer)
        return fail(LOLA_ERR_INVALID_ARG, "the scoring rule can change only before the first token "
                    "(after lola_state_init or lola_state_reset)");
    st->scorer = scorer;
    return LOLA_OK;
}

int lola_set_read_options(lola_state* st, int read_mask, int decode_update_first) {
    if (!st) return fail(LOLA_ERR_INVALID_ARG, "null state");
    if (read_mask & ~(LOLA_READ_HIDE_STATE | LOLA_READ_HIDE_SPARSE))
        return fail(LOLA_ERR_INVALID_ARG, "read_mask=%d has bits other than LOLA_READ_HIDE_STATE | LOLA_READ_HIDE_SPARSE",
                    read_mask);
    if (decode_update_first != 0 && decode_update_first != 1)
        return fail(LOLA_ERR_INVALID_ARG, "decode_update_first=%d must be 0 or 1", decode_update_first);
    st->read_mask = read_mask;
    st->update_first = decode_update_first;
    return LOLA_OK;
}

int lola_profile_enable(lola_state* st, int on) {
    if (!st) return fail(LOLA_ERR_INVALID_ARG, "null state");
    st->prof = on != 0;
    return LOLA_OK;
}

int lola_profile_read(lola_state* st, float* ms, long long* launches, int n) {
    if (!st || !ms || !launches || n < LOLA_KERNEL_CLASSES)
        return fail(LOLA_ERR_INVALID_ARG, "null argument or n < %d", LOLA_KERNEL_CLASSES);
    for (int i = 0; i < LOLA_KERNEL_CLASSES; ++i) { ms[i] = 0.f; launches[i] = 0; }
    int rc = LOLA_OK;
    for (auto& m : st->marks) {
        float t = 0.f;
        cudaError_t e = cudaEventSynchronize(m.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, m.a, m.b);
        if (e != cudaSuccess && rc == LOLA_OK) rc = cuda_fail(e, "reading profile events");
        ms[m.cls] += t;
        launches[m.cls] += 1;
        st->pool.push_back(m.a);
        st->pool.push_back(m.b);
    }
    st->marks.clear();
    return rc;
}

long long lola_launch_count(void) { return g_launches.load(); }

int lola_selftest_umma(int mode, const void* A, const void* B, float* C, int M, int N, int K, int* err,
                       void* stream) {
    if (!A || !B || !C || !err) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    const bool tf32 = mode & 2;
    if (mode < 0 || mode > 255 || ((mode & 4) && !tf32) || ((mode & 128) && !(mode & 4)) || ((mode & 8) && (mode & 16)) ||
        ((mode & 64) && tf32 && (mode & (1 | 8))))
        return fail(LOLA_ERR_INVALID_ARG, "mode=%d", mode);
    if ((mode & 64) && (K % (tf32 ? 32 : 64) || ((mode & 1) && N % 64)))
        return fail(LOLA_ERR_INVALID_ARG, "swizzled operands need 128-byte rows along K (and N %% 64 == 0 for MN-major B)");
    if (M != 128 || N < 16 || N > 256 || N % 16 || K < (tf32 ? 8 : 16) || K % (tf32 ? 8 : 16))
        return fail(LOLA_ERR_INVALID_ARG, "unsupported shape M=%d N=%d K=%d", M, N, K);
    if ((mode & 16) && K % (tf32 ? 16 : 32)) return fail(LOLA_ERR_INVALID_ARG, "A in tensor memory needs K %% 16 == 0 (tf32) or K %% 32 == 0 (bf16)");
    if (lola::selftest_tmem_cols(mode, N, K) > 512)
        return fail(LOLA_ERR_UNSUPPORTED, "accumulator and A need more than 512 tensor-memory columns");
    if (lola::selftest_smem(mode, M, N, K) > (size_t)kMaxSmem)
        return fail(LOLA_ERR_UNSUPPORTED, "operands do not fit in shared memory");
    cudaError_t e = lola::launch_selftest(mode, A, B, C, M, N, K, err, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "self-test kernel");
    g_launches += 1;
    return LOLA_OK;
}

int lola_prefill_chunked(lola_state* st, const void* q, const void* k, const void* v, int T,
                         float* y, void* stream) {
    if (!st || !q || !k || !v || !y) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(y))
        return fail(LOLA_ERR_INVALID_ARG, "q, k, v and y must be 16-byte aligned");
    const lola::Dims& dm = st->dm;
    if (T < 1 || T % dm.C || T > dm.max_tokens)
        return fail(LOLA_ERR_INVALID_ARG, "T=%d must be a positive multiple of chunk=%d and <= max_tokens=%d",
                    T, dm.C, dm.max_tokens);
    if (st->t + (long long)T >= 0x7fffffffLL) return fail(LOLA_ERR_INVALID_ARG, "position overflow");
    lola::PrefillArgs a{};
    a.dm = dm;
    a.sp = state_ptrs(st);
    a.q = q; a.k = k; a.v = v; a.y = y;
    a.T = T;
    a.t_start = (int)st->t;
    a.nc = T / dm.C;
    a.c_begin = 0;
    a.c_end = a.nc;
    a.read_mask = st->read_mask;
    a.scorer = st->scorer;
    a.key_sc = (float*)(st->base + st->L.key_sc);
    a.phik_new = (float*)(st->base + st->L.phik_new);
    a.snap_pos = (int*)(st->base + st->L.snap_pos);
    a.snap_H = (float*)(st->base + st->L.snap_H);
    a.snap_s = (float*)(st->base + st->L.snap_s);
    a.err = (int*)(st->base + st->L.err);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    auto output = [&](cudaStream_t q) {
        return dm.dtype == LOLA_DTYPE_BF16 ? lola::launch_output_tc(a, q) : lola::launch_output(a, q);
    };
    // chunk boundaries of the chain segments (one segment below kSplitMinChunks chunks)
    int bounds[kSplitSegments + 1] = {0};
    int nseg = 1;
    bounds[1] = a.nc;
    if (a.nc >= kSplitMinChunks) {
        int wsum = 0, acc = 0;
        for (int w : kSegWeights) wsum += w;
        nseg = kSplitSegments;
        for (int i = 0; i < nseg; ++i) {
            acc += kSegWeights[i];
            bounds[i + 1] = (int)(((long long)a.nc * acc + wsum - 1) / wsum);
        }
    }
    if (st->scorer != LOLA_SCORE_SRE) {
        // Alternative rules: every key's window score first (it needs the call's queries,
        // not the state), then the chain ranks by those scores, then the output.
        if ((e = traced(st, 0, 1, s, [&] { return lola::launch_phi_keys(a, s); })) != cudaSuccess)
            return cuda_fail(e, "feature-map kernel");
        if ((e = traced(st, 6, 1, s, [&] { return lola::launch_key_scores(a, s); })) != cudaSuccess)
            return cuda_fail(e, "window-score kernel");
        if ((e = traced(st, 1, 1, s, [&] { return lola::launch_scan(a, s); })) != cudaSuccess)
            return cuda_fail(e, "scan kernel");
        if ((e = traced(st, 2, 1, s, [&] { return output(s); })) != cudaSuccess)
            return cuda_fail(e, "output kernel");
        if ((e = traced(st, 3, 1, s, [&] { return lola::launch_finalize_scores(a, s); })) != cudaSuccess)
            return cuda_fail(e, "window-score finalize kernel");
    } else if (st->s_chain && nseg > 1) {
        // The chain of segment i and the output of segment i-1 run at the same time:
        // the chain holds one cluster per stream, the output fills the other SMs.  The
        // feature map of the first segment's keys runs first; the rest of the keys
        // are mapped on the output stream while the first segment's chain runs.
        a.c_end = bounds[1];
        if ((e = traced(st, 0, 1, s, [&] { return lola::launch_phi_keys(a, s); })) != cudaSuccess)
            return cuda_fail(e, "feature-map kernel");
        if ((e = cudaEventRecord(st->ev_fork, s)) || (e = cudaStreamWaitEvent(st->s_chain, st->ev_fork, 0)) ||
            (e = cudaStreamWaitEvent(st->s_out, st->ev_fork, 0)))
            return cuda_fail(e, "forking the prefill streams");
        a.c_begin = bounds[1];
        a.c_end = a.nc;
        if ((e = traced(st, 0, 1, st->s_out, [&] { return lola::launch_phi_keys(a, st->s_out); })) != cudaSuccess)
            return cuda_fail(e, "feature-map kernel");
        if ((e = cudaEventRecord(st->ev_join_out, st->s_out)))
            return cuda_fail(e, "ordering the feature map");
        for (int i = 0; i < nseg; ++i) {
            a.c_begin = bounds[i];
            a.c_end = bounds[i + 1];
            if (a.c_begin == a.c_end) continue;
            if (i == 1 && (e = cudaStreamWaitEvent(st->s_chain, st->ev_join_out, 0)))
                return cuda_fail(e, "ordering the feature map");
            if ((e = traced(st, 1, 1, st->s_chain, [&] { return lola::launch_scan(a, st->s_chain); })) != cudaSuccess)
                return cuda_fail(e, "scan kernel");
            if ((e = cudaEventRecord(st->ev_seg, st->s_chain)) || (e = cudaStreamWaitEvent(st->s_out, st->ev_seg, 0)))
                return cuda_fail(e, "ordering a prefill segment");
            if ((e = traced(st, 2, 1, st->s_out, [&] { return output(st->s_out); })) != cudaSuccess)
                return cuda_fail(e, "output kernel");
        }
        a.c_begin = 0;
        a.c_end = a.nc;
        if ((e = cudaEventRecord(st->ev_join_chain, st->s_chain)) || (e = cudaEventRecord(st->ev_join_out, st->s_out)) ||
            (e = cudaStreamWaitEvent(s, st->ev_join_chain, 0)) || (e = cudaStreamWaitEvent(s, st->ev_join_out, 0)))
            return cuda_fail(e, "joining the prefill streams");
    } else {
        if ((e = traced(st, 0, 1, s, [&] { return lola::launch_phi_keys(a, s); })) != cudaSuccess)
            return cuda_fail(e, "feature-map kernel");
        if ((e = traced(st, 1, 1, s, [&] { return lola::launch_scan(a, s); })) != cudaSuccess)
            return cuda_fail(e, "scan kernel");
        if ((e = traced(st, 2, 1, s, [&] { return output(s); })) != cudaSuccess)
            return cuda_fail(e, "output kernel");
    }
    if ((e = traced(st, 3, dm.lam > 0 ? 2 : 1, s, [&] { return lola::launch_finalize(a, s); })) != cudaSuccess)
        return cuda_fail(e, "finalize kernels");
    st->last_nc = a.nc;
    st->last_t0 = st->t;
    st->t += T;
    st->resid_ok = false;     // recomputed before the next decode step
    return LOLA_OK;
}

int lola_decode_step(lola_state* st, const void* q, const void* k, const void* v, float* y,
                     void* stream) {
    if (!st || !q || !k || !v || !y) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(y))
        return fail(LOLA_ERR_INVALID_ARG, "q, k, v and y must be 16-byte aligned");
    if (st->t + 1 >= 0x7fffffffLL) return fail(LOLA_ERR_INVALID_ARG, "position overflow");
    lola::DecodeArgs a{};
    a.dm = st->dm;
    a.sp = state_ptrs(st);
    a.q = q; a.k = k; a.v = v; a.y = y;
    a.t = (int)st->t;
    a.read_mask = st->read_mask;
    a.update_first = st->update_first;
    a.scorer = st->scorer;
    a.err = (int*)(st->base + st->L.err);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (!st->resid_ok && st->scorer == LOLA_SCORE_SRE) {
        if ((e = traced(st, 4, st->dm.lam > 0 ? 1 : 0, s, [&] { return lola::launch_residual_init(a, s); })) != cudaSuccess)
            return cuda_fail(e, "decode residual init kernel");
        st->resid_ok = true;
    }
    e = traced(st, 4, 1, s, [&] { return lola::launch_decode(a, s); });
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel");
    st->t += 1;
    return LOLA_OK;
}

int lola_prefill_chunked_host(lola_state* st, const void* q, const void* k, const void* v, int T,
                              float* y, void* stream) {
    if (!st || !q || !k || !v || !y) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    const lola::Dims& dm = st->dm;
    if (T < 1 || T % dm.C || T > dm.max_tokens)
        return fail(LOLA_ERR_INVALID_ARG, "T=%d must be a positive multiple of chunk and <= max_tokens", T);
    cudaStream_t s = (cudaStream_t)stream;
    char* b = st->base;
    cudaError_t e;
    const int nc = T / dm.C;
    if (!st->s_in || nc < 2 * kHostSegments) {
        const size_t nq = (size_t)dm.B * T * dm.Hq * dm.d, nk = (size_t)dm.B * T * dm.Hkv * dm.d;
        if ((e = cudaMemcpyAsync(b + st->L.io_q, q, nq * dm.esize, cudaMemcpyHostToDevice, s)) ||
            (e = cudaMemcpyAsync(b + st->L.io_k, k, nk * dm.esize, cudaMemcpyHostToDevice, s)) ||
            (e = cudaMemcpyAsync(b + st->L.io_v, v, nk * dm.esize, cudaMemcpyHostToDevice, s)))
            return cuda_fail(e, "host-to-device copy");
        int rc = lola_prefill_chunked(st, b + st->L.io_q, b + st->L.io_k, b + st->L.io_v, T,
                                      (float*)(b + st->L.io_y), stream);
        if (rc) return rc;
        if ((e = cudaMemcpyAsync(y, b + st->L.io_y, nq * 4, cudaMemcpyDeviceToHost, s)))
            return cuda_fail(e, "device-to-host copy");
        return LOLA_OK;
    }
    // Pipelined: the call is split at chunk boundaries into kHostSegments calls (a
    // split call equals one call).  Segment i's inputs are copied in on s_in while
    // segment i-1 computes on s and segment i-2's output is copied back on s_back;
    // staging is double-buffered inside the io region (two segments fit because a
    // segment is at most half of max_tokens).
    const int seg_chunks = (nc + kHostSegments - 1) / kHostSegments;
    const int Ts = seg_chunks * dm.C;
    const size_t rq = (size_t)dm.Hq * dm.d, rk = (size_t)dm.Hkv * dm.d;      // elements per token
    const size_t half_q = (size_t)dm.B * Ts * rq, half_k = (size_t)dm.B * Ts * rk;
    if ((e = cudaEventRecord(st->ev_fork, s)) || (e = cudaStreamWaitEvent(st->s_in, st->ev_fork, 0)) ||
        (e = cudaStreamWaitEvent(st->s_back, st->ev_fork, 0)))
        return cuda_fail(e, "ordering the host-buffer copies");
    int nseg = 0;
    for (int t0 = 0; t0 < T; t0 += Ts, ++nseg) {
        const int bi = nseg & 1, Tl = std::min(Ts, T - t0);
        char* sq = b + st->L.io_q + bi * half_q * dm.esize;
        char* sk = b + st->L.io_k + bi * half_k * dm.esize;
        char* sv = b + st->L.io_v + bi * half_k * dm.esize;
        float* sy = (float*)(b + st->L.io_y) + bi * half_q;
        // inputs of this segment, once the compute that last used this buffer is done
        if (nseg >= 2 && (e = cudaStreamWaitEvent(st->s_in, st->ev_done[bi], 0))) return cuda_fail(e, "ordering");
        const size_t wq = Tl * rq * dm.esize, wk = Tl * rk * dm.esize;
        if ((e = cudaMemcpy2DAsync(sq, wq, (const char*)q + t0 * rq * dm.esize, (size_t)T * rq * dm.esize, wq, dm.B,
                                   cudaMemcpyHostToDevice, st->s_in)) ||
            (e = cudaMemcpy2DAsync(sk, wk, (const char*)k + t0 * rk * dm.esize, (size_t)T * rk * dm.esize, wk, dm.B,
                                   cudaMemcpyHostToDevice, st->s_in)) ||
            (e = cudaMemcpy2DAsync(sv, wk, (const char*)v + t0 * rk * dm.esize, (size_t)T * rk * dm.esize, wk, dm.B,
                                   cudaMemcpyHostToDevice, st->s_in)) ||
            (e = cudaEventRecord(st->ev_in[bi], st->s_in)))
            return cuda_fail(e, "host-to-device copy");
        // compute, once the inputs are in and the output buffer has been copied back
        if ((e = cudaStreamWaitEvent(s, st->ev_in[bi], 0)) ||
            (nseg >= 2 && (e = cudaStreamWaitEvent(s, st->ev_back[bi], 0))))
            return cuda_fail(e, "ordering");
        int rc = lola_prefill_chunked(st, sq, sk, sv, Tl, sy, stream);
        if (rc) return rc;
        if ((e = cudaEventRecord(st->ev_done[bi], s)) || (e = cudaStreamWaitEvent(st->s_back, st->ev_done[bi], 0)))
            return cuda_fail(e, "ordering");
        const size_t wy = Tl * rq * 4;
        if ((e = cudaMemcpy2DAsync((char*)y + t0 * rq * 4, (size_t)T * rq * 4, sy, wy, wy, dm.B,
                                   cudaMemcpyDeviceToHost, st->s_back)) ||
            (e = cudaEventRecord(st->ev_back[bi], st->s_back)))
            return cuda_fail(e, "device-to-host copy");
    }
    // the caller's stream resumes after the last copies back
    for (int bi = 0; bi < std::min(nseg, 2); ++bi)
        if ((e = cudaStreamWaitEvent(s, st->ev_back[bi], 0))) return cuda_fail(e, "joining the copy streams");
    return LOLA_OK;
}

int lola_decode_step_host(lola_state* st, const void* q, const void* k, const void* v, float* y,
                          void* stream) {
    if (!st || !q || !k || !v || !y) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    const lola::Dims& dm = st->dm;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t nq = (size_t)dm.B * dm.Hq * dm.d, nk = (size_t)dm.B * dm.Hkv * dm.d;
    char* b = st->base;
    cudaError_t e;
    if ((e = cudaMemcpyAsync(b + st->L.io_q, q, nq * dm.esize, cudaMemcpyHostToDevice, s)) ||
        (e = cudaMemcpyAsync(b + st->L.io_k, k, nk * dm.esize, cudaMemcpyHostToDevice, s)) ||
        (e = cudaMemcpyAsync(b + st->L.io_v, v, nk * dm.esize, cudaMemcpyHostToDevice, s)))
        return cuda_fail(e, "host-to-device copy");
    int rc = lola_decode_step(st, b + st->L.io_q, b + st->L.io_k, b + st->L.io_v,
                              (float*)(b + st->L.io_y), stream);
    if (rc) return rc;
    if ((e = cudaMemcpyAsync(y, b + st->L.io_y, nq * 4, cudaMemcpyDeviceToHost, s)))
        return cuda_fail(e, "device-to-host copy");
    return LOLA_OK;
}

int lola_state_check(lola_state* st, void* stream) {
    if (!st) return fail(LOLA_ERR_INVALID_ARG, "null state");
    cudaStream_t s = (cudaStream_t)stream;
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, st->base + st->L.err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (word != 0)
        return fail(LOLA_ERR_TIMEOUT, "a bounded device-side wait gave up (error word 0x%x); the results of "
                    "the calls since the last reset are not valid: reset the state", (unsigned)word);
    return LOLA_OK;
}

int lola_state_export(const lola_state* st, lola_state_view* out) {
    if (!st || !out) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    const lola::StatePtrs p = state_ptrs(st);
    const lola::Dims& dm = st->dm;
    std::memset(out, 0, sizeof *out);
    out->t = st->t;
    const long long left = st->t - dm.eta;
    out->n_cache = (int)(left <= 0 ? 0 : (left < dm.lam ? left : dm.lam));
    out->H = p.H;
    out->s = p.s;
    out->cache_k = p.cache_k;
    out->cache_v = p.cache_v;
    out->cache_phik = p.cache_phik;
    out->cache_pos = p.cache_pos;
    out->win_k = p.win_k;
    out->win_v = p.win_v;
    out->win_phik = p.win_phik;
    out->trace_pos = (int*)(st->base + st->L.snap_pos);
    out->trace_len = st->last_nc < 0 ? 0 : st->last_nc + 1;
    out->trace_stride = (dm.nc_max + 1) * dm.lam;
    out->trace_t0 = st->last_t0;
    out->err_word = (int*)(st->base + st->L.err);
    return LOLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// One-shot prefill for callers that cannot allocate device memory.
//
// Its persistent state and scratch live in a file-scope device array of
// LOLA_NOALLOC_SCRATCH_BYTES, created when the library's module is loaded on a
// device and held by that device until the process exits.  Host code only
// ever sees the array's host-side stand-in symbol; the device address comes
// from cudaGetSymbolAddress, fetched once per device (with that device
// current) on the first call there and cached.
// ---------------------------------------------------------------------------
#include <mutex>

static __device__ __align__(256) unsigned char g_noalloc_scratch[LOLA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(LOLA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch array");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LOLA_OK;
}

}  // namespace

extern "C" int lola_prefill_once_noalloc(const lola_config* cfg, const void* W, const void* q,
                                         const void* k, const void* v, int T, float* y,
                                         void* stream) {
    lola::Dims dm;
    int rc = make_dims(cfg, &dm);
    if (rc) return rc;
    if (!W || !q || !k || !v || !y) return fail(LOLA_ERR_INVALID_ARG, "null argument");
    if (T < 1 || T % dm.C || T > dm.max_tokens)
        return fail(LOLA_ERR_INVALID_ARG, "T=%d must be a positive multiple of chunk=%d and <= max_tokens=%d",
                    T, dm.C, dm.max_tokens);
    const lola::Layout L = make_layout(dm);
    // state + prefill scratch + error word; the host-I/O staging, the only regions
    // after io_q, is never touched by a device-buffer prefill
    const size_t need = L.io_q;
    if (L.err + 256 > need || L.snap_s >= need || L.key_sc >= need)
        return fail(LOLA_ERR_CUDA, "internal layout error: a prefill region lies beyond the one-shot array's need");
    if (need > (size_t)LOLA_NOALLOC_SCRATCH_BYTES)
        return fail(LOLA_ERR_BUF_TOO_SMALL,
                    "this configuration needs %zu bytes of state and scratch; the built-in array holds %zu "
                    "(lower max_tokens, or use lola_state_init with a caller buffer)",
                    need, (size_t)LOLA_NOALLOC_SCRATCH_BYTES);
    void* base = nullptr;
    rc = noalloc_scratch(&base);
    if (rc) return rc;
    lola_state st;
    st.cfg = *cfg;
    st.dm = dm;
    st.L = L;
    st.base = (char*)base;
    st.bytes = need;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(st.base + L.W, W, (size_t)dm.Hkv * dm.d * dm.Dh * dm.esize,
                                    cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copying W");
    rc = clear_state(&st, s);           // the array keeps the previous call's contents
    if (rc) return rc;
    return lola_prefill_chunked(&st, q, k, v, T, y, stream);
}

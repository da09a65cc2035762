"""B200 (sm_100a) LoLA hybrid-attention layer: Python binding of include/lola.h.

The binding only marshals arguments: it checks dtypes, shapes and devices of
torch tensors, passes their device pointers and the current CUDA stream to
the C ABI of liblola.so, and wraps device views of the state.  Every step of
the layer runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or fails to load, every entry point raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, byref, c_int, c_longlong, c_size_t, c_void_p, c_char_p

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblola.so")

DTYPE_F32, DTYPE_BF16 = 0, 1
_TORCH_DTYPE = {DTYPE_F32: torch.float32, DTYPE_BF16: torch.bfloat16}
ERRORS = {0: "OK", -1: "INVALID_ARG", -2: "BUF_TOO_SMALL", -3: "CUDA", -4: "TIMEOUT", -5: "UNSUPPORTED"}

# Every entry point of include/lola.h.
EXPORTS = ("lola_state_bytes", "lola_state_init", "lola_state_reset", "lola_state_free",
           "lola_prefill_chunked", "lola_decode_step", "lola_prefill_chunked_host",
           "lola_decode_step_host", "lola_state_export", "lola_profile_enable",
           "lola_profile_read", "lola_launch_count", "lola_prefill_once_noalloc", "lola_selftest_umma",
           "lola_set_read_options", "lola_sre_map", "lola_set_scorer", "lola_state_check",
           "lola_last_error_string")
KERNEL_CLASSES = ("phi", "scan", "output", "finalize", "decode", "sre_map", "scores")
READ_HIDE_STATE, READ_HIDE_SPARSE = 1, 2
SCORERS = ("sre", "kernel_sq", "kernel_abs", "kernel_ratio", "attn")   # LOLA_SCORE_* in this order


class LolaConfig(ctypes.Structure):
    _fields_ = [("B", c_int), ("Hq", c_int), ("Hkv", c_int), ("d", c_int), ("Dh", c_int),
                ("eta", c_int), ("lambda_", c_int), ("chunk", c_int), ("dtype", c_int),
                ("max_tokens", c_int)]


class LolaStateView(ctypes.Structure):
    _fields_ = [("t", c_longlong), ("n_cache", c_int), ("H", c_void_p), ("s", c_void_p),
                ("cache_k", c_void_p), ("cache_v", c_void_p), ("cache_phik", c_void_p),
                ("cache_pos", c_void_p), ("win_k", c_void_p), ("win_v", c_void_p),
                ("win_phik", c_void_p), ("trace_pos", c_void_p), ("trace_len", c_int),
                ("trace_stride", c_int), ("trace_t0", c_longlong), ("err_word", c_void_p)]


class LolaError(RuntimeError):
    pass


_lib = None


def lib() -> ctypes.CDLL:
    """Load liblola.so (raises if it is missing: there is no other implementation)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise LolaError(f"{LIB_PATH} is missing; build it with `python -m sparse_kv_caching_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp = c_void_p
    L.lola_state_bytes.argtypes = [POINTER(LolaConfig), POINTER(c_size_t)]
    L.lola_state_init.argtypes = [POINTER(LolaConfig), vp, vp, c_size_t, vp, POINTER(vp)]
    L.lola_state_reset.argtypes = [vp, vp]
    L.lola_state_free.argtypes = [vp]
    L.lola_prefill_chunked.argtypes = [vp, vp, vp, vp, c_int, vp, vp]
    L.lola_decode_step.argtypes = [vp, vp, vp, vp, vp, vp]
    L.lola_prefill_chunked_host.argtypes = [vp, vp, vp, vp, c_int, vp, vp]
    L.lola_decode_step_host.argtypes = [vp, vp, vp, vp, vp, vp]
    L.lola_state_export.argtypes = [vp, POINTER(LolaStateView)]
    L.lola_profile_enable.argtypes = [vp, c_int]
    L.lola_profile_read.argtypes = [vp, POINTER(ctypes.c_float), POINTER(c_longlong), c_int]
    L.lola_prefill_once_noalloc.argtypes = [POINTER(LolaConfig), vp, vp, vp, vp, c_int, vp, vp]
    L.lola_selftest_umma.argtypes = [c_int, vp, vp, vp, c_int, c_int, c_int, vp, vp]
    L.lola_set_read_options.argtypes = [vp, c_int, c_int]
    L.lola_sre_map.argtypes = [vp, vp, vp, c_int, vp, vp, vp]
    L.lola_set_scorer.argtypes = [vp, c_int]
    L.lola_state_check.argtypes = [vp, vp]
    L.lola_launch_count.argtypes = []
    L.lola_launch_count.restype = c_longlong
    L.lola_last_error_string.argtypes = []
    L.lola_last_error_string.restype = c_char_p
    for name in EXPORTS:
        if name not in ("lola_launch_count", "lola_last_error_string"):
            getattr(L, name).restype = c_int
    _lib = L
    return L


def _check(rc: int) -> None:
    if rc != 0:
        msg = lib().lola_last_error_string().decode()
        raise LolaError(f"LOLA_ERR_{ERRORS.get(rc, rc)}: {msg}")


def make_config(B, Hq, Hkv, d, Dh, eta, lam, chunk, dtype, max_tokens) -> LolaConfig:
    dt = {"f32": DTYPE_F32, "bf16": DTYPE_BF16}.get(dtype, dtype)
    return LolaConfig(B, Hq, Hkv, d, Dh, eta, lam, chunk, dt, max_tokens)


def state_bytes(cfg: LolaConfig) -> int:
    n = c_size_t()
    _check(lib().lola_state_bytes(byref(cfg), byref(n)))
    return n.value


def launch_count() -> int:
    """Kernels launched by liblola.so in this process."""
    return int(lib().lola_launch_count())


def prefill_once_noalloc(cfg: LolaConfig, W, q, k, v, y, stream=None):
    """One-shot prefill from an empty state using the library's built-in scratch array.

    For callers that cannot allocate device memory: nothing is allocated here
    or in the library; q, k, v, W and y are the caller's device tensors.
    Calls share the built-in array, so overlapping calls race.
    """
    for x in (W, q, k, v, y):
        if not (isinstance(x, torch.Tensor) and x.is_cuda and x.is_contiguous()):
            raise ValueError("W, q, k, v, y must be contiguous CUDA tensors")
    if y.dtype != torch.float32:
        raise ValueError("y must be float32")
    _check(lib().lola_prefill_once_noalloc(byref(cfg), c_void_p(W.data_ptr()), c_void_p(q.data_ptr()),
                                           c_void_p(k.data_ptr()), c_void_p(v.data_ptr()), q.shape[1],
                                           c_void_p(y.data_ptr()), _stream(stream)))
    return y


def _stream(stream=None) -> c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


class LolaLayer:
    """One LoLA attention layer state bound to a caller-owned device buffer.

    W: [Hkv, d, Dh] device tensor in the layer dtype (feature-map weights).
    """

    def __init__(self, cfg: LolaConfig, W: torch.Tensor, device="cuda", stream=None):
        self.cfg = cfg
        self.device = torch.device(device)
        self.dtype = _TORCH_DTYPE[cfg.dtype]
        self.D = 2 * cfg.Dh
        self.S = cfg.B * cfg.Hkv
        self._check_tensor(W, (cfg.Hkv, cfg.d, cfg.Dh), self.dtype, "W")
        self.nbytes = state_bytes(cfg)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=self.device)
        self._off = (-self.buf.data_ptr()) % 256
        self.handle = c_void_p()
        _check(lib().lola_state_init(byref(cfg), c_void_p(W.data_ptr()),
                                     c_void_p(self.buf.data_ptr() + self._off), self.nbytes,
                                     _stream(stream), byref(self.handle)))

    # -- argument checks (marshalling only) --------------------------------
    def _check_tensor(self, x, shape, dtype, name, device=None):
        dev = self.device if device is None else device
        if not isinstance(x, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if tuple(x.shape) != tuple(shape):
            raise ValueError(f"{name}: shape {tuple(x.shape)}, expected {tuple(shape)}")
        if x.dtype != dtype:
            raise ValueError(f"{name}: dtype {x.dtype}, expected {dtype}")
        if x.device.type != dev.type or (dev.type == "cuda" and dev.index is not None
                                           and x.device.index != dev.index):
            raise ValueError(f"{name}: on {x.device}, expected {dev}")
        if not x.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    def _shapes(self, T):
        c = self.cfg
        if T is None:
            return (c.B, c.Hq, c.d), (c.B, c.Hkv, c.d)
        return (c.B, T, c.Hq, c.d), (c.B, T, c.Hkv, c.d)

    # -- calls --------------------------------------------------------------
    def prefill(self, q, k, v, y=None, stream=None) -> torch.Tensor:
        """Chunkwise prefill of T tokens: q [B,T,Hq,d], k/v [B,T,Hkv,d] -> y [B,T,Hq,d] f32."""
        T = q.shape[1]
        sq, sk = self._shapes(T)
        self._check_tensor(q, sq, self.dtype, "q")
        self._check_tensor(k, sk, self.dtype, "k")
        self._check_tensor(v, sk, self.dtype, "v")
        if y is None:
            y = torch.empty(sq, dtype=torch.float32, device=self.device)
        self._check_tensor(y, sq, torch.float32, "y")
        _check(lib().lola_prefill_chunked(self.handle, c_void_p(q.data_ptr()), c_void_p(k.data_ptr()),
                                          c_void_p(v.data_ptr()), T, c_void_p(y.data_ptr()),
                                          _stream(stream)))
        return y

    def decode(self, q, k, v, y=None, stream=None) -> torch.Tensor:
        """One decode step: q [B,Hq,d], k/v [B,Hkv,d] -> y [B,Hq,d] f32."""
        sq, sk = self._shapes(None)
        self._check_tensor(q, sq, self.dtype, "q")
        self._check_tensor(k, sk, self.dtype, "k")
        self._check_tensor(v, sk, self.dtype, "v")
        if y is None:
            y = torch.empty(sq, dtype=torch.float32, device=self.device)
        self._check_tensor(y, sq, torch.float32, "y")
        _check(lib().lola_decode_step(self.handle, c_void_p(q.data_ptr()), c_void_p(k.data_ptr()),
                                      c_void_p(v.data_ptr()), c_void_p(y.data_ptr()), _stream(stream)))
        return y

    def prefill_host(self, q, k, v, y, stream=None) -> torch.Tensor:
        """prefill() with pinned host tensors; copies run inside the library call."""
        cpu = torch.device("cpu")
        T = q.shape[1]
        sq, sk = self._shapes(T)
        for x, s, dt, n in ((q, sq, self.dtype, "q"), (k, sk, self.dtype, "k"), (v, sk, self.dtype, "v"),
                            (y, sq, torch.float32, "y")):
            self._check_tensor(x, s, dt, n, device=cpu)
            if not x.is_pinned():
                raise ValueError(f"{n} must be pinned host memory")
        _check(lib().lola_prefill_chunked_host(self.handle, c_void_p(q.data_ptr()), c_void_p(k.data_ptr()),
                                               c_void_p(v.data_ptr()), T, c_void_p(y.data_ptr()),
                                               _stream(stream)))
        return y

    def decode_host(self, q, k, v, y, stream=None) -> torch.Tensor:
        cpu = torch.device("cpu")
        sq, sk = self._shapes(None)
        for x, s, dt, n in ((q, sq, self.dtype, "q"), (k, sk, self.dtype, "k"), (v, sk, self.dtype, "v"),
                            (y, sq, torch.float32, "y")):
            self._check_tensor(x, s, dt, n, device=cpu)
            if not x.is_pinned():
                raise ValueError(f"{n} must be pinned host memory")
        _check(lib().lola_decode_step_host(self.handle, c_void_p(q.data_ptr()), c_void_p(k.data_ptr()),
                                           c_void_p(v.data_ptr()), c_void_p(y.data_ptr()), _stream(stream)))
        return y

    def set_read_options(self, read_mask: int = 0, decode_update_first: bool = False) -> None:
        """Hide memory branches from later reads (READ_HIDE_* bits); update-first decode order."""
        _check(lib().lola_set_read_options(self.handle, int(read_mask), 1 if decode_update_first else 0))

    def set_scorer(self, scorer) -> None:
        """Scoring rule (a name from SCORERS or its LOLA_SCORE_* number); only before the first token."""
        code = SCORERS.index(scorer) if isinstance(scorer, str) else int(scorer)
        _check(lib().lola_set_scorer(self.handle, code))

    def sre_map(self, k, v, sre=None, rel=None, stream=None):
        """SRE of every folded pair at each state time of the last prefill call, and its change
        since first write: k/v [B,T,Hkv,d] (every position so far) -> sre, rel [B,Hkv,n+1,T] f32."""
        c = self.cfg
        T = k.shape[1]
        _, sk = self._shapes(T)
        self._check_tensor(k, sk, self.dtype, "k")
        self._check_tensor(v, sk, self.dtype, "v")
        v_ = LolaStateView()
        _check(lib().lola_state_export(self.handle, byref(v_)))
        shape = (c.B, c.Hkv, max(v_.trace_len, 1), T)
        if sre is None:
            sre = torch.empty(shape, dtype=torch.float32, device=self.device)
        if rel is None:
            rel = torch.empty(shape, dtype=torch.float32, device=self.device)
        self._check_tensor(sre, shape, torch.float32, "sre")
        self._check_tensor(rel, shape, torch.float32, "rel")
        _check(lib().lola_sre_map(self.handle, c_void_p(k.data_ptr()), c_void_p(v.data_ptr()), T,
                                  c_void_p(sre.data_ptr()), c_void_p(rel.data_ptr()), _stream(stream)))
        return sre, rel

    def profile(self, on: bool = True) -> None:
        """Bracket every kernel launch of this layer with CUDA events (tracing aid)."""
        _check(lib().lola_profile_enable(self.handle, 1 if on else 0))

    def profile_read(self) -> dict:
        """{class: (ms, launches)} accumulated since the last read (waits for the events)."""
        n = len(KERNEL_CLASSES)
        ms = (ctypes.c_float * n)()
        cnt = (c_longlong * n)()
        _check(lib().lola_profile_read(self.handle, ms, cnt, n))
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_CLASSES)}

    def check(self, stream=None) -> None:
        """Sync point: wait for the stream and raise LolaError (LOLA_ERR_TIMEOUT) if a bounded
        device-side wait of this state gave up since the last reset."""
        _check(lib().lola_state_check(self.handle, _stream(stream)))

    def reset(self, stream=None) -> None:
        _check(lib().lola_state_reset(self.handle, _stream(stream)))

    # -- state views ----------------------------------------------------------
    def _view(self, ptr, shape, dtype):
        n = 1
        for x in shape:
            n *= x
        esize = torch.empty(0, dtype=dtype).element_size()
        off = ptr - self.buf.data_ptr()
        assert 0 <= off and off + n * esize <= self.buf.numel()
        return self.buf[off:off + n * esize].view(dtype).view(*shape)

    def export(self) -> dict:
        """Device views (no copy) of the memories and of the last prefill's cache trace."""
        v = LolaStateView()
        _check(lib().lola_state_export(self.handle, byref(v)))
        c, S, D = self.cfg, self.S, self.D
        out = dict(t=v.t, n_cache=v.n_cache, trace_len=v.trace_len, trace_t0=v.trace_t0,
                   H=self._view(v.H, (S, D, c.d), torch.float32),
                   s=self._view(v.s, (S, D), torch.float32),
                   cache_k=self._view(v.cache_k, (S, c.lambda_, c.d), self.dtype),
                   cache_v=self._view(v.cache_v, (S, c.lambda_, c.d), self.dtype),
                   cache_phik=self._view(v.cache_phik, (S, c.lambda_, D), torch.float32),
                   cache_pos=self._view(v.cache_pos, (S, c.lambda_), torch.int32),
                   win_k=self._view(v.win_k, (S, c.eta, c.d), self.dtype),
                   win_v=self._view(v.win_v, (S, c.eta, c.d), self.dtype),
                   win_phik=self._view(v.win_phik, (S, c.eta, D), torch.float32),
                   err_word=self._view(v.err_word, (1,), torch.int32))
        if v.trace_len > 0 and c.lambda_ > 0:
            stride = v.trace_stride
            full = self._view(v.trace_pos, (S, stride), torch.int32)
            out["trace_pos"] = full[:, :v.trace_len * c.lambda_].reshape(S, v.trace_len, c.lambda_)
        return out

    def close(self) -> None:
        if self.handle:
            lib().lola_state_free(self.handle)
            self.handle = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

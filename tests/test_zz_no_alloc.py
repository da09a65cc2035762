"""The allocation-free one-shot prefill entry point (lola_prefill_once_noalloc).

Some callers cannot call cudaMalloc (for example a plugin that only receives
input and output pointers from its host application).  For them the library
offers a prefill whose state and scratch live in an array built into the
library instead of a caller buffer.  This file checks, through the C ABI,
that two calls in a row give the same output as the regular entry point
(lola_prefill_chunked on a fresh state), and that a configuration too large
for the built-in array is refused.  It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import sparse_kv_caching_b200 as lola
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _inputs(w):
    dev = P.to_device(w, synth.full_arrays(w))
    return dev["q"][:, :w.T].contiguous(), dev["k"][:, :w.T].contiguous(), dev["v"][:, :w.T].contiguous(), dev["W"]


def _cfg(w):
    return lola.make_config(w.B, w.Hq, w.Hkv, w.d, w.Dh, w.eta, w.lam, w.chunk, w.dtype, w.T)


def _regular(w, q, k, v, W):
    layer = P.make_layer(w, W, max_tokens=w.T)
    y = layer.prefill(q, k, v)
    torch.cuda.synchronize()
    return y


def _noalloc(w, q, k, v, W):
    y = torch.empty((w.B, w.T, w.Hq, w.d), dtype=torch.float32, device="cuda")
    L = lola.lib()
    rc = L.lola_prefill_once_noalloc(ctypes.byref(_cfg(w)), ctypes.c_void_p(W.data_ptr()),
                                     ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                     ctypes.c_void_p(v.data_ptr()), w.T, ctypes.c_void_p(y.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, L.lola_last_error_string().decode()
    torch.cuda.synchronize()
    return y


def test_noalloc_matches_regular_entry_point_twice():
    """Both entry points run the same kernels on the same inputs, so the outputs are
    bit-identical; a leak of the previous call's contents would show up here."""
    wa = P.small_workload(2, B=1, Hkv=2, Hq=8, T=768, eta=128, lam=96, chunk=64)
    wb = P.small_workload(5, B=2, Hkv=2, Hq=4, T=512, eta=64, lam=80, chunk=64, wid=55)
    ia, ib = _inputs(wa), _inputs(wb)
    ref_a, ref_b = _regular(wa, *ia), _regular(wb, *ib)
    # two calls in a row; the second must not see anything the first left behind
    ya = _noalloc(wa, *ia)
    yb = _noalloc(wb, *ib)
    assert torch.equal(ya, ref_a)
    assert torch.equal(yb, ref_b)
    ya2 = _noalloc(wa, *ia)
    assert torch.equal(ya2, ref_a)


def test_noalloc_at_the_largest_documented_shape():
    """The 8B-shaped 4096-token prefill with B = 1 (documented to fit the built-in
    array): bit-identical to the regular entry point, twice in a row."""
    w = synth.workload(2)
    inp = _inputs(w)
    ref = _regular(w, *inp)
    for _ in range(2):
        assert torch.equal(_noalloc(w, *inp), ref)


def test_noalloc_refuses_configurations_beyond_its_array():
    w = synth.workload(3)                     # 32 streams x 16K tokens: far beyond 64 MiB
    cfg = _cfg(w)
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    L = lola.lib()
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = L.lola_prefill_once_noalloc(ctypes.byref(cfg), p, p, p, p, w.T, p,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -2
    assert "built-in array" in L.lola_last_error_string().decode()

"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
and rejects bad configurations without touching a GPU."""
import os
import re
import subprocess

import pytest

import sparse_kv_caching_b200 as lola
from sparse_kv_caching_b200 import build as lbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    lbuild.build()
    return lola.lib()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^\s*(?:int|long long|const char\*)\s+(lola_\w+)\s*\(", txt, re.M)
    return names


def test_every_declared_symbol_is_exported(L):
    decl = _declared()
    assert len(decl) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", lbuild.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(lola_\w+)", out))
    missing = [n for n in decl if n not in exported]
    assert not missing, missing
    for n in decl:
        assert hasattr(L, n)
    assert set(lola.EXPORTS) <= set(decl)


def _cfg(**kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, Dh=64, eta=256, lam=256, chunk=64, dtype="bf16", max_tokens=4096)
    base.update(kw)
    return lola.make_config(**base)


def test_state_bytes_valid_and_monotone(L):
    n1 = lola.state_bytes(_cfg())
    n2 = lola.state_bytes(_cfg(max_tokens=8192))
    n3 = lola.state_bytes(_cfg(B=2))
    assert 0 < n1 < n2 and n1 < n3
    assert n1 % 256 == 0


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), "UNSUPPORTED"),
    (dict(Dh=48), "UNSUPPORTED"),
    (dict(Hq=30), "INVALID_ARG"),
    (dict(Hq=80, Hkv=8), "UNSUPPORTED"),
    (dict(eta=0), "INVALID_ARG"),
    (dict(lam=4096), "UNSUPPORTED"),
    (dict(chunk=0), "UNSUPPORTED"),
    (dict(max_tokens=100), "INVALID_ARG"),
    (dict(dtype=7), "INVALID_ARG"),
])
def test_bad_configs_rejected(L, kw, code):
    with pytest.raises(lola.LolaError, match=code):
        lola.state_bytes(_cfg(**kw))


def test_error_string_is_set(L):
    with pytest.raises(lola.LolaError) as e:
        lola.state_bytes(_cfg(d=96))
    assert "d=96" in str(e.value)


def test_null_arguments_rejected(L):
    import ctypes
    assert L.lola_state_bytes(None, None) == -1
    assert L.lola_prefill_chunked(None, None, None, None, 64, None, None) == -1
    assert L.lola_decode_step(None, None, None, None, None, None) == -1
    assert L.lola_state_export(None, None) == -1
    assert L.lola_state_free(None) == 0
    assert L.lola_set_read_options(None, 0, 0) == -1
    assert L.lola_set_scorer(None, 0) == -1
    assert L.lola_sre_map(None, None, None, 64, None, None, None) == -1
    n = ctypes.c_size_t()
    assert L.lola_state_bytes(ctypes.byref(_cfg()), ctypes.byref(n)) == 0 and n.value > 0


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="passes fake pointers; only meaningful where no GPU can run the call")
def test_noalloc_size_check_without_a_gpu(L):
    """The one-shot entry point's size check runs before any CUDA call: the 8B-shaped
    4096-token prefill with B = 1 passes it (and then fails only for want of a device),
    the same shape with B = 2 is refused with LOLA_ERR_BUF_TOO_SMALL."""
    import ctypes
    buf = ctypes.create_string_buffer(64)
    p = ctypes.c_void_p(ctypes.addressof(buf))
    rc = L.lola_prefill_once_noalloc(ctypes.byref(_cfg()), p, p, p, p, 4096, p, None)
    assert rc == -3, L.lola_last_error_string().decode()        # LOLA_ERR_CUDA: no device here
    rc = L.lola_prefill_once_noalloc(ctypes.byref(_cfg(B=2)), p, p, p, p, 4096, p, None)
    assert rc == -2
    assert "built-in array" in L.lola_last_error_string().decode()

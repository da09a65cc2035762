"""Parity of the read options, the scoring rules and the SRE map (through the C ABI)
with the CPU oracle.

Read-branch masks (LoLA notes §4.8, App. I, Table 12) on the prefill output
kernels (bf16 tensor-core path and fp32 path) and on decode; update-first
decode (the token equations of notes §2.4 read literally); the alternative
scoring rules of the scoring ablation (notes §4.5, Table 4; App. F) in
prefill, across calls and in decode; the stored-pair SRE map and relative SRE
(notes §4.4, Fig. 3, Fig. 10, Eq. 26) over the prefill's snapshots.  Every
output element of the small cases is compared.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import sre_map as oracle_sre_map
from tests import parity as P

pytestmark = pytest.mark.gpu

MAP_TOL = 1e-4        # fp32 map against the fp64 oracle: max |x - r| / max |sre_r| per stream


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _prefill(w, layer, dev, cuts):
    ys, traces = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        ys.append(layer.prefill(dev["q"][:, a:b].contiguous(), dev["k"][:, a:b].contiguous(),
                                dev["v"][:, a:b].contiguous()))
        torch.cuda.synchronize()
        ex = layer.export()
        traces.append(ex["trace_pos"].cpu().numpy().copy() if w.lam > 0 else None)
    return torch.cat(ys, dim=1), traces


def _oracle_follow(w, b, g, cuts, traces, yg, mask=0, scorer="sre"):
    """Oracle stream for (b, g) stepped through the library's chunks and cache trace."""
    st = P.oracle_stream(w, g)
    st.read_mask = mask
    st.scorer = scorer
    a = synth.stream_arrays(w, b, g)
    err = 0.0
    for ci, (t_lo, t_hi) in enumerate(zip(cuts[:-1], cuts[1:])):
        nch = (t_hi - t_lo) // w.chunk
        tr = traces[ci][b * w.Hkv + g] if w.lam > 0 else np.full((nch + 1, 0), -1)
        e, chain = P.check_prefill_stream(w, st, a, t_lo, t_hi, tr, yg[:, t_lo:t_hi])
        assert chain.hard == 0 and chain.set_mismatch == 0, (chain.hard, chain.set_mismatch)
        err = max(err, chain.abs_err / max(chain.y_max, 1e-30))
    return st, a, err


MASK_CASES = {
    "bf16-d128": dict(base=2, B=1, Hkv=2, Hq=8, T=512, eta=64, lam=64, chunk=64),
    "f32-d64": dict(base=5, B=1, Hkv=2, Hq=4, T=480, eta=72, lam=80, chunk=48, dtype="f32"),
}


@pytest.mark.parametrize("mask", [1, 2, 3])
@pytest.mark.parametrize("case", list(MASK_CASES))
def test_read_mask_prefill(case, mask):
    kw = dict(MASK_CASES[case])
    w = P.small_workload(kw.pop("base"), **kw)
    dev = P.to_device(w, synth.full_arrays(w))
    masked = P.make_layer(w, dev["W"])
    masked.set_read_options(mask)
    plain = P.make_layer(w, dev["W"])
    cuts = [0, w.T]
    y, traces = _prefill(w, masked, dev, cuts)
    _prefill(w, plain, dev, cuts)
    em, ep = masked.export(), plain.export()
    for key in ("H", "s", "cache_pos", "cache_k", "cache_v", "win_k", "win_v"):
        assert torch.equal(em[key], ep[key]), key           # the memories ignore the mask
    worst = 0.0
    for b in range(w.B):
        for g in range(w.Hkv):
            _, _, e = _oracle_follow(w, b, g, cuts, traces, P.gpu_stream_y(y, w, b, g), mask)
            worst = max(worst, e)
    assert worst <= P.TOL[w.dtype], worst


def _decode_variant(w, T_pre, steps, streams, mask, update_first, scorer="sre", cuts=None):
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"], max_tokens=max(T_pre, w.chunk))
    layer.set_read_options(mask, update_first)
    layer.set_scorer(scorer)
    oracles = {}
    if T_pre:
        cuts = cuts or [0, T_pre]
        y0, traces = _prefill(w, layer, dev, cuts)
        for (b, g) in streams:
            st, a, e = _oracle_follow(w, b, g, cuts, traces, P.gpu_stream_y(y0, w, b, g), mask, scorer)
            assert e <= P.TOL[w.dtype]
            oracles[(b, g)] = (st, a)
    else:
        for (b, g) in streams:
            st = P.oracle_stream(w, g)
            st.read_mask = mask
            st.scorer = scorer
            oracles[(b, g)] = (st, synth.stream_arrays(w, b, g))
    worst, ties = 0.0, 0
    for i in range(steps):
        t = T_pre + i
        yd = layer.decode(dev["q"][:, t].contiguous(), dev["k"][:, t].contiguous(), dev["v"][:, t].contiguous())
        torch.cuda.synchronize()
        ex = layer.export()
        cpos = ex["cache_pos"].cpu().numpy()
        ydn = yd.double().cpu().numpy()
        for (b, g), (st, a) in oracles.items():
            chain = P.ChainCheck(w.lam)
            chain.expected = sorted(int(p) for p in cpos[b * w.Hkv + g] if p >= 0)
            yo = st.decode(a["q"][:, t], a["k"][t], a["v"][t], chain.choose, update_first=update_first)
            assert chain.hard == 0 and sorted(st.cache) == chain.expected, (i, b, g)
            ties += chain.ties
            worst = max(worst, P.max_rel(ydn[b, g * w.Gq:(g + 1) * w.Gq], yo))
    ex = layer.export()
    for (b, g), (st, a) in oracles.items():
        S = b * w.Hkv + g
        if st.folded:
            assert P.max_rel(ex["H"][S].double().cpu().numpy(), st.H) <= P.TOL[w.dtype]
            assert P.max_rel(ex["s"][S].double().cpu().numpy(), st.s) <= P.TOL[w.dtype]
    assert worst <= P.TOL[w.dtype], worst
    return worst


@pytest.mark.parametrize("mask,update_first", [(0, True), (1, False), (2, False), (3, True), (2, True)])
def test_decode_options_after_prefill(mask, update_first):
    w = P.small_workload(4, B=2, Hkv=2, Hq=8, T=512, eta=64, lam=48, chunk=64, decode_steps=96)
    _decode_variant(w, 512, 96, [(0, 0), (1, 1)], mask, update_first)


@pytest.mark.parametrize("mask", [0, 3])
def test_update_first_decode_from_empty_state(mask):
    """Window filling, cache filling, then scoring, every step updating before the read."""
    w = P.small_workload(1, T=64, eta=16, lam=12, chunk=64, decode_steps=160)
    _decode_variant(w, 0, 160, [(0, 0)], mask, True)


SCORE_CASES = {
    # GQA 4, several key tiles; two calls so window scores carry across calls
    "bf16-d128": (dict(base=2, B=1, Hkv=2, Hq=8, T=768, eta=128, lam=96, chunk=64), [320]),
    # chunk 48, eta not a multiple of it, Gq = 2, fp32
    "f32-d64": (dict(base=5, B=1, Hkv=2, Hq=4, T=480, eta=72, lam=80, chunk=48, dtype="f32"), None),
}


@pytest.mark.parametrize("rule", ["kernel_sq", "kernel_abs", "kernel_ratio", "attn"])
@pytest.mark.parametrize("case", list(SCORE_CASES))
def test_alternative_scorer_prefill(case, rule):
    kw, splits = SCORE_CASES[case]
    kw = dict(kw)
    w = P.small_workload(kw.pop("base"), **kw)
    cuts = [0] + (splits or []) + [w.T]
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"], max_tokens=max(b - a for a, b in zip(cuts[:-1], cuts[1:])))
    layer.set_scorer(rule)
    y, traces = _prefill(w, layer, dev, cuts)
    ex = layer.export()
    worst = 0.0
    for b in range(w.B):
        for g in range(w.Hkv):
            st, _, e = _oracle_follow(w, b, g, cuts, traces, P.gpu_stream_y(y, w, b, g), 0, rule)
            worst = max(worst, e)
            S = b * w.Hkv + g
            assert sorted(int(p) for p in ex["cache_pos"][S].cpu().numpy() if p >= 0) == sorted(st.cache)
            if st.folded:
                assert P.max_rel(ex["H"][S].double().cpu().numpy(), st.H) <= P.TOL[w.dtype]
    assert worst <= P.TOL[w.dtype], worst


@pytest.mark.parametrize("rule,update_first", [("kernel_sq", False), ("kernel_ratio", True), ("attn", False),
                                               ("kernel_abs", True)])
def test_alternative_scorer_decode_after_prefill(rule, update_first):
    w = P.small_workload(4, B=2, Hkv=2, Hq=8, T=512, eta=64, lam=48, chunk=64, decode_steps=80)
    _decode_variant(w, 512, 80, [(0, 0), (1, 1)], 0, update_first, rule, cuts=[0, 192, 512])


@pytest.mark.parametrize("rule", ["kernel_sq", "attn"])
def test_alternative_scorer_decode_from_empty_state(rule):
    w = P.small_workload(1, T=64, eta=16, lam=12, chunk=64, decode_steps=120)
    _decode_variant(w, 0, 120, [(0, 0)], 0, False, rule)


def test_scorer_change_after_tokens_is_an_error():
    import sparse_kv_caching_b200 as lola
    w = P.small_workload(2, B=1, Hkv=2, Hq=4, T=128, eta=64, lam=64, chunk=64)
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"])
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.set_scorer(7)
    layer.set_scorer("attn")
    layer.prefill(dev["q"], dev["k"], dev["v"])
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.set_scorer("sre")
    layer.reset()
    layer.set_scorer("sre")
    torch.cuda.synchronize()


def _check_map(w, cuts):
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"], max_tokens=max(b - a for a, b in zip(cuts[:-1], cuts[1:])))
    y, traces = _prefill(w, layer, dev, cuts)
    sre, rel = layer.sre_map(dev["k"], dev["v"])
    torch.cuda.synchronize()
    n_last = (cuts[-1] - cuts[-2]) // w.chunk
    assert sre.shape == (w.B, w.Hkv, n_last + 1, w.T)
    first_block = (cuts[-2]) // w.chunk
    worst = 0.0
    members = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            st, _, e = _oracle_follow(w, b, g, cuts, traces, P.gpu_stream_y(y, w, b, g))
            assert e <= P.TOL[w.dtype]
            so, ro = oracle_sre_map(st, first_block)
            sg = sre[b, g].double().cpu().numpy()
            rg = rel[b, g].double().cpu().numpy()
            # membership (integer work) is exact: every pair outside the state is 0
            nfold = [r["folded_before"] for r in st.log[first_block:]] + [len(st.folded)]
            M = np.zeros_like(so, dtype=bool)
            for c, nf in enumerate(nfold):
                M[c, st.folded[:nf]] = True
            assert np.all(sg[~M] == 0) and np.all(rg[~M] == 0)
            members += int(M.sum())
            scale = max(np.abs(so).max(), 1e-30)
            worst = max(worst, np.abs(sg - so).max() / scale, np.abs(rg - ro).max() / scale)
    assert worst <= MAP_TOL, worst
    return members


MAP_CASES = {
    # GQA, several position tiles per stream, two sequences
    "bf16-d128": (dict(base=2, B=2, Hkv=2, Hq=8, T=768, eta=128, lam=96, chunk=64), None),
    # ragged last tile (T = 624 is not a multiple of 64), chunk 48, fp32
    "f32-d64-ragged": (dict(base=5, B=1, Hkv=2, Hq=4, T=624, eta=72, lam=100, chunk=48, dtype="f32"), None),
    # lambda = 0: every leaving pair is folded
    "lambda0": (dict(base=2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=0, chunk=64), None),
    "d128-Dh32": (dict(base=2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=64, chunk=64, Dh=32), None),
    # the map covers the last of two calls; pairs folded earlier are held from its first row
    "split": (dict(base=2, B=1, Hkv=2, Hq=8, T=768, eta=128, lam=96, chunk=64), [320]),
}


@pytest.mark.parametrize("name", list(MAP_CASES))
def test_sre_map(name):
    kw, splits = MAP_CASES[name]
    kw = dict(kw)
    w = P.small_workload(kw.pop("base"), **kw)
    cuts = [0] + (splits or []) + [w.T]
    assert _check_map(w, cuts) > 0


def test_sre_map_and_options_argument_errors():
    import sparse_kv_caching_b200 as lola
    w = P.small_workload(2, B=1, Hkv=2, Hq=4, T=256, eta=64, lam=64, chunk=64, decode_steps=2)
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"], max_tokens=256)
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.set_read_options(4)
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.sre_map(dev["k"][:, :256].contiguous(), dev["v"][:, :256].contiguous())    # no prefill yet
    layer.prefill(dev["q"][:, :256].contiguous(), dev["k"][:, :256].contiguous(), dev["v"][:, :256].contiguous())
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.sre_map(dev["k"][:, :192].contiguous(), dev["v"][:, :192].contiguous())    # T mismatch
    layer.sre_map(dev["k"][:, :256].contiguous(), dev["v"][:, :256].contiguous())
    layer.decode(dev["q"][:, 256].contiguous(), dev["k"][:, 256].contiguous(), dev["v"][:, 256].contiguous())
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.sre_map(dev["k"][:, :257].contiguous(), dev["v"][:, :257].contiguous())    # decode followed
    torch.cuda.synchronize()


# ---- the 8B-shaped 4096-token workload that bench.py times, on sampled streams ----

def _fullsize_rows(w, rng):
    rows = np.zeros((w.Gq, w.T), bool)
    rows[:, rng.choice(w.T, size=96, replace=False)] = True
    rows[:, -w.chunk:] = True
    return rows


def _fullsize_variant(mask=0, scorer="sre", with_map=False):
    w = synth.workload(2)
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"], max_tokens=w.T)
    layer.set_read_options(mask)
    layer.set_scorer(scorer)
    y = layer.prefill(dev["q"], dev["k"], dev["v"])
    torch.cuda.synchronize()
    ex = layer.export()
    tr = ex["trace_pos"].cpu().numpy()
    sre = rel = None
    if with_map:
        sre, rel = layer.sre_map(dev["k"], dev["v"])
        torch.cuda.synchronize()
    rng = np.random.default_rng(17)
    for (b, g) in [(0, 0), (w.B - 1, w.Hkv - 1)]:
        st = P.oracle_stream(w, g)
        st.read_mask = mask
        st.scorer = scorer
        a = synth.stream_arrays(w, b, g)
        e, chain = P.check_prefill_stream(w, st, a, 0, w.T, tr[b * w.Hkv + g], P.gpu_stream_y(y, w, b, g),
                                          _fullsize_rows(w, rng))
        assert chain.hard == 0 and chain.set_mismatch == 0, (b, g, chain.hard, chain.set_mismatch)
        assert e <= P.TOL[w.dtype], (b, g, e)
        S = b * w.Hkv + g
        assert P.max_rel(ex["H"][S].double().cpu().numpy(), st.H) <= P.TOL[w.dtype]
        if with_map:
            so, ro = oracle_sre_map(st)
            sg = sre[b, g].double().cpu().numpy()
            rg = rel[b, g].double().cpu().numpy()
            nfold = [r["folded_before"] for r in st.log] + [len(st.folded)]
            M = np.zeros_like(so, dtype=bool)
            for c, nf in enumerate(nfold):
                M[c, st.folded[:nf]] = True
            assert np.all(sg[~M] == 0) and np.all(rg[~M] == 0)
            scale = np.abs(so).max()
            assert np.abs(sg - so).max() / scale <= MAP_TOL
            assert np.abs(rg - ro).max() / scale <= MAP_TOL


@pytest.mark.slow
@pytest.mark.parametrize("mask", [1, 2])
def test_fullsize_read_mask_sampled(mask):
    _fullsize_variant(mask=mask)


@pytest.mark.slow
@pytest.mark.parametrize("rule", ["kernel_sq", "kernel_ratio"])
def test_fullsize_alternative_scorer_sampled(rule):
    _fullsize_variant(scorer=rule)


@pytest.mark.slow
def test_fullsize_sre_map_sampled():
    """The map of the whole 4096-token prefill (65 state times), two streams element by element."""
    _fullsize_variant(with_map=True)


@pytest.mark.slow
def test_fullsize_update_first_decode_sampled():
    """Update-first decode after the 8B-shaped decode workload's 4096-token prefill."""
    w = synth.workload(4)
    _decode_variant(w, w.T, 48, [(0, 0), (w.B - 1, w.Hkv - 1)], 0, True)


def test_scorer_host_prefill_matches_device():
    """The pipelined host-buffer prefill (four chunk-aligned calls) carries the window
    scores between its calls exactly as one device call does."""
    w = P.small_workload(2, B=2, Hkv=2, Hq=4, T=640, eta=64, lam=96, chunk=64)
    dev = P.to_device(w, synth.full_arrays(w))
    l1 = P.make_layer(w, dev["W"])
    l2 = P.make_layer(w, dev["W"])
    for layer in (l1, l2):
        layer.set_scorer("kernel_abs")
    y1 = l1.prefill(dev["q"], dev["k"], dev["v"])
    hq, hk, hv = (dev[x].cpu().pin_memory() for x in ("q", "k", "v"))
    hy = torch.full(y1.shape, float("nan"), dtype=torch.float32).pin_memory()
    l2.prefill_host(hq, hk, hv, hy)
    torch.cuda.synchronize()
    e1, e2 = l1.export(), l2.export()
    assert torch.equal(e1["cache_pos"], e2["cache_pos"]) and torch.equal(e1["H"], e2["H"])
    assert torch.allclose(hy, y1.cpu(), rtol=0, atol=1e-6 * float(y1.abs().max()))


def test_sre_map_after_alternative_scorer():
    """The map reads the snapshots whatever rule chose the cache."""
    w = P.small_workload(2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=64, chunk=64)
    dev = P.to_device(w, synth.full_arrays(w))
    layer = P.make_layer(w, dev["W"])
    layer.set_scorer("attn")
    y, traces = _prefill(w, layer, dev, [0, w.T])
    sre, rel = layer.sre_map(dev["k"], dev["v"])
    torch.cuda.synchronize()
    for g in range(w.Hkv):
        st, _, e = _oracle_follow(w, 0, g, [0, w.T], traces, P.gpu_stream_y(y, w, 0, g), 0, "attn")
        so, ro = oracle_sre_map(st)
        scale = np.abs(so).max()
        assert np.abs(sre[0, g].double().cpu().numpy() - so).max() / scale <= MAP_TOL
        assert np.abs(rel[0, g].double().cpu().numpy() - ro).max() / scale <= MAP_TOL

"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Small cases compare every output element, the final (H, s) and the retained
cache set of every chunk; full-size workloads compare sampled streams and
sampled query rows in the launch configuration bench.py times.
"""
import numpy as np
import pytest
import torch

import synth
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _run_small(w: synth.Workload, splits=None):
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    layer = P.make_layer(w, dev["W"], max_tokens=w.T)
    T = w.T
    cuts = [0] + (splits or []) + [T]
    ys = []
    traces = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        ys.append(layer.prefill(dev["q"][:, a:b].contiguous(), dev["k"][:, a:b].contiguous(),
                                dev["v"][:, a:b].contiguous()))
        torch.cuda.synchronize()
        ex = layer.export()
        traces.append(ex["trace_pos"].cpu().numpy().copy() if w.lam > 0 else None)
    y = torch.cat(ys, dim=1)
    ex = layer.export()
    torch.cuda.synchronize()
    return layer, y, ex, traces, cuts


def _check_small(w, splits=None, rows_all=True):
    layer, y, ex, traces, cuts = _run_small(w, splits)
    tol = P.TOL[w.dtype]
    worst = dict(y=0.0, H=0.0, s=0.0)
    ties = hard = setmis = 0
    abs_err, y_max = 0.0, 0.0              # max |x - r| / max |r| over the whole y tensor
    for b in range(w.B):
        for g in range(w.Hkv):
            st = P.oracle_stream(w, g)
            a = synth.stream_arrays(w, b, g)
            yg = P.gpu_stream_y(y, w, b, g)
            for ci, (t_lo, t_hi) in enumerate(zip(cuts[:-1], cuts[1:])):
                nchunks = (t_hi - t_lo) // w.chunk
                tr = (traces[ci][b * w.Hkv + g] if w.lam > 0
                      else np.full((nchunks + 1, 0), -1))
                e, chain = P.check_prefill_stream(w, st, a, t_lo, t_hi, tr, yg[:, t_lo:t_hi])
                abs_err = max(abs_err, chain.abs_err)
                y_max = max(y_max, chain.y_max)
                ties += chain.ties
                hard += chain.hard
                setmis += chain.set_mismatch
            S = b * w.Hkv + g
            worst["H"] = max(worst["H"], P.max_rel(ex["H"][S].double().cpu().numpy(), st.H) if st.folded else 0.0)
            worst["s"] = max(worst["s"], P.max_rel(ex["s"][S].double().cpu().numpy(), st.s) if st.folded else 0.0)
            if w.lam > 0:
                got = sorted(int(p) for p in ex["cache_pos"][S].cpu().numpy() if p >= 0)
                assert got == sorted(st.cache)
    worst["y"] = abs_err / y_max
    assert hard == 0 and setmis == 0, (hard, setmis, ties)
    assert worst["y"] <= tol and worst["H"] <= tol and worst["s"] <= tol, worst
    return worst, ties


def test_tiny_f32_workload_full():
    """Workload 1 (tiny single head, fp32) compared element by element."""
    worst, ties = _check_small(synth.workload(1))
    assert worst["y"] < 1e-4


SMALL = {
    # several SRE tiles, lambda off the tile grid, two sequences
    "gqa4-d128": dict(base=2, B=2, Hkv=2, Hq=8, T=768, eta=128, lam=96, chunk=64),
    # chunk not a multiple of 32, eta not a multiple of chunk, Gq = 1
    "ragged-d64": dict(base=5, B=1, Hkv=4, Hq=4, T=624, eta=72, lam=100, chunk=48),
    # lambda = 0: window + linear hybrid
    "lambda0": dict(base=2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=0, chunk=64),
    # eta + lambda >= T: nothing folded, exact causal softmax
    "nofold": dict(base=2, B=1, Hkv=2, Hq=4, T=256, eta=128, lam=160, chunk=32),
    # candidate count above one SRE tile (n = lambda + C = 428)
    "many-cands": dict(base=3, B=1, Hkv=2, Hq=8, T=1024, eta=256, lam=300, chunk=128, n_needles=4),
    # mixed feature/head widths
    "d64-Dh64": dict(base=5, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=64, chunk=64, Dh=64),
    "d64-gqa4": dict(base=5, B=1, Hkv=2, Hq=8, T=512, eta=64, lam=64, chunk=64),
    "d128-Dh32": dict(base=2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=64, chunk=64, Dh=32),
    # fp32 inputs at the 8B head shape
    "f32-d128": dict(base=2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=64, chunk=64, dtype="f32"),
    # every pair identical: every selection is an exact tie, broken by position
    "all-equal-pairs": dict(base=2, B=1, Hkv=2, Hq=4, T=512, eta=64, lam=64, chunk=64, dup_every=1),
    # a third of the pairs identical, among distinct ones
    "dup-thirds": dict(base=2, B=1, Hkv=2, Hq=4, T=768, eta=64, lam=96, chunk=64, dup_every=3),
    # lambda + C beyond a shared-memory row pool: candidate rows streamed from global memory
    "rows-global-d128": dict(base=3, B=1, Hkv=2, Hq=4, T=1024, eta=64, lam=480, chunk=64),
    "rows-global-d64": dict(base=5, B=1, Hkv=2, Hq=4, T=1280, eta=64, lam=768, chunk=64),
    "rows-global-f32": dict(base=2, B=1, Hkv=2, Hq=4, T=1024, eta=64, lam=480, chunk=64, dtype="f32"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(name):
    kw = dict(SMALL[name])
    base = kw.pop("base")
    w = P.small_workload(base, **kw)
    _check_small(w)


def test_split_calls_match_single_call():
    w = P.small_workload(2, B=1, Hkv=2, Hq=8, T=768, eta=128, lam=96, chunk=64)
    _, y1, ex1, _, _ = _run_small(w)
    _, y2, ex2, _, _ = _run_small(w, splits=[128, 448])
    assert torch.equal(y1, y2)
    assert torch.equal(ex1["H"], ex2["H"]) and torch.equal(ex1["s"], ex2["s"])
    assert torch.equal(ex1["cache_pos"], ex2["cache_pos"])
    # and the split run matches the oracle
    _check_small(w, splits=[128, 448])


def test_segmented_call_matches_unsegmented_calls():
    """A call of >= 32 chunks runs its chain in segments with the outputs overlapped;
    it must equal, bit for bit, calls of one segment each (which do not split)."""
    w = P.small_workload(2, B=1, Hkv=2, Hq=4, T=2048, eta=64, lam=64, chunk=64)
    _, y1, ex1, _, _ = _run_small(w)
    _, y2, ex2, _, _ = _run_small(w, splits=[512, 1024, 1536])
    assert torch.equal(y1, y2)
    assert torch.equal(ex1["H"], ex2["H"]) and torch.equal(ex1["s"], ex2["s"])
    assert torch.equal(ex1["cache_pos"], ex2["cache_pos"])


def _decode_check(w, T_pre, steps, streams, chunk_pre=None):
    """Prefill T_pre tokens, then `steps` decode steps; compare sampled streams each step."""
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    layer = P.make_layer(w, dev["W"], max_tokens=T_pre)
    y0 = layer.prefill(dev["q"][:, :T_pre].contiguous(), dev["k"][:, :T_pre].contiguous(),
                       dev["v"][:, :T_pre].contiguous())
    torch.cuda.synchronize()
    ex = layer.export()
    tr = ex["trace_pos"].cpu().numpy() if w.lam > 0 else None
    oracles = {}
    tol = P.TOL[w.dtype]
    ties = hard = 0
    worst = 0.0
    for (b, g) in streams:
        st = P.oracle_stream(w, g)
        a = synth.stream_arrays(w, b, g)
        rows = np.zeros((w.Gq, T_pre), bool)
        rows[:, -w.chunk:] = True
        rows[:, ::97] = True
        yg = P.gpu_stream_y(y0, w, b, g)
        e, chain = P.check_prefill_stream(w, st, a, 0, T_pre, tr[b * w.Hkv + g], yg, rows)
        assert chain.hard == 0 and chain.set_mismatch == 0
        ties += chain.ties
        worst = max(worst, e)
        oracles[(b, g)] = (st, a)
    for i in range(steps):
        t = T_pre + i
        yd = layer.decode(dev["q"][:, t].contiguous(), dev["k"][:, t].contiguous(), dev["v"][:, t].contiguous())
        torch.cuda.synchronize()
        cpos = ex["cache_pos"].cpu().numpy()
        ydn = yd.double().cpu().numpy()
        for (b, g), (st, a) in oracles.items():
            S = b * w.Hkv + g
            chain = P.ChainCheck(w.lam)
            chain.expected = sorted(int(p) for p in cpos[S] if p >= 0)
            yo = st.decode(a["q"][:, t], a["k"][t], a["v"][t], chain.choose)
            hard += chain.hard
            ties += chain.ties
            assert sorted(st.cache) == chain.expected, (i, b, g)
            worst = max(worst, P.max_rel(ydn[b, g * w.Gq:(g + 1) * w.Gq], yo))
    for (b, g), (st, a) in oracles.items():
        S = b * w.Hkv + g
        if st.folded:
            assert P.max_rel(ex["H"][S].double().cpu().numpy(), st.H) <= tol
            assert P.max_rel(ex["s"][S].double().cpu().numpy(), st.s) <= tol
    assert hard == 0
    assert worst <= tol, worst
    return worst, ties


def test_decode_small():
    w = P.small_workload(4, B=2, Hkv=2, Hq=8, T=512, eta=64, lam=48, chunk=64, decode_steps=160)
    _decode_check(w, 512, 160, [(0, 0), (1, 1)])


@pytest.mark.parametrize("base,Hq,Hkv", [(4, 16, 2), (1, 4, 2)])
def test_decode_head_groups(base, Hq, Hkv):
    """Decode after a prefill that fills the cache, with 8 query heads per kv head
    (bf16, d 128) and with 2 (f32, d 64): both per-head register bounds of the kernel."""
    w = P.small_workload(base, B=1, Hkv=Hkv, Hq=Hq, T=384, eta=64, lam=48, chunk=64, decode_steps=96)
    _decode_check(w, 384, 96, [(0, 0), (0, Hkv - 1)])


def test_decode_from_empty_state_equals_oracle():
    """Decode from t = 0 (window filling, cache filling, then scoring) is a prefill with C = 1."""
    w = P.small_workload(1, T=64, eta=16, lam=12, chunk=64, decode_steps=200)
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    layer = P.make_layer(w, dev["W"], max_tokens=64)
    st = P.oracle_stream(w, 0)
    a = synth.stream_arrays(w, 0, 0)
    worst = 0.0
    for t in range(200):
        yd = layer.decode(dev["q"][:, t].contiguous(), dev["k"][:, t].contiguous(), dev["v"][:, t].contiguous())
        torch.cuda.synchronize()
        ex = layer.export()
        chain = P.ChainCheck(w.lam)
        chain.expected = sorted(int(p) for p in ex["cache_pos"][0].cpu().numpy() if p >= 0)
        yo = st.decode(a["q"][:, t], a["k"][t], a["v"][t], chain.choose)
        assert chain.hard == 0 and sorted(st.cache) == chain.expected
        worst = max(worst, P.max_rel(yd[0].double().cpu().numpy(), yo))
    assert worst <= P.TOL["f32"], worst


def test_host_buffer_entry_points_match_device():
    w = P.small_workload(2, B=1, Hkv=2, Hq=8, T=256, eta=64, lam=64, chunk=64, decode_steps=4)
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    l1 = P.make_layer(w, dev["W"], max_tokens=256)
    l2 = P.make_layer(w, dev["W"], max_tokens=256)
    y1 = l1.prefill(dev["q"][:, :256].contiguous(), dev["k"][:, :256].contiguous(), dev["v"][:, :256].contiguous())
    hq = dev["q"][:, :256].cpu().pin_memory()
    hk = dev["k"][:, :256].cpu().pin_memory()
    hv = dev["v"][:, :256].cpu().pin_memory()
    hy = torch.empty(y1.shape, dtype=torch.float32).pin_memory()
    l2.prefill_host(hq, hk, hv, hy)
    torch.cuda.synchronize()
    assert torch.equal(hy, y1.cpu())
    for t in range(256, 260):
        yd = l1.decode(dev["q"][:, t].contiguous(), dev["k"][:, t].contiguous(), dev["v"][:, t].contiguous())
        hyd = torch.empty(yd.shape, dtype=torch.float32).pin_memory()
        l2.decode_host(dev["q"][:, t].cpu().pin_memory(), dev["k"][:, t].cpu().pin_memory(),
                       dev["v"][:, t].cpu().pin_memory(), hyd)
        torch.cuda.synchronize()
        assert torch.equal(hyd, yd.cpu())


@pytest.mark.parametrize("T,Tpad", [(640, 640), (2240, 2560)])
def test_pipelined_host_prefill_matches_device(T, Tpad):
    """Host-buffer prefill of >= 8 chunks runs as segments whose copies overlap the
    compute (strided copies for B > 1, a short last segment, a state with spare
    capacity); it must equal the device-buffer call bit for bit, state included."""
    w = P.small_workload(2, B=2, Hkv=2, Hq=4, T=T, eta=64, lam=96, chunk=64)
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    l1 = P.make_layer(w, dev["W"], max_tokens=Tpad)
    l2 = P.make_layer(w, dev["W"], max_tokens=Tpad)
    y1 = l1.prefill(dev["q"], dev["k"], dev["v"])
    hq, hk, hv = (dev[x].cpu().pin_memory() for x in ("q", "k", "v"))
    hy = torch.full(y1.shape, float("nan"), dtype=torch.float32).pin_memory()
    l2.prefill_host(hq, hk, hv, hy)
    torch.cuda.synchronize()
    assert torch.equal(hy, y1.cpu())
    e1, e2 = l1.export(), l2.export()
    for key in ("H", "s", "cache_pos", "cache_k", "cache_v", "win_k", "win_v"):
        assert torch.equal(e1[key], e2[key]), key


@pytest.mark.slow
def test_repeated_full_batch_prefill_is_deterministic():
    """The 16K workload's shapes (B 4, lambda 1024, eta 512, C 128) on a 4096-token
    prefix, prefilled eight times from a reset state: every pass must finish
    without a device-side wait giving up (the kernels' barrier phases must not
    alias under any interleaving of their roles) and give the same bits."""
    w = synth.workload(3, T=4096)
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    q, k, v = (dev[x][:, :w.T].contiguous() for x in ("q", "k", "v"))
    layer = P.make_layer(w, dev["W"], max_tokens=w.T)
    y0 = None
    for _ in range(8):
        layer.reset()
        y = layer.prefill(q, k, v)
        layer.check()
        if y0 is None:
            y0 = y.clone()
        else:
            assert torch.equal(y, y0)


def test_invalid_arguments_are_errors():
    import sparse_kv_caching_b200 as lola
    w = P.small_workload(2, B=1, Hkv=2, Hq=8, T=256, eta=64, lam=64, chunk=64)
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    layer = P.make_layer(w, dev["W"], max_tokens=256)
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.prefill(dev["q"][:, :96].contiguous(), dev["k"][:, :96].contiguous(), dev["v"][:, :96].contiguous())
    big = torch.zeros((1, 320, 8, 128), dtype=torch.bfloat16, device="cuda")
    bigk = torch.zeros((1, 320, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lola.LolaError, match="INVALID_ARG"):
        layer.prefill(big, bigk, bigk)
    # nothing was processed by the failed calls
    assert layer.export()["t"] == 0


# ---------------------------------------------------------------------------
# Full-size workloads: sampled streams and rows
# ---------------------------------------------------------------------------
def _sample_rows(w, rng):
    rows = np.zeros((w.Gq, w.T), bool)
    rows[:, rng.choice(w.T, size=min(w.T, 96), replace=False)] = True
    rows[:, -w.chunk:] = True                      # the last block, incl. needle re-queries
    return rows


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_fullsize_prefill_sampled(cfg):
    _sampled_prefill_check(synth.workload(cfg), cfg)


@pytest.mark.slow
@pytest.mark.parametrize("eta,lam", [(64, 512), (512, 256)])
def test_layer_sweep_sampled(eta, lam):
    """Corners of the per-layer (eta, lambda) grid that bench.py --sweep times."""
    _sampled_prefill_check(synth.sweep_workload(eta, lam), eta + lam)


def _sampled_prefill_check(w, seed):
    cfg = w.name
    full = synth.full_arrays(w)
    dev = P.to_device(w, full)
    layer = P.make_layer(w, dev["W"], max_tokens=w.T)
    y = layer.prefill(dev["q"], dev["k"], dev["v"])
    torch.cuda.synchronize()
    ex = layer.export()
    tr = ex["trace_pos"].cpu().numpy()
    assert torch.isfinite(y).all()
    rng = np.random.default_rng(seed)
    streams = [(0, 0), (w.B - 1, w.Hkv - 1)]
    tol = P.TOL[w.dtype]
    ties = 0
    for (b, g) in streams:
        st = P.oracle_stream(w, g)
        a = synth.stream_arrays(w, b, g)
        yg = P.gpu_stream_y(y, w, b, g)
        e, chain = P.check_prefill_stream(w, st, a, 0, w.T, tr[b * w.Hkv + g], yg, _sample_rows(w, rng))
        assert chain.hard == 0 and chain.set_mismatch == 0, (b, g, chain.hard, chain.set_mismatch)
        assert e <= tol, (b, g, e)
        S = b * w.Hkv + g
        assert P.max_rel(ex["H"][S].double().cpu().numpy(), st.H) <= tol
        assert P.max_rel(ex["s"][S].double().cpu().numpy(), st.s) <= tol
        ties += chain.ties
    print(f"workload {cfg}: tie swaps {ties}")


@pytest.mark.slow
def test_fullsize_decode_sampled():
    w = synth.workload(4)
    _decode_check(w, w.T, w.decode_steps, [(0, 0), (w.B - 1, w.Hkv - 1)])

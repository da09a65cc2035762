"""bench.py's code paths that need a GPU cannot run here; at least every global
name its functions read must exist (catches a renamed or removed variable)."""
import builtins
import os
import symtable

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _global_reads(table, out):
    for child in table.get_children():
        for sym in child.get_symbols():
            if sym.is_referenced() and sym.is_global() and not sym.is_local():
                out.add((child.get_name(), sym.get_name()))
        _global_reads(child, out)


def test_bench_reads_only_defined_globals():
    path = os.path.join(ROOT, "bench.py")
    with open(path) as f:
        src = f.read()
    mod = symtable.symtable(src, path, "exec")
    defined = {s.get_name() for s in mod.get_symbols() if s.is_assigned() or s.is_imported()}
    defined |= set(dir(builtins))
    reads = set()
    _global_reads(mod, reads)
    missing = sorted((fn, name) for fn, name in reads if name not in defined)
    assert not missing, missing


# The work counts behind bench.py's roofline numbers, checked against the oracle's
# own bookkeeping on small workloads (every count the roofline divides by).

def _small(**kw):
    from dataclasses import replace
    import synth
    base = dict(B=1, Hq=4, Hkv=1, T=96, d=8, Dh=4, eta=12, lam=6, chunk=8, dtype="f32")
    base.update(kw)
    return replace(synth.workload(1), **base)


def _oracle_stream(w):
    import synth
    from oracle import LolaStream
    st = LolaStream(synth.weights(w)[0], w.eta, w.lam)
    a = synth.stream_arrays(w, 0, 0)
    return st, a


def test_sre_map_work_counts_folded_pairs():
    import bench
    for kw in (dict(), dict(lam=0), dict(eta=20, lam=3, chunk=4)):
        w = _small(**kw)
        st, a = _oracle_stream(w)
        st.prefill(a["q"], a["k"], a["v"], w.chunk)
        pairs = sum(r["folded_before"] for r in st.log) + len(st.folded)   # folded pairs at each state time
        got_pairs, flops = bench.sre_map_work(w)
        assert got_pairs == pairs
        assert flops == pairs * (2 * w.D * w.d + 2 * w.D + 3 * w.d)


def test_scorer_work_counts_window_reads():
    import bench
    import numpy as np
    for kw in (dict(), dict(eta=20, chunk=4)):
        w = _small(**kw)
        st, a = _oracle_stream(w)
        st.scorer = "attn"
        # q = 0 makes every credit worth exactly 1 (a = exp(0)), so a key's window score
        # counts the (query, head) pairs that read it through the window or its block
        st.prefill(np.zeros_like(a["q"]), a["k"], a["v"], w.chunk)
        credits = float(st._acc[:w.T].sum())
        want = bench.scorer_work(w)
        per_credit = 2 * w.d + 2 * w.D + 3
        assert want == int(round(credits)) * per_credit + w.T * w.Gq * 2 * w.d * w.Dh


def test_prefill_chain_work_matches_scored_blocks():
    import bench
    for kw in (dict(), dict(eta=20, lam=3, chunk=4), dict(lam=0)):
        w = _small(**kw)
        st, a = _oracle_stream(w)
        st.prefill(a["q"], a["k"], a["v"], w.chunk)
        D, d = w.D, w.d
        fl = 0
        for r in st.log:
            if r["score"] is None and not (w.lam == 0 and r["fold"]):
                continue
            n, f = len(r["E"]), len(r["fold"])
            fl += 2 * n * D * d + 2 * n * D + 3 * n * d + 2 * f * D * d + f * D
        assert bench.prefill_work(w)["scan"]["flops"] == w.B * w.Hkv * fl


def test_profile_summaries_give_runnable_commands():
    """Every committed ncu summary names the command that made it, with the clocks
    left alone, and runs committed files only."""
    import glob
    import json
    mds = glob.glob(os.path.join(ROOT, "profiles", "*.md"))
    assert mds
    for p in mds:
        txt = open(p).read()
        assert "ncu " in txt and "--clock-control none" in txt, p
        assert "_work" not in txt and "/root/" not in txt, p
    traffic = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, ent in traffic.items():
        assert "--clock-control none" in ent["capture"] and "_work" not in ent["capture"], key

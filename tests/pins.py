"""Independent checks that pin the CPU oracle to what the LoLA pages fix.

Each check recomputes its expectation from a closed form, a textbook routine
or brute force; none reuses the oracle's loop.  They are plain functions so
that tests/test_oracle_pins.py can run them on the oracle as written and on
deliberately broken copies of it (planted mistakes must be caught).
"""
from __future__ import annotations

import numpy as np
import torch

import synth


def small(T=48, d=8, Dh=4, eta=8, lam=6, C=4, Gq=2, **kw):
    """A tiny workload (fp32 values) built from the shared seeded generator."""
    base = dict(B=1, Hq=Gq, Hkv=1, T=T, d=d, Dh=Dh, eta=eta, lam=lam, chunk=C, dtype="f32",
                cluster_frac=0.5, n_clusters=3, cluster_std=0.05, n_needles=0,
                needle_place="none", decode_steps=0, wid=101)
    base.update(kw)
    w = synth.Workload("pin-small", **base)
    a = synth.stream_arrays(w, 0, 0)
    W = synth.weights(w)[0]
    return w, a, W


def softmax_fm(x, W):
    """phi via torch.softmax (a library routine), fp64."""
    z = torch.from_numpy(np.asarray(x, np.float64) @ np.asarray(W, np.float64))
    return torch.cat([torch.softmax(z, -1), torch.softmax(-z, -1)], -1).numpy()


def run(Stream, w, a, W, C=None):
    st = Stream(W, w.eta, w.lam)
    y = st.prefill(a["q"], a["k"], a["v"], C or w.chunk)
    return st, y


# (b) eta + lambda >= T: nothing is ever folded and y is causal softmax attention
def check_full_softmax(Stream, seed_kw=None) -> float:
    w, a, W = small(T=40, eta=16, lam=24, C=8, **(seed_kw or {}))
    st, y = run(Stream, w, a, W)
    q, k, v = (np.asarray(a[x], np.float64) for x in "qkv")
    ref = np.zeros_like(y)
    for h in range(q.shape[0]):           # textbook loop
        for t in range(w.T):
            l = k[:t + 1] @ q[h, t] / np.sqrt(w.d)
            p = np.exp(l - l.max())
            ref[h, t] = (p / p.sum()) @ v[:t + 1]
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k)[None].expand(q.shape[0], -1, -1),
        torch.from_numpy(v)[None].expand(q.shape[0], -1, -1), is_causal=True).numpy()
    assert np.abs(ref - sd).max() < 1e-12
    assert len(st.folded) == 0
    return float(np.abs(y - ref).max())


# (a) lambda = 0: the sliding-window + linear-attention hybrid (LoLCATs) in kernel form
def check_lambda0(Stream) -> float:
    w, a, W = small(T=48, eta=8, lam=0, C=4)
    st, y = run(Stream, w, a, W)
    q, k, v = (np.asarray(a[x], np.float64) for x in "qkv")
    pk = softmax_fm(k, W)
    err = 0.0
    for h in range(q.shape[0]):
        pq = softmax_fm(q[h], W)
        for t in range(w.T):
            t0 = (t // w.chunk) * w.chunk
            lo = max(0, t0 - w.eta)
            e = np.exp(k[lo:t + 1] @ q[h, t] / np.sqrt(w.d))
            kern = pk[:lo] @ pq[t]                    # phi(q)^T phi(k_i), i < t0 - eta
            num = e @ v[lo:t + 1] + kern @ v[:lo]
            den = e.sum() + kern.sum()
            err = max(err, float(np.abs(y[h, t] - num / den).max()))
    return err


# (c) brute-force state and its closed-form sums
def check_state(Stream) -> float:
    w, a, W = small()
    st, _ = run(Stream, w, a, W)
    k, v = np.asarray(a["k"], np.float64), np.asarray(a["v"], np.float64)
    F = st.folded
    assert len(set(F)) == len(F)
    H = np.zeros((2 * w.Dh, w.d))
    s = np.zeros(2 * w.Dh)
    for f in F:
        p = softmax_fm(k[f:f + 1], W)[0]
        H += np.outer(p, v[f])
        s += p
    e1 = np.abs(H - st.H).max()
    e2 = abs(st.s.sum() - 2 * len(F))                       # each half of phi sums to 1
    e3 = np.abs(st.H.sum(axis=0) - 2 * v[F].sum(axis=0)).max() if F else np.abs(st.H).max()
    return float(max(e1, np.abs(s - st.s).max(), e2, e3))


# (d) every retained set is the exhaustive top-lambda of E by an independently computed SRE
def check_selection(Stream) -> int:
    w, a, W = small(T=64, eta=8, lam=5, C=4)
    st, _ = run(Stream, w, a, W)
    k, v = np.asarray(a["k"], np.float64), np.asarray(a["v"], np.float64)
    bad = 0
    for rec in st.log:
        if rec["sre"] is None:
            continue
        F = st.folded[:rec["folded_before"]]
        D = 2 * w.Dh
        H = np.zeros((D, w.d))
        s = np.zeros(D)
        for f in F:
            p = softmax_fm(k[f:f + 1], W)[0]
            H += np.outer(p, v[f])
            s += p
        sre = {}
        for e in rec["E"]:
            p = softmax_fm(k[e:e + 1], W)[0]
            den = p @ s
            pred = (p @ H) / den if den > 0 else np.zeros(w.d)
            sre[e] = float(((pred - v[e]) ** 2).sum())
        keep = set(rec["keep"])
        drop = [e for e in rec["E"] if e not in keep]
        if len(keep) != w.lam:
            bad += 1
        for i in keep:                       # pairwise: each kept beats each dropped
            for j in drop:
                if not (sre[i] > sre[j] or (sre[i] == sre[j] and i < j)):
                    bad += 1
        if sorted(drop) != sorted(rec["fold"]):
            bad += 1
    return bad


# (e) identical keys: phi is the same for all, so pred is the mean of the folded values
def check_identical_keys(Stream) -> float:
    w, a, W = small(T=40, eta=4, lam=3, C=4)
    k0 = a["k"][0].copy()
    a = dict(a, k=np.tile(k0, (w.T, 1)))
    st, y = run(Stream, w, a, W)
    v = np.asarray(a["v"], np.float64)
    q = np.asarray(a["q"], np.float64)
    err = 0.0
    for rec in st.log:
        if rec["sre"] is None:
            continue
        F = st.folded[:rec["folded_before"]]
        vbar = v[F].mean(axis=0) if F else np.zeros(w.d)
        for i, e in enumerate(rec["E"]):
            err = max(err, abs(rec["sre"][i] - ((vbar - v[e]) ** 2).sum()))
    # output closed form: one logit per query, one kernel value per query
    pk = softmax_fm(k0[None], W)[0]
    for rec in st.log:
        t0 = rec["t0"]
        exact = rec["cache_before"] + [p for p in range(max(0, t0 - w.eta), t0)]
        F = st.folded[:rec["folded_before"]]
        for h in range(q.shape[0]):
            for t in range(t0, t0 + rec["n"]):
                ex = exact + list(range(t0, t + 1))
                ea = np.exp(q[h, t] @ k0 / np.sqrt(w.d))
                c = softmax_fm(q[h, t][None], W)[0] @ pk
                ref = (ea * v[ex].sum(0) + c * v[F].sum(0)) / (ea * len(ex) + c * len(F))
                err = max(err, float(np.abs(ref - y[h, t]).max()))
    return err


# (f) partition: every past position lives in exactly one of G, W, F
def check_partition(Stream) -> int:
    w, a, W = small(T=64, eta=8, lam=5, C=4)
    st = Stream(W, w.eta, w.lam)
    bad = 0
    for c0 in range(0, w.T, w.chunk):
        sl = slice(c0, c0 + w.chunk)
        st.step(a["q"][:, sl], a["k"][sl], a["v"][sl])
        t = c0 + w.chunk
        G, Wn, F = st.cache, st.window, st.folded
        allp = sorted(G + Wn + F)
        if allp != list(range(t)):
            bad += 1
        if Wn != list(range(max(0, t - w.eta), t)):
            bad += 1
        if len(G) != min(w.lam, max(0, t - w.eta)):
            bad += 1
    return bad


# (g) API identities: split calls == one call; decode == blocks of one token
def check_identities(Stream) -> float:
    w, a, W = small(T=48, eta=8, lam=5, C=4)
    st1, y1 = run(Stream, w, a, W)
    st2 = Stream(W, w.eta, w.lam)
    y2a = st2.prefill(a["q"][:, :20], a["k"][:20], a["v"][:20], 4)
    y2b = st2.prefill(a["q"][:, 20:], a["k"][20:], a["v"][20:], 4)
    e = np.abs(np.concatenate([y2a, y2b], 1) - y1).max()
    e = max(e, np.abs(st1.H - st2.H).max())
    st3, y3 = run(Stream, w, a, W, C=1)
    st4 = Stream(W, w.eta, w.lam)
    y4 = np.stack([st4.decode(a["q"][:, t], a["k"][t], a["v"][t]) for t in range(w.T)], 1)
    e = max(e, np.abs(y3 - y4).max(), np.abs(st3.H - st4.H).max())
    if st3.cache != st4.cache or st1.cache != st2.cache:
        e = np.inf
    return float(e)


# SRE closed forms: empty state recalls zero; one folded pair recalls its own value
def check_sre_closed_form(sre_fn) -> float:
    rng = np.random.default_rng(7)
    D, d = 6, 5
    phi = rng.random((4, D)) + 0.1
    v = rng.standard_normal((4, d))
    e = np.abs(sre_fn(phi, v, np.zeros((D, d)), np.zeros(D)) - (v * v).sum(1)).max()
    pf, vf = rng.random(D) + 0.1, rng.standard_normal(d)
    got = sre_fn(phi, v, np.outer(pf, vf), pf)
    return float(max(e, np.abs(got - ((v - vf) ** 2).sum(1)).max()))


# R5 tie order on exact ties: the older position is kept, the cap is exact
def check_tie_order(top_fn) -> int:
    cases = [([7, 3, 5], [2.0, 2.0, 2.0], 1, [3]),
             ([7, 3, 5], [2.0, 2.0, 2.0], 2, [3, 5]),
             ([1, 2, 3, 4], [1.0, 3.0, 3.0, 0.0], 1, [2]),
             ([9, 4, 6, 2], [5.0, 1.0, 5.0, 1.0], 3, [2, 6, 9])]
    return sum(sorted(top_fn(E, np.array(s), lam)) != want for E, s, lam, want in cases)


def _hybrid_ref(q, k, v, W, exact, F, read_state=True):
    """Eq. 14 by brute force for one query: softmax terms over `exact`, linear terms over F."""
    e = np.exp(k[exact] @ q / np.sqrt(len(q)))
    num, den = e @ v[exact], e.sum()
    if read_state and F:
        kern = softmax_fm(k[F], W) @ softmax_fm(q[None], W)[0]     # phi(q)^T phi(k_i)
        num, den = num + kern @ v[F], den + kern.sum()
    return num / den


# Read-branch masks, window only (notes §4.8, App. I): a banded causal softmax
def check_mask_window_only(Stream) -> float:
    w, a, W = small(T=48, eta=8, lam=6, C=4)
    st = Stream(W, w.eta, w.lam)
    st.read_mask = 3
    y = st.prefill(a["q"], a["k"], a["v"], w.chunk)
    q, k, v = (np.asarray(a[x], np.float64) for x in "qkv")
    t = np.arange(w.T)
    lo = np.maximum(0, (t // w.chunk) * w.chunk - w.eta)
    allowed = (t[None, :] <= t[:, None]) & (t[None, :] >= lo[:, None])
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k)[None].expand(q.shape[0], -1, -1),
        torch.from_numpy(v)[None].expand(q.shape[0], -1, -1), attn_mask=torch.from_numpy(allowed)).numpy()
    err = 0.0
    for h in range(q.shape[0]):            # textbook loop beside the library routine
        for tt in range(w.T):
            l = k[lo[tt]:tt + 1] @ q[h, tt] / np.sqrt(w.d)
            p = np.exp(l - l.max())
            ref = (p / p.sum()) @ v[lo[tt]:tt + 1]
            err = max(err, float(np.abs(ref - sd[h, tt]).max()), float(np.abs(ref - y[h, tt]).max()))
    return err


# Read-branch masks, one branch hidden: brute-force hybrids over the logged memories;
# the memories themselves evolve exactly as in the unmasked run
def check_mask_one_branch(Stream) -> float:
    w, a, W = small(T=64, eta=8, lam=5, C=4)
    q, k, v = (np.asarray(a[x], np.float64) for x in "qkv")
    ref_st, _ = run(Stream, w, a, W)
    err = 0.0
    for mask in (1, 2):
        st = Stream(W, w.eta, w.lam)
        st.read_mask = mask
        y = st.prefill(a["q"], a["k"], a["v"], w.chunk)
        for rec in st.log:
            t0 = rec["t0"]
            G = [] if mask == 2 else rec["cache_before"]
            F = st.folded[:rec["folded_before"]]
            for h in range(q.shape[0]):
                for t in range(t0, t0 + rec["n"]):
                    ex = G + list(range(max(0, t0 - w.eta), t + 1))
                    ref = _hybrid_ref(q[h, t], k, v, W, ex, F, read_state=(mask != 1))
                    err = max(err, float(np.abs(ref - y[h, t]).max()))
        if st.cache != ref_st.cache or st.folded != ref_st.folded:
            return np.inf
        err = max(err, float(np.abs(st.H - ref_st.H).max()), float(np.abs(st.s - ref_st.s).max()))
    return err


# Update-first decode (Eqs. 11-14 read literally): lambda = 0 gives a window of
# the eta most recent pairs (self included) plus the linear state over all older
# pairs; eta + lambda >= T gives causal softmax; the memories match read-first decode
def check_update_first(Stream) -> float:
    err = 0.0
    for T, eta, lam in ((40, 6, 0), (24, 10, 16), (48, 8, 5)):
        w, a, W = small(T=T, eta=eta, lam=lam, C=1)
        q, k, v = (np.asarray(a[x], np.float64) for x in "qkv")
        st = Stream(W, eta, lam)
        rf = Stream(W, eta, lam)
        for t in range(T):
            y = st.decode(a["q"][:, t], a["k"][t], a["v"][t], update_first=True)
            rf.decode(a["q"][:, t], a["k"][t], a["v"][t])
            if st.cache != rf.cache or st.folded != rf.folded or st.window != rf.window:
                return np.inf
            err = max(err, float(np.abs(st.H - rf.H).max()))
            lo = max(0, t - eta + 1)
            if lam == 0:
                for h in range(q.shape[0]):
                    ref = _hybrid_ref(q[h, t], k, v, W, list(range(lo, t + 1)), list(range(lo)))
                    err = max(err, float(np.abs(ref - y[h]).max()))
            elif eta + lam >= T:
                for h in range(q.shape[0]):
                    l = k[:t + 1] @ q[h, t] / np.sqrt(w.d)
                    p = np.exp(l - l.max())
                    err = max(err, float(np.abs((p / p.sum()) @ v[:t + 1] - y[h]).max()))
            else:                              # general case over the updated memories
                for h in range(q.shape[0]):
                    ref = _hybrid_ref(q[h, t], k, v, W, st.cache + list(range(lo, t + 1)), st.folded)
                    err = max(err, float(np.abs(ref - y[h]).max()))
    return err


# Stored-pair SRE map (Fig. 3) and relative SRE (Eq. 26): closed forms
def check_sre_map(Stream, map_fn) -> float:
    err = 0.0
    # one folded pair is recalled exactly; two folded pairs a, b:
    # SRE_a = (k_ab / (k_aa + k_ab))^2 ||v_b - v_a||^2, k = phi^T phi
    for C in (1, 2):
        w, a, W = small(T=16, eta=4, lam=0, C=C)
        st, _ = run(Stream, w, a, W)
        sre, rel = map_fn(st)
        n_folded = [r["folded_before"] for r in st.log] + [len(st.folded)]
        c = n_folded.index(C)
        v = np.asarray(a["v"], np.float64)
        if C == 1:
            err = max(err, abs(sre[c, 0]))
        else:
            pk = softmax_fm(a["k"][:2], W)
            K = pk @ pk.T
            for i, j in ((0, 1), (1, 0)):
                want = (K[i, j] / (K[i, i] + K[i, j])) ** 2 * ((v[j] - v[i]) ** 2).sum()
                err = max(err, abs(sre[c, i] - want) / want)
        if np.any(sre[:c, :] != 0) or np.any(rel[c] != 0):
            return np.inf
    # identical keys: the state recalls the mean of the folded values
    w, a, W = small(T=40, eta=4, lam=3, C=4)
    a = dict(a, k=np.tile(a["k"][0], (w.T, 1)))
    st, _ = run(Stream, w, a, W)
    sre, rel = map_fn(st)
    v = np.asarray(a["v"], np.float64)
    bounds = [r["t0"] for r in st.log] + [w.T]
    first = {}
    for c, t in enumerate(bounds):
        F = set(range(max(0, t - w.eta))) - set(st.log[c]["cache_before"] if c < len(st.log) else st.cache)
        vbar = v[sorted(F)].mean(axis=0) if F else None
        for i in range(w.T):
            if i not in F:
                if sre[c, i] != 0 or rel[c, i] != 0:
                    return np.inf
                continue
            want = ((vbar - v[i]) ** 2).sum()
            first.setdefault(i, want)
            err = max(err, abs(sre[c, i] - want), abs(rel[c, i] - (want - first[i])))
    return err


# Alternative scoring rules (R18): a key's score sums one term per query that reads it
# through the window or its own block.  Closed forms and a brute-force recount.
_RULE_CONST = {"kernel_sq": lambda a, f: (a - f) ** 2, "kernel_abs": lambda a, f: abs(a - f),
               "kernel_ratio": lambda a, f: f / a, "attn": lambda a, f: a}


def _window_reads(i, eta, C, T):
    """Queries that read key i exactly before it leaves the window (R2), by hand:
    its own block from i on, then the blocks whose preceding eta pairs hold it."""
    return list(range(i, min(T, ((i + eta) // C + 1) * C)))


def check_scorers(Stream) -> float:
    err = 0.0
    for rule, term in _RULE_CONST.items():
        # (1) q = 0: a = 1 and f = phi(0)^T phi(k) = 2 / Dh for every key (each half of phi sums to 1)
        w, a, W = small(T=64, eta=8, lam=5, C=4)
        a0 = dict(a, q=np.zeros_like(a["q"]))
        st = Stream(W, w.eta, w.lam)
        st.scorer = rule
        st.prefill(a0["q"], a0["k"], a0["v"], w.chunk)
        const = term(1.0, 2.0 / w.Dh)
        n_scored = 0
        for rec in st.log:
            if rec["score"] is None:
                continue
            n_scored += 1
            for e, sc in zip(rec["E"], rec["score"]):
                want = w.Gq * const * len(_window_reads(e, w.eta, w.chunk, w.T))
                err = max(err, abs(sc - want) / want)
        if n_scored == 0:
            return np.inf
        # per-token decode: eta + 1 reads (read first) or eta reads (update first)
        for uf in (False, True):
            st = Stream(W, w.eta, w.lam)
            st.scorer = rule
            for t in range(40):
                st.decode(a0["q"][:, t], a0["k"][t], a0["v"][t], update_first=uf)
            for rec in st.log:
                if rec["score"] is not None:
                    for sc in rec["score"]:
                        err = max(err, abs(sc - w.Gq * const * (w.eta + (0 if uf else 1))) / sc)
        # (2) every key and query the same vector x: a = exp(|x|^2 / sqrt(d)), f = |phi(x)|^2
        x = a["k"][3].astype(np.float64)
        ax = dict(a, k=np.tile(x, (w.T, 1)), q=np.tile(x, (w.Gq, w.T, 1)))
        st = Stream(W, w.eta, w.lam)
        st.scorer = rule
        st.prefill(ax["q"], ax["k"], ax["v"], w.chunk)
        av = float(np.exp(np.linalg.norm(x) ** 2 / np.sqrt(w.d)))
        fv = float(np.linalg.norm(softmax_fm(x[None], W)[0]) ** 2)
        for rec in st.log:
            if rec["score"] is not None:
                for e, sc in zip(rec["E"], rec["score"]):
                    want = w.Gq * term(av, fv) * len(_window_reads(e, w.eta, w.chunk, w.T))
                    err = max(err, abs(sc - want) / want)
        # (3) general inputs: scores recounted key by key; each kept key beats each folded one
        st = Stream(W, w.eta, w.lam)
        st.scorer = rule
        st.prefill(a["q"], a["k"], a["v"], w.chunk)
        q, k = np.asarray(a["q"], np.float64), np.asarray(a["k"], np.float64)
        pk = softmax_fm(k, W)
        for rec in st.log:
            if rec["score"] is None:
                continue
            got = dict(zip(rec["E"], rec["score"]))
            for e in rec["E"]:
                want = 0.0
                for t in _window_reads(e, w.eta, w.chunk, w.T):
                    for h in range(w.Gq):
                        want += term(np.exp(q[h, t] @ k[e] / np.sqrt(w.d)), softmax_fm(q[h, t][None], W)[0] @ pk[e])
                err = max(err, abs(got[e] - want) / abs(want))
            keep = set(rec["keep"])
            for i in keep:
                for j in rec["E"]:
                    if j not in keep and not (got[i] > got[j] or (got[i] == got[j] and i < j)):
                        return np.inf
    return err

"""Pins of the CPU oracle against what the LoLA pages and the mathematics fix.

CPU only (no GPU marker).  Every check comes from tests/pins.py and computes
its expectation independently of the oracle's own loop.  The planted-mistake
tests break the oracle on purpose (on the CPU, by monkeypatching) and require
that at least one pin notices.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.lola_oracle as lo
from oracle import LolaStream, feature_map, self_recall_error, state_elements, full_elements, sre_map
from tests import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_feature_map_halves_and_library_softmax():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 16))
    W = rng.standard_normal((16, 8)) / 4
    phi = feature_map(x, W)
    assert phi.shape == (5, 16)
    assert np.all(phi > 0)
    np.testing.assert_allclose(phi[:, :8].sum(1), 1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(phi[:, 8:].sum(1), 1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(phi, pins.softmax_fm(x, W), rtol=0, atol=1e-14)
    # x = 0 (or W = 0): both halves are uniform
    np.testing.assert_allclose(feature_map(np.zeros((1, 16)), W), 1 / 8, atol=1e-15)
    # the negative half of x is the positive half of -x
    np.testing.assert_allclose(feature_map(-x, W)[:, :8], phi[:, 8:], atol=1e-15)


def test_sre_closed_forms():
    assert pins.check_sre_closed_form(self_recall_error) < 1e-12


def test_full_softmax_reduction():
    assert pins.check_full_softmax(LolaStream) < 1e-12


def test_lambda0_is_window_plus_linear():
    assert pins.check_lambda0(LolaStream) < 1e-12


def test_bruteforce_state_and_sums():
    assert pins.check_state(LolaStream) < 1e-12


def test_selection_exhaustive():
    assert pins.check_selection(LolaStream) == 0


def test_identical_keys_closed_form():
    assert pins.check_identical_keys(LolaStream) < 1e-12


def test_mask_window_only_is_banded_softmax():
    assert pins.check_mask_window_only(LolaStream) < 1e-12


def test_mask_one_branch_hidden():
    assert pins.check_mask_one_branch(LolaStream) < 1e-12


def test_update_first_decode():
    assert pins.check_update_first(LolaStream) < 1e-12


def test_alternative_scorers():
    assert pins.check_scorers(LolaStream) < 1e-12


def test_sre_map_closed_forms():
    assert pins.check_sre_map(LolaStream, sre_map) < 1e-12


def test_partition_invariant():
    assert pins.check_partition(LolaStream) == 0


def test_api_identities():
    assert pins.check_identities(LolaStream) == 0.0


def test_selection_really_happens():
    """The small cases used by the pins exercise scoring, ties aside."""
    w, a, W = pins.small(T=64, eta=8, lam=5, C=4)
    st, _ = pins.run(LolaStream, w, a, W)
    scored = [r for r in st.log if r["sre"] is not None]
    assert len(scored) >= 10 and len(st.folded) > 20
    # at least one incumbent cache member was evicted and one newcomer retained
    assert any(set(r["fold"]) & set(r["cache_before"]) for r in scored)
    assert any(set(r["keep"]) & set(r["L"]) for r in scored)


def test_tie_order():
    assert pins.check_tie_order(lo.top_lambda) == 0


def test_valid_alternative_band():
    E = [0, 1, 2, 3]
    sre = np.array([5.0, 4.0, 4.0 * (1 + 5e-6), 1.0])
    assert lo.valid_alternative(E, sre, 2, [0, 1])
    assert lo.valid_alternative(E, sre, 2, [0, 2])
    assert not lo.valid_alternative(E, sre, 2, [0, 3])
    assert not lo.valid_alternative(E, sre, 2, [1, 2])
    assert lo.top_lambda(E, sre, 2) == [0, 2]
    # exact tie: older position first
    assert lo.top_lambda([7, 3], np.array([2.0, 2.0]), 1) == [3]


def test_choose_hook_rejects_invalid_sets():
    w, a, W = pins.small(T=64, eta=8, lam=5, C=4)
    st = LolaStream(W, w.eta, w.lam)

    def bad(rec):
        return sorted(rec["E"])[:w.lam]          # oldest lambda: generally not top-lambda

    with pytest.raises(ValueError):
        st.prefill(a["q"], a["k"], a["v"], w.chunk, choose=bad)


def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "app_b_memory_count.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                t, eta, lam, dk, dv, D, r, dig, mode = line.split()
                rows.append((int(t), int(eta), int(lam), int(dk), int(dv), int(D), float(r), int(dig), mode))
    return rows


@pytest.mark.parametrize("row", _golden_rows())
def test_golden_memory_count(row):
    t, eta, lam, dk, dv, D, printed, digits, mode = row
    ratio = full_elements(t, dk, dv) / state_elements(t, eta, lam, dk, dv, D)
    scale = 10 ** digits
    got = math.floor(ratio * scale) / scale if mode == "floor" else round(ratio, digits)
    assert got == pytest.approx(printed, abs=1e-9)


# ---------------------------------------------------------------------------
# Planted mistakes: each broken oracle must fail at least one pin.
# ---------------------------------------------------------------------------
def _all_pins_pass(Stream, sre_fn=None, map_fn=None):
    ok = True
    try:
        ok &= pins.check_mask_window_only(Stream) < 1e-9
        ok &= pins.check_mask_one_branch(Stream) < 1e-9
        ok &= pins.check_update_first(Stream) < 1e-9
        ok &= pins.check_sre_map(Stream, map_fn or lo.sre_map) < 1e-9
        ok &= pins.check_scorers(Stream) < 1e-9
        ok &= pins.check_sre_closed_form(sre_fn or lo.self_recall_error) < 1e-9
        ok &= pins.check_full_softmax(Stream) < 1e-9
        ok &= pins.check_lambda0(Stream) < 1e-9
        ok &= pins.check_state(Stream) < 1e-9
        ok &= pins.check_selection(Stream) == 0
        ok &= pins.check_identical_keys(Stream) < 1e-9
        ok &= pins.check_partition(Stream) == 0
        ok &= pins.check_identities(Stream) == 0.0
        ok &= pins.check_tie_order(lo.top_lambda) == 0
    except (AssertionError, ValueError, IndexError):
        return False
    return bool(ok)


def test_pins_pass_on_oracle():
    assert _all_pins_pass(LolaStream)


def _sre_no_division(phik, v, H, s):
    r = phik @ H - v
    return (r * r).sum(1)


def _sre_wrong_sign(phik, v, H, s):
    den = phik @ s
    pred = np.zeros((len(phik), H.shape[1]))
    ok = den > 0
    pred[ok] = (phik @ H)[ok] / den[ok, None]
    r = pred + v
    return (r * r).sum(1)


def _sre_unsquared_transposed(phik, v, H, s):       # H^T read as H (square case D == d)
    den = phik @ s
    pred = np.zeros_like(v)
    ok = den > 0
    pred[ok] = (phik @ H.T)[ok] / den[ok, None]
    return ((pred - v) ** 2).sum(1)


def _top_lowest(E, sre, lam):
    order = sorted(range(len(E)), key=lambda i: (sre[i], E[i]))
    return sorted(E[i] for i in order[:lam])


def _top_newest_on_ties(E, sre, lam):
    order = sorted(range(len(E)), key=lambda i: (-round(float(sre[i]), 1), -E[i]))
    return sorted(E[i] for i in order[:lam])


def _fm_same_half(x, W):
    z = np.asarray(x, np.float64) @ np.asarray(W, np.float64)
    e = np.exp(z - z.max(-1, keepdims=True))
    p = e / e.sum(-1, keepdims=True)
    return np.concatenate([p, p], -1)


class _NoS(LolaStream):
    def _fold(self, S):
        self.H = self.H + self.phiK[S].T @ self.V[S]
        self.folded.extend(S)


class _FoldTransposed(LolaStream):
    def _fold(self, S):
        self.H = self.H + self.V[S].T @ self.phiK[S]
        self.s = self.s + self.phiK[S].sum(axis=0)
        self.folded.extend(S)


class _NoLinearRead(LolaStream):
    def _read(self, Q, P, rows):
        H, s = self.H, self.s
        self.H, self.s = np.zeros_like(H), np.zeros_like(s)
        try:
            return super()._read(Q, P, rows)
        finally:
            self.H, self.s = H, s


class _MaskIgnored(LolaStream):
    def _read(self, Q, P, rows):
        m = self.read_mask
        self.read_mask = 0
        try:
            return super()._read(Q, P, rows)
        finally:
            self.read_mask = m


class _MaskHidesBothSums(LolaStream):         # hidden state dropped from the numerator only
    def _read(self, Q, P, rows):
        if not self.read_mask & lo.HIDE_STATE:
            return super()._read(Q, P, rows)
        H = self.H
        self.H = np.zeros_like(H)
        self.read_mask &= ~lo.HIDE_STATE
        try:
            return super()._read(Q, P, rows)
        finally:
            self.H = H
            self.read_mask |= lo.HIDE_STATE


class _UpdateFirstReadsEarly(LolaStream):
    def decode(self, q, k, v, choose=None, update_first=False):
        return super().decode(q, k, v, choose, False)


class _ScoreNoScale(LolaStream):               # exp kernel without the 1/sqrt(d)
    def _accumulate(self, Q, P, qpos):
        d = self.d
        self.d = 1
        try:
            super()._accumulate(Q, P, qpos)
        finally:
            self.d = d


class _ScoreSkipsBlock(LolaStream):           # the block's own causal keys are not credited
    def _accumulate(self, Q, P, qpos):
        super()._accumulate(Q, [], qpos)


def _map_state_off_by_one(st, first_block=0):
    sre, rel = lo.sre_map(st, first_block)
    return np.vstack([np.zeros((1, sre.shape[1])), sre[:-1]]), np.vstack([np.zeros((1, rel.shape[1])), rel[:-1]])


def _map_rel_from_previous(st, first_block=0):
    sre, _ = lo.sre_map(st, first_block)
    rel = np.zeros_like(sre)
    rel[1:] = np.where(sre[1:] != 0, sre[1:] - sre[:-1], 0)
    return sre, rel


class _WindowOffByOne(LolaStream):
    def __init__(self, W, eta, lam):
        super().__init__(W, eta + 1, lam)


@pytest.mark.parametrize("name", ["sre_no_division", "sre_wrong_sign", "sre_transposed",
                                  "keep_lowest", "tie_rule", "feature_same_half", "no_s_update",
                                  "fold_transposed", "no_linear_read", "window_off_by_one",
                                  "mask_ignored", "mask_numerator_only", "update_first_reads_early",
                                  "map_state_off_by_one", "map_rel_from_previous",
                                  "ratio_inverted", "score_no_scale", "score_skips_block"])
def test_planted_mistakes_are_caught(monkeypatch, name):
    Stream = LolaStream
    sre_fn = None
    map_fn = None
    if name == "sre_no_division":
        monkeypatch.setattr(lo, "self_recall_error", _sre_no_division); sre_fn = _sre_no_division
    elif name == "sre_wrong_sign":
        monkeypatch.setattr(lo, "self_recall_error", _sre_wrong_sign); sre_fn = _sre_wrong_sign
    elif name == "sre_transposed":
        monkeypatch.setattr(lo, "self_recall_error", _sre_unsquared_transposed)
        sre_fn = _sre_unsquared_transposed
    elif name == "keep_lowest":
        monkeypatch.setattr(lo, "top_lambda", _top_lowest)
    elif name == "tie_rule":
        monkeypatch.setattr(lo, "top_lambda", _top_newest_on_ties)
    elif name == "feature_same_half":
        monkeypatch.setattr(lo, "feature_map", _fm_same_half)
    elif name == "no_s_update":
        Stream = _NoS
    elif name == "fold_transposed":
        Stream = _FoldTransposed
    elif name == "no_linear_read":
        Stream = _NoLinearRead
    elif name == "window_off_by_one":
        Stream = _WindowOffByOne
    elif name == "mask_ignored":
        Stream = _MaskIgnored
    elif name == "mask_numerator_only":
        Stream = _MaskHidesBothSums
    elif name == "update_first_reads_early":
        Stream = _UpdateFirstReadsEarly
    elif name == "map_state_off_by_one":
        map_fn = _map_state_off_by_one
    elif name == "map_rel_from_previous":
        map_fn = _map_rel_from_previous
    elif name == "ratio_inverted":
        orig = lo.window_score_terms
        monkeypatch.setattr(lo, "window_score_terms",
                            lambda a, f, rule: a / f if rule == "kernel_ratio" else orig(a, f, rule))
    elif name == "score_no_scale":
        Stream = _ScoreNoScale
    elif name == "score_skips_block":
        Stream = _ScoreSkipsBlock
    assert not _all_pins_pass(Stream, sre_fn, map_fn)

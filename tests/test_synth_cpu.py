"""The seeded input recipe holds the structure the design notes state (CPU only).

Determinism, the bf16 rounding (round to nearest even, checked against
torch's own float32 -> bfloat16 conversion), the needles (planted keys
re-queried by the last queries of every head, at the stated depths), the
clustered-key fraction, the duplicate knob and the layouts of the assembled
arrays.
"""
import numpy as np
import torch

import synth


def test_streams_are_deterministic_and_distinct():
    w = synth.workload(2, T=256)
    a1, a2 = synth.stream_arrays(w, 0, 0), synth.stream_arrays(w, 0, 0)
    for x in "qkv":
        assert np.array_equal(a1[x], a2[x])
    b = synth.stream_arrays(w, 0, 1)
    assert not np.array_equal(a1["k"], b["k"])
    assert np.array_equal(synth.weights(w), synth.weights(w))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100_000).astype(np.float32) * 1e3,
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], np.float32)])
    ours = synth.round_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours, ref)
    bits = synth.bf16_bits(ours)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back, ours)


def test_needles_planted_and_requeried():
    w = synth.workload(3, T=2048, B=1)
    a = synth.stream_arrays(w, 0, 0)
    n = w.n_needles
    pos = synth.needle_positions(w)
    span = w.T - n
    assert list(pos) == [int(np.floor((i + 0.5) * span / n)) for i in range(n)]
    for h in range(w.Gq):
        assert np.array_equal(a["q"][h, w.T - n:w.T], a["k"][pos])      # q := k_needle, in order
    # the needles are fresh vectors, not members of a key cluster
    others = np.delete(a["k"], pos, axis=0)
    dmin = np.sqrt(((a["k"][pos][:, None, :] - others[None]) ** 2).sum(-1)).min()
    assert dmin > 5.0


def test_random_needles_inside_the_prefix():
    w = synth.workload(1)
    a = synth.stream_arrays(w, 0, 0)
    n = w.n_needles
    tail = a["q"][0, w.T - n:w.T]
    hits = [int(np.nonzero((a["k"] == tail[i]).all(1))[0][0]) for i in range(n)]
    assert hits == sorted(hits) and max(hits) < w.T - n and len(set(hits)) == n


def test_cluster_fraction():
    """Workload 2: about 20 % of the keys sit within a few sigma of a shared centre,
    so they have a near neighbour; independent N(0, I) keys never do."""
    w = synth.workload(2, T=4096)
    k = synth.stream_arrays(w, 0, 0)["k"].astype(np.float32)
    sq = (k * k).sum(1)
    d2 = sq[:, None] + sq[None, :] - 2.0 * (k @ k.T)
    np.fill_diagonal(d2, np.inf)
    near = (d2.min(1) < 4.0)                       # members: |k_i - k_j| ~ 0.05 sqrt(2 d) = 0.8
    frac = near.mean()
    assert 0.17 < frac < 0.23, frac


def test_duplicate_knob_copies_pair_zero():
    w = synth.workload(2, T=192, dup_every=3)
    a = synth.stream_arrays(w, 0, 0)
    idx = np.arange(0, w.T, 3)
    assert (a["k"][idx] == a["k"][0]).all() and (a["v"][idx] == a["v"][0]).all()
    assert not (a["k"][1] == a["k"][0]).all()


def test_full_arrays_layout():
    w = synth.workload(2, T=128, B=2)
    full = synth.full_arrays(w)
    assert full["q"].shape == (2, 128, 32, 128) and full["q"].dtype == np.uint16
    assert full["k"].shape == (2, 128, 8, 128) and full["W"].shape == (8, 128, 64)
    a = synth.stream_arrays(w, 1, 3)
    got = (full["k"][1, :, 3].astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(got, a["k"])
    gq = (full["q"][1, :, 3 * w.Gq:(3 + 1) * w.Gq].astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(gq.transpose(1, 0, 2), a["q"])

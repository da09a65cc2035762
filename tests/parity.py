"""Helpers that compare the CUDA library with the CPU oracle on the same inputs.

Tolerances: max relative error = max |x - r| / max |r| per tensor, 2e-3 for
bf16 inputs and 1e-4 for fp32 inputs (y, H and s separately).  Retained cache
sets must equal the oracle's except where the oracle itself accepts the
library's set as a top-lambda set up to ties within 1e-5 relative of the
lambda-th SRE (oracle.valid_alternative); such chunks are counted as ties and
the oracle continues along that branch.  Any other difference is a hard
mismatch.
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import torch

import synth
from oracle import LolaStream, valid_alternative

TOL = {"f32": 1e-4, "bf16": 2e-3}


def max_rel(x, r) -> float:
    x = np.asarray(x, np.float64)
    r = np.asarray(r, np.float64)
    den = np.abs(r).max()
    return float(np.abs(x - r).max() / (den if den > 0 else 1.0))


def to_device(w: synth.Workload, arrays: dict, device="cuda") -> dict:
    """Upload generator arrays (uint16 bf16 bits or float32) as device tensors."""
    out = {}
    for k, x in arrays.items():
        if x.dtype == np.uint16:
            out[k] = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(x)).to(device)
    return out


def make_layer(w: synth.Workload, W_dev: torch.Tensor, max_tokens: int | None = None):
    import sparse_kv_caching_b200 as lola
    cfg = lola.make_config(w.B, w.Hq, w.Hkv, w.d, w.Dh, w.eta, w.lam, w.chunk, w.dtype,
                           max_tokens or w.T)
    return lola.LolaLayer(cfg, W_dev)


class ChainCheck:
    """Follows the library's retained sets inside the oracle, classifying differences."""

    def __init__(self, lam: int):
        self.lam = lam
        self.ties = 0
        self.hard = 0
        self.scored = 0
        self.expected = None          # library set (sorted list) for the next oracle step

    def choose(self, rec):
        self.scored += 1
        gpu = self.expected
        if gpu is None or gpu == rec["keep"]:
            return None
        if valid_alternative(rec["E"], rec["score"], self.lam, gpu):
            self.ties += 1
            return gpu
        self.hard += 1
        return None


def oracle_stream(w: synth.Workload, g: int) -> LolaStream:
    W = synth.weights(w)[g]
    return LolaStream(W, w.eta, w.lam)


def check_prefill_stream(w, st: LolaStream, a: dict, t_lo: int, t_hi: int, trace: np.ndarray,
                         y_gpu: np.ndarray, rows: np.ndarray | None = None):
    """Run the oracle over positions [t_lo, t_hi) of stream arrays `a`, chunk by chunk,
    following the library's trace [chunks+1][lambda]; returns (max_rel_y, chain)."""
    C = w.chunk
    chain = ChainCheck(w.lam)
    ys = []
    set_mismatch = 0
    for ci, c0 in enumerate(range(t_lo, t_hi, C)):
        sl = slice(c0, c0 + C)
        entering = sorted(int(p) for p in trace[ci] if p >= 0)
        if w.lam > 0 and entering != sorted(st.cache):
            set_mismatch += 1
        after = sorted(int(p) for p in trace[ci + 1] if p >= 0) if w.lam > 0 else []
        chain.expected = after
        r = None if rows is None else rows[:, c0 - t_lo:c0 - t_lo + C]
        ys.append(st.step(a["q"][:, sl], a["k"][sl], a["v"][sl], r, chain.choose))
        if w.lam > 0 and sorted(st.cache) != after:
            set_mismatch += 1
    y = np.concatenate(ys, axis=1)
    mask = ~np.isnan(y)
    err = max_rel(y_gpu[mask], y[mask]) if mask.any() else 0.0
    chain.set_mismatch = set_mismatch
    chain.abs_err = float(np.abs(y_gpu[mask] - y[mask]).max()) if mask.any() else 0.0
    chain.y_max = float(np.abs(y[mask]).max()) if mask.any() else 0.0
    return err, chain


def gpu_stream_y(y: torch.Tensor, w, b: int, g: int) -> np.ndarray:
    """y [B, T, Hq, d] -> the stream's [Gq, T, d] block as float64 numpy."""
    return y[b, :, g * w.Gq:(g + 1) * w.Gq, :].permute(1, 0, 2).double().cpu().numpy()


def small_workload(base: int, **kw) -> synth.Workload:
    return replace(synth.workload(base), **kw)

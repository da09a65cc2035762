"""Seeded synthetic workloads for the LoLA chunkwise hybrid-attention layer.

This module only draws random numbers and places them: it holds none of the
method's arithmetic (no feature map, no attention, no scoring, no fold).  Both
the CPU oracle (tests) and the CUDA library (tests, bench) consume the arrays
it returns, so the two sides always see bit-identical inputs.

Recipe (per stream = one (sequence b, kv head g)):
  * a Generator seeded with (SEED_BASE, workload id, b, g) draws, in order:
    cluster centres [n_clusters, d] ~ N(0,1); cluster membership (uniform < frac);
    cluster choice (uniform over centres); key noise z [T, d] ~ N(0,1) with
    k = centre + std * z for members and k = z otherwise; queries [Gq, T, d]
    ~ N(0,1); values [T, d] ~ N(0,1); then needles.
  * needles: fresh N(0,1) key/value vectors written at their positions; the
    last n_needles query positions of every query head in the group re-query
    them in order (q := k_needle).  Positions are seeded-uniform without
    replacement ("random") or floor((i + 1/2) (T - N) / N) ("uniform").
  * duplicates (dup_every = m > 0, test workloads only): every position p with
    p % m == 0 gets an exact copy of the pair (k, v) at position 0, so many
    candidates carry bit-identical SRE scores (m = 1: all pairs equal).
  * W for kv head g comes from a Generator seeded with (SEED_BASE, workload id,
    W_STREAM, g): W ~ N(0, 1/d), shape [d, Dh].
  * bf16 workloads round q, k, v and W to bf16 (round to nearest even) before
    either side sees them.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

SEED_BASE = 20250529
W_STREAM = 1_000_003


@dataclass(frozen=True)
class Workload:
    """Shape, budget and value recipe of one synthetic layer workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    T: int            # prefill tokens per sequence
    d: int            # head dim (d_k = d_v)
    Dh: int           # feature-map half width; D = 2 * Dh
    eta: int          # sliding-window size
    lam: int          # sparse-cache capacity (lambda)
    chunk: int        # prefill chunk length C
    dtype: str        # "f32" or "bf16"
    cluster_frac: float = 0.0
    n_clusters: int = 0
    cluster_std: float = 0.0
    n_needles: int = 0
    needle_place: str = "none"   # "random" | "uniform" | "none"
    decode_steps: int = 0        # tokens appended one by one after prefill
    wid: int = 0                 # seed id
    dup_every: int = 0           # > 0: pairs at positions p % dup_every == 0 copy pair 0

    @property
    def Gq(self) -> int:
        return self.Hq // self.Hkv

    @property
    def D(self) -> int:
        return 2 * self.Dh

    @property
    def T_total(self) -> int:
        return self.T + self.decode_steps

    @property
    def streams(self) -> int:
        return self.B * self.Hkv


WORKLOADS = {
    1: Workload("tiny-f32", B=1, Hq=1, Hkv=1, T=512, d=64, Dh=32, eta=64, lam=64,
                chunk=64, dtype="f32", cluster_frac=1.0, n_clusters=8,
                cluster_std=0.1, n_needles=4, needle_place="random", wid=1),
    2: Workload("llama8b-4k", B=1, Hq=32, Hkv=8, T=4096, d=128, Dh=64, eta=256,
                lam=256, chunk=64, dtype="bf16", cluster_frac=0.2, n_clusters=64,
                cluster_std=0.05, wid=2),
    3: Workload("llama8b-16k", B=4, Hq=32, Hkv=8, T=16384, d=128, Dh=64, eta=512,
                lam=1024, chunk=128, dtype="bf16", cluster_frac=0.2, n_clusters=64,
                cluster_std=0.05, n_needles=16, needle_place="uniform", wid=3),
    4: Workload("llama8b-decode", B=64, Hq=32, Hkv=8, T=4096, d=128, Dh=64, eta=64,
                lam=256, chunk=64, dtype="bf16", decode_steps=1024, wid=4),
    5: Workload("llama1b-32k", B=8, Hq=32, Hkv=8, T=32768, d=64, Dh=32, eta=128,
                lam=512, chunk=64, dtype="bf16", cluster_frac=0.5, n_clusters=256,
                cluster_std=0.1, wid=5),
}


# Per-layer (eta, lambda) grid at the single-layer shape of the App. B latency
# tables (batch 2, 4096 tokens, 32 heads, head dim 128), Llama-3.1-8B grouping
# 32/8, values drawn as in workload 2.  The recipe does not depend on (eta,
# lambda), so every grid point sees the same q, k, v and W.
SWEEP_ETAS = (64, 128, 256, 512)
SWEEP_LAMBDAS = (0, 64, 128, 256, 512)


def sweep_workload(eta: int, lam: int) -> Workload:
    """One point of the per-layer (eta, lambda) grid."""
    return Workload(f"layer-e{eta}-l{lam}", B=2, Hq=32, Hkv=8, T=4096, d=128, Dh=64, eta=eta, lam=lam,
                    chunk=64, dtype="bf16", cluster_frac=0.2, n_clusters=64, cluster_std=0.05, wid=6)


def workload(i: int, **overrides) -> Workload:
    """Workload `i` (1..5), optionally with fields replaced (smaller T, B, ...)."""
    w = WORKLOADS[i]
    return replace(w, **overrides) if overrides else w


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _cast(w: Workload, x: np.ndarray) -> np.ndarray:
    return round_bf16(x) if w.dtype == "bf16" else x.astype(np.float32)


def needle_positions(w: Workload, rng: np.random.Generator | None = None) -> np.ndarray:
    """Positions of the planted needles inside [0, T - n_needles)."""
    n = w.n_needles
    if n == 0:
        return np.zeros(0, np.int64)
    span = w.T - n
    if w.needle_place == "uniform":
        return np.array([((2 * i + 1) * span) // (2 * n) for i in range(n)], np.int64)
    if w.needle_place == "random":
        return np.sort(rng.choice(span, size=n, replace=False)).astype(np.int64)
    raise ValueError(w.needle_place)


def stream_arrays(w: Workload, b: int, g: int) -> dict:
    """q [Gq, T_total, d], k [T_total, d], v [T_total, d] (float32) for stream (b, g)."""
    T, d, Gq = w.T_total, w.d, w.Gq
    rng = np.random.default_rng([SEED_BASE, w.wid, b, g])
    centres = rng.standard_normal((max(w.n_clusters, 1), d), dtype=np.float32)
    member = rng.random(T) < w.cluster_frac
    choice = rng.integers(0, max(w.n_clusters, 1), size=T)
    z = rng.standard_normal((T, d), dtype=np.float32)
    if w.n_clusters > 0 and w.cluster_frac > 0:
        k = np.where(member[:, None], centres[choice] + np.float32(w.cluster_std) * z, z)
    else:
        k = z
    q = rng.standard_normal((Gq, T, d), dtype=np.float32)
    v = rng.standard_normal((T, d), dtype=np.float32)
    if w.n_needles:
        pos = needle_positions(w, rng)
        kn = rng.standard_normal((w.n_needles, d), dtype=np.float32)
        vn = rng.standard_normal((w.n_needles, d), dtype=np.float32)
        k[pos] = kn
        v[pos] = vn
        q[:, w.T - w.n_needles:w.T, :] = kn[None]
    if w.dup_every > 0:
        idx = np.arange(0, T, w.dup_every)
        k[idx] = k[0]
        v[idx] = v[0]
    return dict(q=_cast(w, q), k=_cast(w, k), v=_cast(w, v))


def weights(w: Workload) -> np.ndarray:
    """Feature-map weights W [Hkv, d, Dh] (float32, bf16-representable for bf16)."""
    out = np.empty((w.Hkv, w.d, w.Dh), np.float32)
    for g in range(w.Hkv):
        rng = np.random.default_rng([SEED_BASE, w.wid, W_STREAM, g])
        out[g] = rng.standard_normal((w.d, w.Dh), dtype=np.float32) / np.float32(np.sqrt(w.d))
    return _cast(w, out)


def full_arrays(w: Workload, bits: bool = True, threads: int | None = None) -> dict:
    """All streams assembled in the library's layouts.

    q [B, T_total, Hq, d], k/v [B, T_total, Hkv, d], W [Hkv, d, Dh].  With
    bits=True and a bf16 workload the arrays are uint16 bf16 bit patterns
    (ready to reinterpret as bf16 on the device); otherwise float32.
    """
    T, d, Gq = w.T_total, w.d, w.Gq
    as_bits = bits and w.dtype == "bf16"
    et = np.uint16 if as_bits else np.float32
    q = np.empty((w.B, T, w.Hq, d), et)
    k = np.empty((w.B, T, w.Hkv, d), et)
    v = np.empty((w.B, T, w.Hkv, d), et)

    def fill(bg):
        b, g = bg
        a = stream_arrays(w, b, g)
        cv = bf16_bits if as_bits else (lambda x: x)
        q[b, :, g * Gq:(g + 1) * Gq, :] = cv(a["q"]).transpose(1, 0, 2)
        k[b, :, g, :] = cv(a["k"])
        v[b, :, g, :] = cv(a["v"])

    jobs = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    n = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(n) as ex:
        list(ex.map(fill, jobs))
    Wt = weights(w)
    return dict(q=q, k=k, v=v, W=bf16_bits(Wt) if as_bits else Wt)

"""Plain, slow, fp64 CPU oracle for LoLA's chunkwise hybrid attention.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import this module.  It shares no code with
the CUDA library (sparse_kv_caching_b200) and never imports it; the only input
both sides share is the seeded generator in `synth`, which holds none of the
method's arithmetic.

Source: "LoLA: Low-Rank Linear Attention With Sparse Caching" (McDermott,
Heath, Parhi; arXiv 2505.23666v3), as restated by its close-reading notes
(cc.laoqi.cc, LoLA reading notes): §2.2 (Eqs. 3-5, linear attention state),
§2.3 (Eq. 10, Self-Recall Error), §2.4 (Fig. 1, Eqs. 11-13, candidate set,
top-lambda retention, fold), §2.5 (Eq. 14, shared normaliser), §2.6 (Eq. 15,
Fig. 2, chunkwise inference) and §2.7 (App. B memory count).

Readings taken where the pages leave a step open (each is listed, with its
reason and under the same number, in the design notes of this repository):
  R1  SRE is the squared L2 residual (the summaries' form); the ranking equals
      that of the unsquared norm of §2.3.
  R2  eta counts the exact pairs that precede the current block; the block's
      own causal pairs are read in addition.  After the block is appended to
      the window, the oldest pairs beyond eta leave it (the set L).
  R3  Read first with the state entering the block, then update (§2.6: the
      queries of a block share the existing state; scoring follows the block).
      The per-token decode step is the same rule with a block of one token.
  R4  With H = 0 and s = 0 (nothing folded yet) the memory recalls the zero
      vector, so SRE = ||v||^2.  phi > 0, hence phi(k)^T s > 0 once anything
      has been folded; no epsilon is added anywhere.
  R5  Ties at the lambda-th score: exact cap of lambda, order (SRE descending,
      position ascending): the older pair is kept.
  R6  |E| <= lambda keeps every candidate: no scoring, no fold (§2.4).
  R7  GQA: kv head floor(h / Gq) serves query head h; W, H, s, G and the window
      are per kv head and the selection is shared by the head group.
  R8  The output is Eq. 14 evaluated as written (no max-stabiliser: the fp64
      exponent stays far from overflow for these inputs; this is asserted).
  R15 Read-branch masks (notes §4.8, App. I, Table 12): a hidden branch is
      dropped from both the numerator and the shared denominator of Eq. 14;
      the memories are updated exactly as without the mask.
  R16 Update-first decode (the token equations of notes §2.4, Eqs. 11-14
      taken literally): the new pair enters the window, the pair eta steps
      back leaves it and is scored with the cache against the state, and
      only then does the query read; it sees the eta most recent pairs,
      itself included.  The memories evolve exactly as under R3.
  R18 Alternative scoring rules (notes §4.5, Table 4; App. F, whose Eqs.
      22-25 the pages do not print): with a = exp(q.k / sqrt(d)) (the
      exponential kernel of Eq. 14) and f = phi(q)^T phi(k) (the feature
      kernel), a key's score is the sum over every query that reads it
      exactly through the window or its own block (any head of the group) of
      (a - f)^2 ("kernel_sq"), |a - f| ("kernel_abs"), f / a ("kernel_ratio":
      keys the linear kernel over-weights score high) or a ("attn").  The sum
      stops when the key leaves the window (the scores are accumulated while
      the key is in the window, never from later queries) and is frozen while
      the key is cached.  The lambda highest scores are kept, as for SRE.
  R17 Stored-pair SRE map (notes §4.4, Fig. 3): at each state time (a block
      boundary) every folded pair's SRE against that state; pairs not in the
      state are 0.  Relative SRE (notes §4.4, Fig. 10, Eq. 26): that value
      minus the pair's SRE at the first state time that held it.

Parity status of every function here: pinned by the tests in
tests/test_oracle_pins.py (closed forms, reductions to textbook softmax
attention and to the window+linear hybrid, brute-force state, exhaustive
pairwise check of the selection, identical-key closed form, partition
invariant, decode == one-token blocks, split calls == one call, and the
printed App. B / Table 10 memory counts).  The read masks, the update-first
decode and the SRE map are pinned the same way (banded softmax, brute-force
hybrids over the logged memories, the one-, two- and identical-pair closed
forms of the map).
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-5   # relative band around the lambda-th SRE inside which swaps are valid
HIDE_STATE = 1   # read mask bit: the queries do not read (H, s)            (R15)
HIDE_SPARSE = 2  # read mask bit: the queries do not read the sparse cache G (R15)
SCORERS = ("sre", "kernel_sq", "kernel_abs", "kernel_ratio", "attn")   # R1 and R18


def window_score_terms(a: np.ndarray, f: np.ndarray, rule: str) -> np.ndarray:
    """Per-(query, key) term of an alternative scoring rule (R18), a = exp kernel, f = feature kernel."""
    if rule == "kernel_sq":
        return (a - f) ** 2
    if rule == "kernel_abs":
        return np.abs(a - f)
    if rule == "kernel_ratio":
        return f / a
    if rule == "attn":
        return a
    raise ValueError(f"unknown scoring rule {rule!r}")


# ---------------------------------------------------------------------------
# Feature map (notes §2.1 notation table: learned phi: R^{d_k} -> R^D; the
# Hedgehog form [softmax(xW), softmax(-xW)] is the form fixed here)
# ---------------------------------------------------------------------------
def _softmax(z: np.ndarray) -> np.ndarray:
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def feature_map(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """phi(x) = [softmax(x W), softmax(-x W)] in fp64; x [..., d], W [d, Dh] -> [..., 2 Dh]."""
    z = np.asarray(x, np.float64) @ np.asarray(W, np.float64)
    return np.concatenate([_softmax(z), _softmax(-z)], axis=-1)


# ---------------------------------------------------------------------------
# Memory count of App. B (notes §2.7): elements held per head after t tokens.
# ---------------------------------------------------------------------------
def state_elements(t: int, eta: int, lam: int, d_k: int, d_v: int, D: int) -> int:
    """M_LoLA(t) = min{ t (d_k + d_v), (eta + lam)(d_k + d_v) + D d_v + D }."""
    return min(t * (d_k + d_v), (eta + lam) * (d_k + d_v) + D * d_v + D)


def full_elements(t: int, d_k: int, d_v: int) -> int:
    """M_full(t) = t (d_k + d_v): the softmax KV cache of the same head."""
    return t * (d_k + d_v)


# ---------------------------------------------------------------------------
# Self-Recall Error (notes §2.3, Eq. 10; squared per R1; zero state per R4)
# ---------------------------------------------------------------------------
def self_recall_error(phik: np.ndarray, v: np.ndarray, H: np.ndarray, s: np.ndarray) -> np.ndarray:
    """SRE(k, v | H, s) = || H^T phi(k) / (phi(k)^T s) - v ||^2 for each row.

    phik [n, D], v [n, d], H [D, d], s [D] -> [n].  Where phi(k)^T s == 0 the
    prediction is the zero vector (R4).
    """
    den = phik @ s
    num = phik @ H
    pred = np.zeros_like(num)
    ok = den > 0
    pred[ok] = num[ok] / den[ok, None]
    r = pred - v
    return (r * r).sum(axis=1)


def top_lambda(E: list[int], sre: np.ndarray, lam: int) -> list[int]:
    """Top_lambda of Eq. 11 with the exact cap and tie order of R5."""
    order = sorted(range(len(E)), key=lambda i: (-sre[i], E[i]))
    return sorted(E[i] for i in order[:lam])


def valid_alternative(E: list[int], sre: np.ndarray, lam: int, keep: list[int],
                      rel: float = TIE_REL) -> bool:
    """True if `keep` is a top-lambda set of E under scores `sre` up to ties.

    A set is valid when it has lambda distinct members of E, every kept score is
    >= tau (1 - rel) and every dropped score is <= tau (1 + rel), tau being the
    lambda-th largest score.  Only these sets count as correct results when the
    lambda-th score is (nearly) tied.
    """
    ks = set(keep)
    if len(ks) != lam or len(keep) != lam or not ks <= set(E):
        return False
    tau = float(np.sort(sre)[::-1][lam - 1])
    band = rel * abs(tau)
    for i, e in enumerate(E):
        if e in ks and sre[i] < tau - band:
            return False
        if e not in ks and sre[i] > tau + band:
            return False
    return True


class LolaStream:
    """The three memories of one LoLA head stream: window W, sparse cache G, state (H, s).

    One instance serves one (sequence, kv head) pair and its group of query
    heads.  Every token ever seen is kept in a plain history so that positions
    index it; the memories themselves hold positions only.
    """

    def __init__(self, W: np.ndarray, eta: int, lam: int, read_mask: int = 0, scorer: str = "sre"):
        self.W = np.asarray(W, np.float64)
        self.read_mask = int(read_mask)
        if scorer not in SCORERS:
            raise ValueError(f"unknown scoring rule {scorer!r}")
        self.scorer = scorer
        self.d, self.Dh = self.W.shape
        self.D = 2 * self.Dh
        self.eta, self.lam = int(eta), int(lam)
        self._K = np.zeros((0, self.d))
        self._V = np.zeros((0, self.d))
        self._phiK = np.zeros((0, self.D))
        self._acc = np.zeros(0)         # accumulated window score of each key (R18)
        self.t = 0
        self.window: list[int] = []     # W: positions, oldest first
        self.cache: list[int] = []      # G: positions (sorted)
        self.folded: list[int] = []     # F: positions absorbed into (H, s)
        self.H = np.zeros((self.D, self.d))
        self.s = np.zeros(self.D)
        self.log: list[dict] = []

    # -- history (positions 0 .. t-1; storage grows geometrically) -------
    @property
    def K(self) -> np.ndarray:
        return self._K[:self.t]

    @property
    def V(self) -> np.ndarray:
        return self._V[:self.t]

    @property
    def phiK(self) -> np.ndarray:
        return self._phiK[:self.t]

    def _append(self, k: np.ndarray, v: np.ndarray) -> list[int]:
        k = np.asarray(k, np.float64).reshape(-1, self.d)
        v = np.asarray(v, np.float64).reshape(-1, self.d)
        n = len(k)
        if self.t + n > len(self._K):
            cap = max(self.t + n, 2 * len(self._K), 64)
            for name, width in (("_K", self.d), ("_V", self.d), ("_phiK", self.D)):
                grown = np.zeros((cap, width))
                grown[:self.t] = getattr(self, name)[:self.t]
                setattr(self, name, grown)
            acc = np.zeros(cap)
            acc[:self.t] = self._acc[:self.t]
            self._acc = acc
        self._acc[self.t:self.t + n] = 0.0
        self._K[self.t:self.t + n] = k
        self._V[self.t:self.t + n] = v
        self._phiK[self.t:self.t + n] = feature_map(k, self.W)
        P = list(range(self.t, self.t + n))
        self.t += n
        return P

    # -- read (Eq. 14 with the memories as they stand; R3, R8, R15) --------
    def _read(self, Q: np.ndarray, P: list[int], rows: np.ndarray | None) -> np.ndarray:
        """Eq. 14 for queries Q [Gq, n, d]; P = the block's own positions, read causally."""
        Gq, n, d = Q.shape
        y = np.full((Gq, n, d), np.nan)
        exact = ([] if self.read_mask & HIDE_SPARSE else self.cache) + self.window
        read_state = not self.read_mask & HIDE_STATE
        Ke, Ve = self.K[exact], self.V[exact]
        Kb, Vb = self.K[P], self.V[P]
        causal = np.tril(np.ones((n, len(P))))     # block key j visible to query i iff j <= i
        scale = 1.0 / np.sqrt(d)
        for h in range(Gq):
            sel = np.arange(n) if rows is None else np.nonzero(rows[h])[0]
            if len(sel) == 0:
                continue
            q = np.asarray(Q[h, sel], np.float64)
            le = (q @ Ke.T) * scale
            lb = (q @ Kb.T) * scale
            assert le.size == 0 or le.max() < 700.0
            assert lb.size == 0 or lb.max() < 700.0
            ae = np.exp(le)
            ab = np.exp(lb) * causal[sel]
            num = ae @ Ve + ab @ Vb
            den = ae.sum(axis=1) + ab.sum(axis=1)
            if read_state:
                phq = feature_map(q, self.W)
                num = num + phq @ self.H
                den = den + phq @ self.s
            y[h, sel] = num / den[:, None]
        return y

    # -- one update interval (notes §2.4 and §2.6) -------------------------
    def _accumulate(self, Q: np.ndarray, P: list[int], qpos: list[int]) -> None:
        """R18: add every query's term to the keys it reads exactly through the window
        or its own block (P, causally).  Q [Gq, n, d] are the queries at positions qpos."""
        if self.scorer == "sre":
            return
        scale = 1.0 / np.sqrt(self.d)
        for qi, t in enumerate(qpos):
            keys = self.window + [j for j in P if j <= t]
            q = np.asarray(Q[:, qi], np.float64)                     # [Gq, d]
            a = np.exp((q @ self.K[keys].T) * scale)                  # [Gq, n_keys]
            f = feature_map(q, self.W) @ self.phiK[keys].T
            self._acc[keys] += window_score_terms(a, f, self.scorer).sum(axis=0)

    def step(self, Q, K, V, rows=None, choose=None) -> np.ndarray:
        """Process one block of new tokens: read, advance window, score, keep, fold.

        Q [Gq, n, d], K/V [n, d].  `rows` (bool [Gq, n]) limits which outputs
        are computed (others are NaN).  `choose(record)` may return another
        retained set; it is adopted only if `valid_alternative` accepts it
        under this oracle's own scores (tie handling, R5).
        """
        Q = np.asarray(Q, np.float64)
        if Q.ndim == 2:
            Q = Q[:, None, :]
        P = self._append(K, V)
        y = self._read(Q, P, rows)
        self._accumulate(Q, P, P)
        self._update(P, choose)
        return y

    def _update(self, P: list[int], choose=None) -> None:
        """Window advance, candidates, scores (SRE or R18), top-lambda and fold for the new positions P."""
        # advance the window: the block enters, the oldest pairs beyond eta leave (R2)
        self.window.extend(P)
        n_leave = max(0, len(self.window) - self.eta)
        L, self.window = self.window[:n_leave], self.window[n_leave:]
        E = self.cache + L                          # candidate set E
        rec = dict(t0=P[0], n=len(P), E=E, L=L, sre=None, score=None, keep=None, fold=[], adopted=False,
                   cache_before=list(self.cache), window_after=list(self.window),
                   folded_before=len(self.folded))
        if len(E) <= self.lam:                      # R6
            self.cache = sorted(E)
        else:
            if self.scorer == "sre":
                score = self_recall_error(self.phiK[E], self.V[E], self.H, self.s)   # pre-fold state
                rec.update(sre=score)
            else:
                score = self._acc[E].copy()          # frozen window accumulations (R18)
            keep = top_lambda(E, score, self.lam)
            rec.update(score=score, keep=keep)
            if choose is not None:
                alt = choose(rec)
                if alt is not None and sorted(alt) != keep:
                    if not valid_alternative(E, score, self.lam, list(alt)):
                        raise ValueError("rejected retained set: not a top-lambda set up to ties")
                    keep = sorted(alt)
                    rec.update(keep=keep, adopted=True)
            ks = set(keep)
            S = [e for e in E if e not in ks]
            self._fold(S)
            self.cache = keep
            rec["fold"] = S
        self.log.append(rec)

    def _fold(self, S: list[int]) -> None:
        """Eqs. 12-13: H += sum phi(k) v^T, s += sum phi(k) over the pairs S leaving E."""
        self.H = self.H + self.phiK[S].T @ self.V[S]
        self.s = self.s + self.phiK[S].sum(axis=0)
        self.folded.extend(S)

    def prefill(self, Q, K, V, chunk: int, rows=None, choose=None) -> np.ndarray:
        """Chunkwise prefill (Eq. 15): blocks of `chunk` tokens, in order."""
        Q = np.asarray(Q)
        n = K.shape[0]
        assert n % chunk == 0
        out = []
        for c0 in range(0, n, chunk):
            r = None if rows is None else rows[:, c0:c0 + chunk]
            out.append(self.step(Q[:, c0:c0 + chunk], K[c0:c0 + chunk], V[c0:c0 + chunk], r, choose))
        return np.concatenate(out, axis=1)

    def decode(self, q, k, v, choose=None, update_first: bool = False) -> np.ndarray:
        """Per-token decode step: one block of a single token (R3), or update then read (R16)."""
        Q = np.asarray(q, np.float64).reshape(-1, 1, self.d)
        if not update_first:
            return self.step(Q, k, v, None, choose)[:, 0]
        P = self._append(k, v)
        self._update(P, choose)
        self._accumulate(Q, [], P)               # the new pair is now the newest window member
        return self._read(Q, [], None)[:, 0]


# ---------------------------------------------------------------------------
# Stored-pair SRE over time (notes §4.4: Fig. 3; Fig. 10 and Eq. 26; R17)
# ---------------------------------------------------------------------------
def sre_map(st: LolaStream, first_block: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """SRE of every folded pair at each state time, and its change since first write.

    State time c (0 <= c <= n, n = logged blocks from `first_block` on) is the
    state entering block first_block + c; c = n is the state after the last
    block.  Returns (sre, rel), both [n + 1, t] fp64 over positions 0 .. t-1:
      sre[c, i] = SRE(k_i, v_i | H_c, s_c) if pair i is folded at time c, else 0,
      rel[c, i] = sre[c, i] - sre[c_i, i], c_i the first state time holding i.
    H_c and s_c are summed again from their definition over the folded set
    (Eqs. 12-13 accumulated), not taken from the running state.
    """
    recs = st.log[first_block:]
    n_folded = [r["folded_before"] for r in recs] + [len(st.folded)]
    sre = np.zeros((len(n_folded), st.t))
    rel = np.zeros_like(sre)
    first: dict[int, int] = {}
    for c, nf in enumerate(n_folded):
        F = st.folded[:nf]
        if not F:
            continue
        H = st.phiK[F].T @ st.V[F]
        s = st.phiK[F].sum(axis=0)
        sre[c, F] = self_recall_error(st.phiK[F], st.V[F], H, s)
        for i in F:
            first.setdefault(i, c)
            rel[c, i] = sre[c, i] - sre[first[i], i]
    return sre, rel

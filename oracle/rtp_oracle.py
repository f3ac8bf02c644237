"""CPU oracle for the RTPurbo inference path -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, the package's ``__graft_entry__.smoke()`` check and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never imports, links or calls it,
and this module imports nothing from the product.

Everything is plain NumPy in float64, one query at a time, in the order the
pages give the method.  The pages that define what is computed:

* [A] "Full Attention Strikes Back: Transferring Full Attention into Sparse
  within Hundred Training Steps (RTPurbo)" (research-wiki page), TL;DR and
  "Key findings": retrieval heads keep the full KV cache, a lightweight
  16-dimensional token indexer picks tokens, dynamic top-p replaces top-k.
* [B] "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a
  Few Hundred Training Steps" (forum post), "Three Key Insights":
  1 - retrieval heads keep the full KV cache, local heads keep only a local
  window; 2 - a 16-dimensional low-frequency projection of rotary
  coordinates ranks tokens; 3 - cumulative top-p selection per query.
  "The RTPurbo Method" 2: projection-based top-p rankings stand in for the
  full-dimension ones.
* [C] arXiv abstract (aiqbench page, "Full Attention Strikes Back..."),
  observations (1)-(3): the same three statements.

Readings where the pages are silent (each one is a choice of this build):

R1  indexer score s_j = (P q) . (P k_j) / 4, i.e. the 16-dim dot product
    scaled by 1/sqrt(16); P is applied to post-rotary q and k.
R2  the top-p mass is the softmax over the indexer scores s (no other
    temperature); the selected set is the smallest prefix of the keys
    ordered by (s descending, position ascending) whose mass reaches p*Z.
R3  ties in s are broken by lower position first.
R4  p >= 1 selects every candidate; p <= 0 is invalid.
R5  decode candidates are positions 0..n-1 of the sequence (the current
    token's key included); a prefill query at position i sees 0..i.
R6  retrieval heads attend exactly their selected set (no added window or
    sink); local heads attend the last W keys up to and including their own
    position.
R7  attention is softmax(q.k / sqrt(128)) over the attended keys, with the
    full 128-dim q and k, renormalised over that set; an empty set gives 0.
R8  query head h reads KV head h // G (grouped-query attention).
R9  the projected keys are stored in the workload's storage type (bf16,
    round-to-nearest-even, or fp32) and the scores are computed from the
    stored values; the oracle's own bf16 rounding below is written from the
    IEEE definition.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

D_IDX = 16
INDEXER_SCALE = 0.25  # R1: 1/sqrt(16)


# --------------------------------------------------------------------------
# storage rounding (R9)
# --------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), as float64.

    bf16 keeps 8 significant bits: for |x| in [2^e, 2^(e+1)) the spacing is
    2^(e-7).  Below the smallest normal (2^-126) the spacing stays 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    _, e2 = np.frexp(x[nz])               # x = m * 2^e2, 0.5 <= |m| < 1
    e = np.maximum(e2.astype(np.int64) - 1, -126)
    ulp = np.ldexp(1.0, e - 7)
    out[nz] = np.rint(x[nz] / ulp) * ulp  # np.rint: round half to even
    return out


def round_storage(x: np.ndarray, storage: str) -> np.ndarray:
    if storage == "bf16":
        return round_bf16(x)
    if storage == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    if storage == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(storage)


# --------------------------------------------------------------------------
# step 1: the 16-dim token indexer ([B] insight 2, [A] TL;DR)
# --------------------------------------------------------------------------

def index_project(x: np.ndarray, P: np.ndarray, storage: str = "f64") -> np.ndarray:
    """x_idx = P x for each row of x[..., 128]; P is [16, 128].  Rounded to ``storage``."""
    x = np.asarray(x, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    return round_storage(x @ P.T, storage)


def indexer_scores(q_idx: np.ndarray, k_idx: np.ndarray) -> np.ndarray:
    """s_j = (q_idx . k_idx[j]) / 4 for every candidate row j (R1)."""
    q_idx = np.asarray(q_idx, dtype=np.float64)
    k_idx = np.asarray(k_idx, dtype=np.float64)
    return (k_idx @ q_idx) * INDEXER_SCALE


# --------------------------------------------------------------------------
# step 2: dynamic top-p ([B] insight 3, [C] observation 3)
# --------------------------------------------------------------------------

@dataclass
class Selection:
    """The selected set of one query.

    idx     selected key positions, ascending
    count   |S|
    tau     score of the last key taken in (s desc, pos asc) order (the cut score)
    tiepos  position of that key: a key j is selected iff s_j > tau, or
            s_j == tau and j <= tiepos
    Z       sum over all candidates of exp(s - max s)
    mass    sum over S of exp(s - max s)
    order   all candidate positions in (s desc, pos asc) order
    """

    idx: np.ndarray
    count: int
    tau: float
    tiepos: int
    Z: float
    mass: float
    order: np.ndarray


def topp_select(s: np.ndarray, p: float) -> Selection:
    """Smallest set of keys, taken in (score desc, position asc) order, whose
    softmax-over-s mass reaches p (R2-R4).  ``s`` holds the candidates' scores,
    candidate j at position j."""
    s = np.asarray(s, dtype=np.float64)
    n = s.shape[0]
    if not (p > 0.0):
        raise ValueError("p must be > 0")
    if n == 0:
        return Selection(np.zeros(0, np.int64), 0, float("-inf"), -1, 0.0, 0.0, np.zeros(0, np.int64))
    # softmax over the indexer scores: weights relative to the largest score
    w = np.exp(s - s.max())
    Z = float(w.sum())
    # order by score descending, then position ascending (np.lexsort: last key is primary)
    pos = np.arange(n)
    order = np.lexsort((pos, -s))
    if p >= 1.0:
        k = n
    else:
        cum = np.cumsum(w[order])
        k = int(np.searchsorted(cum, p * Z, side="left")) + 1  # first k with cum[k-1] >= p*Z
        k = min(k, n)
    chosen = order[:k]
    last = int(order[k - 1])
    return Selection(idx=np.sort(chosen), count=k, tau=float(s[last]), tiepos=last,
                     Z=Z, mass=float(w[chosen].sum()), order=order)


def topk_select(s: np.ndarray, k: int) -> Selection:
    """The fixed top-k budget the pages set dynamic top-p against ([A] "Key
    findings", [B] insight 3): the min(k, n) keys of highest score, ties taken
    by lower position (R3).  Same fields as ``topp_select`` (Z and mass are the
    softmax masses of that set, for comparison)."""
    s = np.asarray(s, dtype=np.float64)
    n = s.shape[0]
    if k < 1:
        raise ValueError("k must be >= 1")
    if n == 0:
        return Selection(np.zeros(0, np.int64), 0, float("-inf"), -1, 0.0, 0.0, np.zeros(0, np.int64))
    w = np.exp(s - s.max())
    order = np.lexsort((np.arange(n), -s))
    kk = min(k, n)
    chosen = order[:kk]
    last = int(order[kk - 1])
    return Selection(idx=np.sort(chosen), count=kk, tau=float(s[last]), tiepos=last,
                     Z=float(w.sum()), mass=float(w[chosen].sum()), order=order)


# --------------------------------------------------------------------------
# step 3: attention over a key set ([A] TL;DR "sparse attention", R7)
# --------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, scale: float) -> np.ndarray:
    """softmax_j(q . K[j] * scale) weighted sum of V[j] over j in idx (float64)."""
    q = np.asarray(q, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size == 0:
        return np.zeros(q.shape[-1], dtype=np.float64)
    Ks = np.asarray(K[idx], dtype=np.float64)
    Vs = np.asarray(V[idx], dtype=np.float64)
    logits = (Ks @ q) * scale
    e = np.exp(logits - logits.max())
    return (e[:, None] * Vs).sum(axis=0) / e.sum()


def attend_lse(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray,
               scale: float) -> Tuple[np.ndarray, float]:
    """attend() over idx, and ln sum_j exp(q . K[j] * scale) over the same keys
    (-inf for an empty set): what one device reports for the keys it holds
    when a sequence's keys are split by position over several devices."""
    o = attend(q, K, V, idx, scale)
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size == 0:
        return o, -np.inf
    logits = (np.asarray(K[idx], dtype=np.float64) @ np.asarray(q, dtype=np.float64)) * scale
    m = logits.max()
    return o, float(m + np.log(np.exp(logits - m).sum()))


def combine_partials(parts: Sequence[Tuple[np.ndarray, float]]) -> np.ndarray:
    """Attention over a union of disjoint key sets from the per-set results
    (o_s, lse_s): softmax weights over the union split as exp(lse_s) per set,
    so o = sum_s exp(lse_s) o_s / sum_s exp(lse_s); all sets empty gives 0."""
    lses = np.array([lse for _, lse in parts], dtype=np.float64)
    if lses.size == 0 or np.all(np.isneginf(lses)):
        return np.zeros(np.asarray(parts[0][0]).shape if parts else 0, dtype=np.float64)
    m = lses.max()
    w = np.exp(lses - m)
    return sum(wi * np.asarray(o, dtype=np.float64) for wi, (o, _) in zip(w, parts)) / w.sum()


def window_keys(pos: int, W: int) -> np.ndarray:
    """Local-head keys of a query at ``pos``: the last W positions up to pos ([B] insight 1, R6)."""
    if W < 1:
        raise ValueError("W must be >= 1")
    return np.arange(max(0, pos - W + 1), pos + 1, dtype=np.int64)


# --------------------------------------------------------------------------
# the layer: retrieval heads -> indexer, top-p, sparse attention;
#            local heads -> window attention ([B] insights 1-3)
# --------------------------------------------------------------------------

@dataclass
class QueryResult:
    o: np.ndarray                  # [128] float64
    sel: Optional[Selection]       # None for local heads
    scores: Optional[np.ndarray]   # indexer scores of the candidates (retrieval heads)


def retrieval_query(q: np.ndarray, q_idx: np.ndarray, K: np.ndarray, V: np.ndarray,
                    K_idx: np.ndarray, pos: int, p: float, scale: float) -> QueryResult:
    """One retrieval-head query at position ``pos``: candidates 0..pos (R5)."""
    if pos < 0:
        return QueryResult(np.zeros(q.shape[-1]), topp_select(np.zeros(0), p), np.zeros(0))
    s = indexer_scores(q_idx, K_idx[: pos + 1])
    sel = topp_select(s, p)
    return QueryResult(attend(q, K, V, sel.idx, scale), sel, s)


def local_query(q: np.ndarray, K: np.ndarray, V: np.ndarray, pos: int, W: int, scale: float) -> QueryResult:
    if pos < 0:
        return QueryResult(np.zeros(q.shape[-1]), None, None)
    return QueryResult(attend(q, K, V, window_keys(pos, W), scale), None, None)


class LayerOracle:
    """The whole path for one layer, evaluated lazily query by query.

    q [B, Hq, T, D], k/v [B, Hkv, N, D], P [R, 16, D]; the first R KV heads are
    retrieval heads; lens[b] keys in sequence b; its T queries sit at
    positions lens[b] - T .. lens[b] - 1.
    """

    def __init__(self, q, k, v, P, lens, R: int, W: int, p: float, storage: str,
                 scale: Optional[float] = None):
        self.q, self.k, self.v, self.P = q, k, v, np.asarray(P, np.float64)
        self.B, self.Hq, self.T, self.D = q.shape
        self.Hkv, self.N = k.shape[1], k.shape[2]
        self.G = self.Hq // self.Hkv
        self.R, self.W, self.p, self.storage = R, W, p, storage
        self.lens = np.asarray(lens, dtype=np.int64)
        self.scale = (1.0 / np.sqrt(self.D)) if scale is None else scale
        self._kidx: Dict[Tuple[int, int], np.ndarray] = {}

    def is_retrieval(self, h: int) -> bool:
        return h // self.G < self.R

    def pos(self, b: int, t: int) -> int:
        return int(self.lens[b]) - self.T + t

    def k_idx(self, b: int, kvh: int) -> np.ndarray:
        """Projected keys of a retrieval KV head, rounded to storage (computed once)."""
        key = (b, kvh)
        if key not in self._kidx:
            n = int(self.lens[b])
            self._kidx[key] = index_project(self.k[b, kvh, :n], self.P[kvh], self.storage)
        return self._kidx[key]

    def q_idx(self, b: int, h: int, t: int) -> np.ndarray:
        return index_project(self.q[b, h, t], self.P[h // self.G], self.storage)

    def query(self, b: int, h: int, t: int) -> QueryResult:
        kvh = h // self.G
        K, V = self.k[b, kvh], self.v[b, kvh]
        pos = self.pos(b, t)
        if self.is_retrieval(h):
            return retrieval_query(self.q[b, h, t], self.q_idx(b, h, t), K, V, self.k_idx(b, kvh),
                                   pos, self.p, self.scale)
        return local_query(self.q[b, h, t], K, V, pos, self.W, self.scale)

    def run(self, queries: Optional[Sequence[Tuple[int, int, int]]] = None):
        """Outputs (and selections) for ``queries`` (all of them by default)."""
        if queries is None:
            queries = [(b, h, t) for b in range(self.B) for h in range(self.Hq) for t in range(self.T)]
        return {key: self.query(*key) for key in queries}


def needle_recall(results: Dict[Tuple[int, int, int], QueryResult],
                  needles: List[Tuple[int, int, int, int, int]]) -> Tuple[int, int]:
    """(recalled, total) planted needles whose key is in their query's selected set."""
    hit = tot = 0
    for b, _kvh, h, t, j in needles:
        r = results.get((b, h, t))
        if r is None or r.sel is None:
            continue
        tot += 1
        hit += int(np.isin(j, r.sel.idx))
    return hit, tot

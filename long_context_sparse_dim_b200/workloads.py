"""Seeded synthetic inputs for the RTPurbo sparse-attention path.

This module only *draws* inputs: queries, keys and values after rotary
position embedding, planted "needle" keys, the 16-row low-frequency
projection and the head split.  It holds none of the method's arithmetic
(no indexer score, no top-p cut, no attention), so both the CUDA path and
the CPU oracle can be fed from it without sharing any of the method's code.

Shapes follow a Llama-3-8B-like attention layer (32 query heads, 8 KV heads,
GQA 4:1, head_dim 128, RoPE base 500000).  The pages fix only the 16-dim
indexer built from low-frequency rotary coordinates ("RTPurbo: Turning Dense
LLMs into Sparse Attention Models with Just a Few Hundred Training Steps",
"Three Key Insights" 2) and the split into a few retrieval heads and many
local heads (same page, insight 1); everything else here is a stated
synthetic recipe.

Conventions
-----------
* Rotary pairing is the half-split ("rotate_half") form: coordinate i pairs
  with i+64, angle pos * base**(-2i/128).  The 8 lowest-frequency pairs are
  i = 56..63, so the projection selects dims 56..63 and 120..127.
* Needles are planted in pre-rotary content space, ``k = 3 q/|q| + 0.3 eps``
  with ``q`` the pre-rotary query of the targeted head and token, and then
  rotated at the needle's own position, like every other key.
* Retrieval KV heads are the first ``R`` KV heads; query head ``h`` reads KV
  head ``h // G``.  So retrieval query heads are ``0 .. R*G-1``.
* Queries are the last ``T`` tokens of an ``N``-token context: token ``t`` of
  sequence ``b`` sits at position ``lens[b] - T + t``.
* Every array is drawn from its own PCG64 stream keyed by
  ``SeedSequence([seed, tag, b, head])`` so a single head can be regenerated
  without drawing the rest (the oracle's sampled checks rely on that).
* bf16 workloads store float32 arrays whose values are exactly bf16
  (round-to-nearest-even); ``bf16_bits`` gives the 16-bit patterns to upload.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

D_HEAD = 128
D_IDX = 16
ROPE_BASE = 500000.0

# Stream tags (one PCG64 stream per tag, batch element and head).
_TAG_Q, _TAG_K, _TAG_V, _TAG_NEEDLE_POS, _TAG_NEEDLE_NOISE, _TAG_LENS = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Workload:
    """One synthetic attention-layer workload.

    mode      "decode" (T == 1) or "prefill" (T > 1; causal, chunked when T < N)
    B         batch size
    Hq, Hkv   query / KV heads (G = Hq // Hkv query heads share a KV head)
    R         number of retrieval KV heads (the first R); the rest are local
    N         context length (keys in the cache, current tokens included)
    T         query tokens per sequence (the last T positions)
    W         local sliding window (keys including the query's own position)
    p         top-p mass
    dtype     "f32" or "bf16" storage of q/k/v and of the projected keys
    needles   decode: needles per retrieval query head (int) or a tuple of
              choices drawn per query; prefill: see ``needle_mode``
    needle_mode  "per_query" (decode), "fraction" (prefill: a fraction of
              tokens get one needle each) or "strata" (prefill: a count per
              retrieval KV head spread over equal strata of the prefix)
    needle_fraction / needle_count  parameters of the prefill modes
    ragged    if True, sequence lengths are drawn in [N/2, N] per batch
              element (decode only); otherwise every sequence has N tokens
    seed      base seed
    """

    name: str
    mode: str
    B: int
    Hq: int
    Hkv: int
    R: int
    N: int
    T: int
    W: int
    p: float
    dtype: str
    needles: object = 0
    needle_mode: str = "per_query"
    needle_fraction: float = 0.0
    needle_count: int = 0
    ragged: bool = False
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def Hq_ret(self) -> int:
        return self.R * self.G

    @property
    def L(self) -> int:
        return self.Hkv - self.R

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the measurements are quoted on, by shape.
DECODE_N4K_F32 = Workload(
    name="decode_b1_n4096_f32_1ret1loc", mode="decode", B=1, Hq=2, Hkv=2, R=1,
    N=4096, T=1, W=512, p=0.9, dtype="f32", needles=16, seed=0)
DECODE_B8_N32K = Workload(
    name="decode_b8_n32768_llama8b_2ret6loc", mode="decode", B=8, Hq=32, Hkv=8, R=2,
    N=32768, T=1, W=4096, p=0.95, dtype="bf16", needles=64, seed=1)
DECODE_B4_N128K = Workload(
    name="decode_b4_n131072_llama8b_2ret6loc", mode="decode", B=4, Hq=32, Hkv=8, R=2,
    N=131072, T=1, W=4096, p=0.95, dtype="bf16", needles=(4, 64, 1024), seed=2)
PREFILL_N32K = Workload(
    name="prefill_t32768_llama8b_2ret6loc", mode="prefill", B=1, Hq=32, Hkv=8, R=2,
    N=32768, T=32768, W=4096, p=0.95, dtype="bf16", needle_mode="fraction",
    needle_fraction=0.10, seed=3)
# Same layer and recipe at 8192 tokens: small enough for detailed profiler captures.
PREFILL_N8K = Workload(
    name="prefill_t8192_llama8b_2ret6loc", mode="prefill", B=1, Hq=32, Hkv=8, R=2,
    N=8192, T=8192, W=4096, p=0.95, dtype="bf16", needle_mode="fraction",
    needle_fraction=0.10, seed=5)
PREFILL_CHUNK_1M = Workload(
    name="prefill_chunk_t8192_n1048576_llama8b_2ret6loc", mode="prefill", B=1, Hq=32,
    Hkv=8, R=2, N=1048576, T=8192, W=8192, p=0.95, dtype="bf16", needle_mode="strata",
    needle_count=256, seed=4)

WORKLOADS: Dict[str, Workload] = {w.name: w for w in (
    DECODE_N4K_F32, DECODE_B8_N32K, DECODE_B4_N128K, PREFILL_N32K, PREFILL_N8K, PREFILL_CHUNK_1M)}


# --------------------------------------------------------------------------
# helpers (input synthesis only)
# --------------------------------------------------------------------------

def _rng(seed: int, tag: int, b: int = 0, h: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, b, h])))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest-even bf16 value, returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> 16) & 1
    r = ((u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Top 16 bits of float32 values that are exactly bf16 (uint16 array)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("array holds values that are not exactly bf16")
    return (u >> 16).astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rope_inv_freq(d: int = D_HEAD, base: float = ROPE_BASE) -> np.ndarray:
    """theta_i = base**(-2i/d), i in [0, d/2)."""
    return base ** (-np.arange(0, d // 2, dtype=np.float64) * 2.0 / d)


def apply_rope(x: np.ndarray, positions: np.ndarray, base: float = ROPE_BASE) -> np.ndarray:
    """Half-split rotary embedding of ``x[..., n, d]`` at ``positions[n]`` (float32 out)."""
    d = x.shape[-1]
    half = d // 2
    out = np.empty(x.shape, dtype=np.float32)
    inv = rope_inv_freq(d, base)
    pos = np.asarray(positions, dtype=np.float64)
    step = 1 << 16
    for s in range(0, pos.shape[0], step):
        ang = pos[s:s + step, None] * inv[None, :]
        c = np.cos(ang).astype(np.float32)
        sn = np.sin(ang).astype(np.float32)
        x1 = x[..., s:s + step, :half]
        x2 = x[..., s:s + step, half:]
        out[..., s:s + step, :half] = x1 * c - x2 * sn
        out[..., s:s + step, half:] = x2 * c + x1 * sn
    return out


def lowfreq_dims(d: int = D_HEAD, d_idx: int = D_IDX) -> np.ndarray:
    """The d_idx rotary coordinates with the lowest rotation frequency."""
    half = d // 2
    pairs = np.arange(half - d_idx // 2, half)          # 56..63 for d=128, d_idx=16
    return np.concatenate([pairs, pairs + half])       # dims 56..63, 120..127


def lowfreq_projection(d: int = D_HEAD, d_idx: int = D_IDX) -> np.ndarray:
    """P[d_idx, d]: coordinate selection of the low-frequency rotary dims."""
    P = np.zeros((d_idx, d), dtype=np.float32)
    P[np.arange(d_idx), lowfreq_dims(d, d_idx)] = 1.0
    return P


# --------------------------------------------------------------------------
# the generated instance
# --------------------------------------------------------------------------

@dataclass
class Instance:
    """A drawn workload.  Arrays are float32; bf16 workloads hold bf16 values.

    q     [B, Hq, T, D]   post-rotary queries
    k, v  [B, Hkv, N, D]  post-rotary keys, values
    P     [R, 16, D]      projection of each retrieval KV head
    lens  [B] int32       keys per sequence (== N unless ragged)
    needles  list of (b, kv_head, q_head, t, key_pos)
    """

    wl: Workload
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    P: np.ndarray
    lens: np.ndarray
    needles: List[Tuple[int, int, int, int, int]] = field(default_factory=list)

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(D_HEAD))

    def q_positions(self, b: int) -> np.ndarray:
        return np.arange(self.wl.T) + int(self.lens[b]) - self.wl.T


def _round(wl: Workload, x: np.ndarray) -> np.ndarray:
    return round_to_bf16(x) if wl.dtype == "bf16" else x.astype(np.float32)


def _draw_lens(wl: Workload) -> np.ndarray:
    if not wl.ragged:
        return np.full((wl.B,), wl.N, dtype=np.int32)
    rng = _rng(wl.seed, _TAG_LENS)
    lo = max(wl.T, wl.N // 2)
    lens = rng.integers(lo, wl.N + 1, size=wl.B).astype(np.int32)
    lens[-1] = wl.N  # the longest sequence fixes N
    return lens


def _plan_needles(wl: Workload, lens: np.ndarray) -> List[Tuple[int, int, int, int, int]]:
    """Needle placements (b, kv_head, q_head, t, key_pos); positions are distinct per (b, kv_head)."""
    out: List[Tuple[int, int, int, int, int]] = []
    G = wl.G
    for b in range(wl.B):
        n_b = int(lens[b])
        for kvh in range(wl.R):
            rng = _rng(wl.seed, _TAG_NEEDLE_POS, b, kvh)
            heads = list(range(kvh * G, (kvh + 1) * G))
            if wl.mode == "decode":
                if isinstance(wl.needles, tuple):
                    counts = [int(rng.choice(wl.needles)) for _ in heads]
                else:
                    counts = [int(wl.needles)] * len(heads)
                total = sum(counts)
                avail = n_b - 1                      # the query's own position is excluded
                total = min(total, avail)
                pos = rng.choice(avail, size=total, replace=False)
                i = 0
                for h, c in zip(heads, counts):
                    for _ in range(c):
                        if i >= total:
                            break
                        out.append((b, kvh, h, 0, int(pos[i])))
                        i += 1
            elif wl.needle_mode == "fraction":
                q0 = n_b - wl.T
                cand = [t for t in range(wl.T) if q0 + t >= 1]
                n_sel = int(round(wl.needle_fraction * len(cand)))
                toks = np.sort(rng.choice(cand, size=n_sel, replace=False)) if n_sel else []
                used = set()
                for t in toks:
                    h = int(rng.choice(heads))
                    qpos = q0 + int(t)
                    for _ in range(64):
                        j = int(rng.integers(0, qpos))
                        if j not in used:
                            break
                    if j in used:
                        continue
                    used.add(j)
                    out.append((b, kvh, h, int(t), j))
            elif wl.needle_mode == "strata":
                span = n_b - wl.T
                n = min(wl.needle_count, max(span, 0))
                for s in range(n):
                    lo = s * span // n
                    hi = (s + 1) * span // n
                    j = int(rng.integers(lo, max(hi, lo + 1)))
                    t = int(rng.integers(0, wl.T))
                    h = int(rng.choice(heads))
                    out.append((b, kvh, h, t, j))
            else:
                raise ValueError(wl.needle_mode)
    return out


def generate(wl: Workload, heads_kv: Optional[List[int]] = None) -> Instance:
    """Draw ``wl``.  ``heads_kv`` restricts k/v (and their query heads) to some KV heads;
    the other heads are left zero.  Values for the drawn heads do not depend on it."""
    B, Hq, Hkv, N, T, D, G = wl.B, wl.Hq, wl.Hkv, wl.N, wl.T, D_HEAD, wl.G
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    kv_list = list(range(Hkv)) if heads_kv is None else list(heads_kv)
    lens = _draw_lens(wl)
    q_pre = np.zeros((B, Hq, T, D), dtype=np.float32)
    for b in range(B):
        for kvh in kv_list:
            for h in range(kvh * G, (kvh + 1) * G):
                q_pre[b, h] = _rng(wl.seed, _TAG_Q, b, h).standard_normal((T, D), dtype=np.float32)
    k_pre = np.zeros((B, Hkv, N, D), dtype=np.float32)
    v = np.zeros((B, Hkv, N, D), dtype=np.float32)
    for b in range(B):
        for kvh in kv_list:
            k_pre[b, kvh] = _rng(wl.seed, _TAG_K, b, kvh).standard_normal((N, D), dtype=np.float32)
            v[b, kvh] = _rng(wl.seed, _TAG_V, b, kvh).standard_normal((N, D), dtype=np.float32)
    needles = _plan_needles(wl, lens)
    for b, kvh, h, t, j in needles:
        if kvh not in kv_list:
            continue
        eps = _rng(wl.seed, _TAG_NEEDLE_NOISE, b, kvh * 1_000_003 + j).standard_normal(D, dtype=np.float32)
        qv = q_pre[b, h, t].astype(np.float64)
        k_pre[b, kvh, j] = (3.0 * qv / np.linalg.norm(qv) + 0.3 * eps).astype(np.float32)
    q = np.zeros_like(q_pre)
    k = np.zeros_like(k_pre)
    for b in range(B):
        qpos = np.arange(T) + int(lens[b]) - T
        for kvh in kv_list:
            k[b, kvh] = _round(wl, apply_rope(k_pre[b, kvh], np.arange(N)))
            v[b, kvh] = _round(wl, v[b, kvh])
            for h in range(kvh * G, (kvh + 1) * G):
                q[b, h] = _round(wl, apply_rope(q_pre[b, h], qpos))
    P = np.stack([lowfreq_projection()] * wl.R) if wl.R else np.zeros((0, D_IDX, D), np.float32)
    return Instance(wl=wl, q=q, k=k, v=v, P=P, lens=lens, needles=needles)


def small(wl: Workload, **kw) -> Workload:
    """A scaled-down copy of ``wl`` for tests (same structure, smaller sizes)."""
    return wl.replace(**kw)

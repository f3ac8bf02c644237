"""Decode of long sequences whose keys are split by position over the ranks of
a process group (one rank per GPU).

Retrieval heads keep the full KV cache ("RTPurbo: Turning Dense LLMs into
Sparse Attention Models ...", "Three Key Insights" 1), so at a million tokens
their K/V rows dominate a decode step's HBM traffic.  Splitting the positions
0 .. N-1 into one contiguous range per rank divides that traffic by the
number of ranks.  What every rank does in one step:

  1. replicated: project the queries (rtp_index_project) and run the exact
     top-p selection over the FULL projected-key cache (rtp_topp_select).  The
     projected keys are 32 bytes per key and head against 512 for the K/V rows,
     so every rank keeps all of them, and the deterministic selection gives
     identical bits on every rank: the cut needs no exchange;
  2. its range: attention of the retrieval heads over the selected keys among
     its rows, with the log-sum-exp of each row (rtp_sparse_attn_decode_range);
     its share of the local heads: window attention over their last W keys
     (every rank holds the local heads' W-row windows; rank r computes a
     contiguous block of them and reports lse 0 for those heads, -inf for the
     others, so the merge passes its result through);
  3. one all-gather of the per-rank (output, lse) rows: (128 + 1) floats per
     (sequence, query head) and rank;
  4. the merge (rtp_attn_combine), identical on every rank.

The exchange is that one small collective per step; it runs over NCCL (NVLink
/ NVSwitch) on GPUs and over gloo in the CPU tests of this module's host
logic.  ``ops`` lets those tests substitute CPU implementations of the five
library calls; the default is the library itself.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

KEY_ALIGN = 64  # rtp_sparse_attn_decode_range takes ranges starting at multiples of 64


def key_ranges(N: int, world: int, align: int = KEY_ALIGN) -> List[Tuple[int, int]]:
    """(key_lo, rows) of each rank: equal ranges of `rows` positions, a multiple
    of `align`, covering 0 .. N-1 (the last range may run past N)."""
    if N < 1 or world < 1:
        raise ValueError("need N >= 1 and world >= 1")
    per = -(-N // world)
    rows = -(-per // align) * align
    return [(r * rows, rows) for r in range(world)]


def local_head_block(L: int, world: int, rank: int) -> Tuple[int, int]:
    """The contiguous block [l0, l1) of the L local KV heads that `rank` computes."""
    return rank * L // world, (rank + 1) * L // world


class KeyRangeDecodeLayer:
    """One rank's share of a decode step (see the module docstring).

    q        [B, Hq, 1, D] all query heads (the same on every rank)
    k_range, v_range  [B, R, rows, D] retrieval-head rows key_lo .. key_lo + rows - 1
    k_idx    [B, R, N, 16] projected keys of every position (the same on every rank)
    P        [R, 16, D] f32
    k_win, v_win  [B, L, Wc, D] the local heads' window rows (for instance the
             rings rtp_kv_append keeps), win_lens [B] their row counts
    lens     [B] int32 sequence lengths (whole sequences)
    """

    def __init__(self, q, k_range, v_range, k_idx, P, key_lo: int, k_win, v_win, win_lens, lens,
                 R: int, W: int, p: float, group=None, ops=None, out_dtype: torch.dtype = torch.float32,
                 scale: Optional[float] = None):
        if ops is None:
            from . import rtp as ops
        self.ops = ops
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        B, Hq, _, D = q.shape
        Hkv = R + k_win.shape[1]
        G = Hq // Hkv
        self.B, self.Hq, self.Hkv, self.G, self.R, self.W, self.D = B, Hq, Hkv, G, R, W, D
        self.p = float(p)
        self.scale = (D ** -0.5) if scale is None else scale
        self.key_lo = int(key_lo)
        self.q, self.k_range, self.v_range, self.k_idx, self.P = q, k_range, v_range, k_idx, P
        self.k_win, self.v_win, self.win_lens, self.lens = k_win, v_win, win_lens, lens
        dev = q.device
        N = k_idx.shape[2]
        Hr = R * G
        self.q_ret = q[:, :Hr]
        self.q_idx = torch.zeros(B, Hr, 1, 16, dtype=k_idx.dtype, device=dev)
        self.sel = ops.Selection.empty(B * Hr, N, dev)
        # this rank's (output, lse) rows, and everyone's after the all-gather
        n_o = B * Hq * D
        self.part = torch.zeros(n_o + B * Hq, dtype=torch.float32, device=dev)
        self.o_part = self.part[:n_o].view(B, Hq, 1, D)
        self.lse_part = self.part[n_o:].view(B, Hq)
        self.gathered = torch.zeros(self.world * (n_o + B * Hq), dtype=torch.float32, device=dev)
        rows = self.gathered.view(self.world, n_o + B * Hq)
        self.o_all = rows[:, :n_o].view(self.world, B, Hq, D)
        self.lse_all = rows[:, n_o:].view(self.world, B, Hq)
        self.o = torch.zeros(B, Hq, 1, D, dtype=out_dtype, device=dev)
        L = Hkv - R
        self.l0, self.l1 = local_head_block(L, self.world, self.rank)
        own = torch.full((B, L * G), float("-inf"), dtype=torch.float32)
        own[:, self.l0 * G: self.l1 * G] = 0.0
        self.lse_part[:, Hr:].copy_(own.to(dev))
        self.ws_sel = ops.workspace(ops.topp_select_workspace_size(B, Hr, 1, R, N), dev)
        self.ws_ret = ops.workspace(ops.sparse_attn_decode_workspace_size(B, Hr, R, k_range.shape[2]), dev)
        nl = self.l1 - self.l0
        self.ws_win = (ops.workspace(ops.window_attn_workspace_size(B, nl * G, 1, nl, k_win.shape[2], W), dev)
                       if nl else None)

    def step(self) -> torch.Tensor:
        """One decode step on the current stream (the collective's too); returns
        o [B, Hq, 1, D], the same on every rank."""
        ops, G, Hr = self.ops, self.G, self.R * self.G
        stream = None
        ops.index_project(self.q_ret, self.P, self.q_idx, stream)
        ops.topp_select(self.q_idx, self.k_idx, self.lens, self.p, self.sel, self.ws_sel, stream)
        ops.sparse_attn_decode_range(self.q_ret, self.k_range, self.v_range, self.lens, self.sel, self.key_lo,
                                     self.scale, self.o_part[:, :Hr], self.lse_part[:, :Hr], self.ws_ret, stream)
        if self.l1 > self.l0:
            h0, h1 = Hr + self.l0 * G, Hr + self.l1 * G
            ops.window_attn(self.q[:, h0:h1], self.k_win[:, self.l0:self.l1], self.v_win[:, self.l0:self.l1],
                            self.win_lens, self.W, self.scale, self.o_part[:, h0:h1], self.ws_win, stream)
        dist.all_gather_into_tensor(self.gathered, self.part, group=self.group)
        ops.attn_combine(self.o_all, self.lse_all, self.o, stream)
        return self.o

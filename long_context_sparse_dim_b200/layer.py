"""One attention layer's RTPurbo decode step, sequenced over the C ABI.

Holds the device buffers of one layer (KV cache views, projected-key cache,
selection, outputs, workspaces) and issues the calls of one decode step:

    a1  rtp_index_project   newest key row -> projected-key cache; queries -> q_idx
    a3  rtp_topp_select     indexer scores + dynamic top-p cut (retrieval heads)
    a4  rtp_sparse_attn_decode   attention over the selected keys
    a5  rtp_window_attn     sliding-window attention (local heads)

The first R KV heads are the retrieval heads ("RTPurbo: Turning Dense LLMs
into Sparse Attention Models ...", "Three Key Insights" 1); every step of the
computation runs in librtp.so.  ``DecodeLayer`` works on a resident cache of
all heads, ``CachedDecodeLayer`` keeps its own caches (full for the retrieval
heads, a W-row ring for the local heads) and appends each step's new token.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import rtp


class DecodeLayer:
    def __init__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: torch.Tensor,
                 R: int, W: int, p: float, lens: Optional[torch.Tensor] = None,
                 out_dtype: torch.dtype = torch.float32, scale: Optional[float] = None):
        B, Hq, T, D = q.shape
        _, Hkv, N, _ = k.shape
        if T != 1:
            raise ValueError("decode takes one query token per sequence")
        self.B, self.Hq, self.Hkv, self.N, self.D = B, Hq, Hkv, N, D
        self.G = Hq // Hkv
        self.R, self.W, self.p = R, W, float(p)
        self.scale = (D ** -0.5) if scale is None else scale
        dev = q.device
        G = self.G
        self.q, self.k, self.v, self.P = q, k, v, P
        self.lens = lens
        self.lens_host = None if lens is None else [int(x) for x in lens.cpu().tolist()]
        self.q_ret, self.q_loc = q[:, : R * G], q[:, R * G:]
        self.k_ret, self.v_ret = k[:, :R], v[:, :R]
        self.k_loc, self.v_loc = k[:, R:], v[:, R:]
        self.o = torch.zeros(B, Hq, 1, D, dtype=out_dtype, device=dev)
        self.o_ret, self.o_loc = self.o[:, : R * G], self.o[:, R * G:]
        idx_dtype = k.dtype
        self.k_idx = torch.zeros(B, R, N, 16, dtype=idx_dtype, device=dev)
        self.q_idx = torch.zeros(B, R * G, 1, 16, dtype=idx_dtype, device=dev)
        self.sel = rtp.Selection.empty(B * R * G, N, dev)
        self.ws_sel = rtp.workspace(rtp.topp_select_workspace_size(B, R * G, 1, R, N), dev)
        self.ws_ret = rtp.workspace(rtp.sparse_attn_decode_workspace_size(B, R * G, R, N), dev) if R else None
        self.ws_loc = (rtp.workspace(rtp.window_attn_workspace_size(B, Hq - R * G, 1, Hkv - R, N, W), dev)
                       if Hkv > R else None)
        self._plans = {}
        self._host_graphs = {}  # host_step: (graph, stream) per set of host buffers

    def build_index(self, stream=None) -> None:
        """Project every cached key of the retrieval heads (done once, before decoding)."""
        if self.R:
            rtp.index_project(self.k_ret, self.P, self.k_idx, stream)

    def _plan(self, main: torch.cuda.Stream, side: Optional[torch.cuda.Stream], new_rows=None):
        """The step's C-ABI calls with their arguments marshalled once, for
        this pair of streams: projections, window attention, and the chain
        selection -> sparse attention.  With ``new_rows`` = (k_new, v_new, pos)
        the step first appends each sequence's new K/V row (staged on the
        device) at position pos[b] with rtp_kv_append, which also writes its
        projected key, in place of the projection of a row already in the cache."""
        pre, win, chain = [], [], []
        R, H = self.R, self.Hkv
        if new_rows is not None:
            k_new, v_new, pos = new_rows
            # the local heads' full caches serve as rings of N rows: position p goes to row p mod N = p
            pre.append(rtp.bind_kv_append(k_new, v_new, pos, R, self.P if R else None,
                                          self.k_ret if R else None, self.v_ret if R else None,
                                          self.k_idx if R else None, self.k_loc if H > R else None,
                                          self.v_loc if H > R else None, None, None, main))
        if self.R:
            if new_rows is None and self.lens_host is None:
                n = self.N
                pre.append(rtp.bind_index_project(self.k_ret[:, :, n - 1: n], self.P, self.k_idx[:, :, n - 1: n],
                                                  main))
            elif new_rows is None:
                for b, n in enumerate(self.lens_host):
                    if n > 0:
                        pre.append(rtp.bind_index_project(self.k_ret[b: b + 1, :, n - 1: n], self.P,
                                                          self.k_idx[b: b + 1, :, n - 1: n], main))
            pre.append(rtp.bind_index_project(self.q_ret, self.P, self.q_idx, main))
            chain.append(rtp.bind_topp_select(self.q_idx, self.k_idx, self.lens, self.p, self.sel, self.ws_sel, main))
            chain.append(rtp.bind_sparse_attn_decode(self.q_ret, self.k_ret, self.v_ret, self.lens, self.sel,
                                                     self.scale, self.o_ret, self.ws_ret, main))
        if self.Hkv > self.R:
            win.append(rtp.bind_window_attn(self.q_loc, self.k_loc, self.v_loc, self.lens, self.W, self.scale,
                                            self.o_loc, self.ws_loc, main if side is None else side))
        return pre, win, chain

    def step(self, stream=None, side_stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """One decode step over the resident cache; returns o [B, Hq, 1, D].

        With ``side_stream`` the local heads' window attention (which does not
        depend on the selection) runs there, forked from the main stream after
        the projections and joined back at the end: its CTAs share the SMs with
        the selection, which is bound by latency rather than by HBM traffic.
        The calls' arguments are marshalled on the first step with a given pair
        of streams and reused afterwards (the layer's buffers are fixed)."""
        main = torch.cuda.current_stream() if stream is None else stream
        key = (main.cuda_stream, None if side_stream is None else side_stream.cuda_stream)
        plan = self._plans.get(key)
        if plan is None:
            plan = self._plans[key] = self._plan(main, side_stream)
        self._run(plan, main, side_stream)
        return self.o

    @staticmethod
    def _run(plan, main, side_stream) -> None:
        pre, win, chain = plan
        for call in pre:
            call()
        if win and side_stream is not None:
            side_stream.wait_stream(main)
            for call in win:
                call()
            for call in chain:
                call()
            main.wait_stream(side_stream)
        else:
            for call in chain:
                call()
            for call in win:
                call()

    def host_step(self, h_q: torch.Tensor, h_k: torch.Tensor, h_v: torch.Tensor, h_o: torch.Tensor) -> torch.Tensor:
        """One decode step end to end from host memory: copy the new token's
        queries h_q [B, Hq, 1, D] and key/value rows h_k, h_v [B, Hkv, 1, D] (pinned
        host tensors of the cache dtype) in, run the step, copy the output to h_o
        [B, Hq, 1, D] (pinned) and wait for it.  The new rows land at each
        sequence's last position: they are copied to a contiguous device staging
        buffer and rtp_kv_append writes them into the caches together with the
        projected key (one launch, no strided host copies).  The first call with a
        set of buffers captures the copies and the calls in one CUDA graph (with
        the window attention on a forked stream); later calls replay it, so a token
        costs one graph launch and one synchronisation on the host."""
        key = (h_q.data_ptr(), h_k.data_ptr(), h_v.data_ptr(), h_o.data_ptr())
        ent = self._host_graphs.get(key)
        if ent is None:
            ent = self._host_graphs[key] = self._capture_host(h_q, h_k, h_v, h_o)
        graph, stream = ent
        graph.replay()
        stream.synchronize()
        return h_o

    def _capture_host(self, h_q, h_k, h_v, h_o):
        for t in (h_q, h_k, h_v, h_o):
            if t.device.type != "cpu" or not t.is_pinned():
                raise ValueError("host_step takes pinned host tensors")
        dev = self.q.device
        stream = torch.cuda.Stream(dev)
        side = torch.cuda.Stream(dev)
        k_new = torch.empty(self.B, self.Hkv, 1, self.D, dtype=self.k.dtype, device=dev)
        v_new = torch.empty_like(k_new)
        lens = [self.N] * self.B if self.lens_host is None else self.lens_host
        pos = torch.tensor([n - 1 for n in lens], dtype=torch.int32, device=dev)  # -1 (empty): nothing written
        plan = self._plan(stream, side, new_rows=(k_new, v_new, pos))

        def body():
            self.q.copy_(h_q, non_blocking=True)
            k_new.copy_(h_k, non_blocking=True)
            v_new.copy_(h_v, non_blocking=True)
            self._run(plan, stream, side)
            h_o.copy_(self.o, non_blocking=True)

        stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(stream):
            body()                                   # marshals the calls for these streams (not captured)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            body()
        return graph, stream


class PrefillLayer:
    """One attention layer's RTPurbo prefill: T query tokens per sequence (the
    last T of its N-token context), causal.

        a1  rtp_index_project   keys and queries of the retrieval heads -> 16-dim
        a3  rtp_topp_select     per-token top-p over the causal prefix (tensor-core score tiles)
        a4  rtp_sparse_attn_prefill   attention over each token's selected keys
        a5  rtp_window_attn     sliding-window attention of the local heads
    """

    def __init__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: torch.Tensor,
                 R: int, W: int, p: float, lens: Optional[torch.Tensor] = None,
                 out_dtype: torch.dtype = torch.float32, scale: Optional[float] = None,
                 with_mask: bool = False):
        B, Hq, T, D = q.shape
        _, Hkv, N, _ = k.shape
        self.B, self.Hq, self.Hkv, self.N, self.T, self.D = B, Hq, Hkv, N, T, D
        self.G = Hq // Hkv
        self.R, self.W, self.p = R, W, float(p)
        self.scale = (D ** -0.5) if scale is None else scale
        dev = q.device
        G = self.G
        self.q, self.k, self.v, self.P, self.lens = q, k, v, P, lens
        self.q_ret, self.q_loc = q[:, : R * G], q[:, R * G:]
        self.k_ret, self.v_ret = k[:, :R], v[:, :R]
        self.k_loc, self.v_loc = k[:, R:], v[:, R:]
        self.o = torch.zeros(B, Hq, T, D, dtype=out_dtype, device=dev)
        self.o_ret, self.o_loc = self.o[:, : R * G], self.o[:, R * G:]
        self.k_idx = torch.zeros(B, R, N, 16, dtype=torch.bfloat16, device=dev)
        self.q_idx = torch.zeros(B, R * G, T, 16, dtype=torch.bfloat16, device=dev)
        self.sel = rtp.Selection.empty(B * R * G * T, N, dev, with_mask=with_mask)
        self.ws_loc = (rtp.workspace(rtp.window_attn_workspace_size(B, Hq - R * G, T, Hkv - R, N, W), dev)
                       if Hkv > R else None)
        self._host_streams = None  # host_step: its two streams, made on first use

    def step(self, stream=None, side_stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        main = torch.cuda.current_stream() if stream is None else stream
        local = self.Hkv > self.R
        if side_stream is not None and local:
            side_stream.wait_stream(main)
            with torch.cuda.stream(side_stream):
                rtp.window_attn(self.q_loc, self.k_loc, self.v_loc, self.lens, self.W, self.scale, self.o_loc,
                                self.ws_loc, side_stream)
            local = False
        if self.R:
            rtp.index_project(self.k_ret, self.P, self.k_idx, stream)
            rtp.index_project(self.q_ret, self.P, self.q_idx, stream)
            rtp.topp_select(self.q_idx, self.k_idx, self.lens, self.p, self.sel, None, stream)
            rtp.sparse_attn_prefill(self.q_ret, self.k_ret, self.v_ret, self.q_idx, self.k_idx, self.lens,
                                    self.sel, self.scale, self.o_ret, None, stream)
        if local:
            rtp.window_attn(self.q_loc, self.k_loc, self.v_loc, self.lens, self.W, self.scale, self.o_loc,
                            self.ws_loc, stream)
        if side_stream is not None and self.Hkv > self.R:
            main.wait_stream(side_stream)
        return self.o

    def host_step(self, h_q: torch.Tensor, h_k: torch.Tensor, h_v: torch.Tensor, h_o: torch.Tensor) -> torch.Tensor:
        """One prefill end to end from host memory: h_q [B, Hq, T, D], h_k, h_v
        [B, Hkv, N, D] (pinned, the layer's dtypes) in, the output to h_o [B, Hq,
        T, D] (pinned), then wait for it.  The copies are pipelined with the
        work: the retrieval heads' inputs cross first and their chain (projection,
        selection, sparse attention, output copy) starts at once on one stream,
        while the local heads' inputs, their window attention and their output
        copy run on a second stream beside the selection."""
        for t in (h_q, h_k, h_v, h_o):
            if t.device.type != "cpu" or not t.is_pinned():
                raise ValueError("host_step takes pinned host tensors")
        for h, d in ((h_q, self.q), (h_k, self.k), (h_v, self.v), (h_o, self.o)):
            if h.shape != d.shape or h.dtype != d.dtype or not h.is_contiguous():
                raise ValueError("host buffers must be contiguous and match the layer's tensors")
        dev = self.q.device
        if self._host_streams is None:
            self._host_streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        main, side = self._host_streams
        main.wait_stream(torch.cuda.current_stream(dev))
        R, RG, H = self.R, self.R * self.G, self.Hkv
        with torch.cuda.stream(main):
            for b in range(self.B):  # per sequence: contiguous slices on both sides
                if R:
                    self.q[b, :RG].copy_(h_q[b, :RG], non_blocking=True)
                    self.k[b, :R].copy_(h_k[b, :R], non_blocking=True)
                    self.v[b, :R].copy_(h_v[b, :R], non_blocking=True)
        if H > R:
            side.wait_stream(main)  # the retrieval inputs cross first
            with torch.cuda.stream(side):
                for b in range(self.B):
                    self.q[b, RG:].copy_(h_q[b, RG:], non_blocking=True)
                    self.k[b, R:].copy_(h_k[b, R:], non_blocking=True)
                    self.v[b, R:].copy_(h_v[b, R:], non_blocking=True)
                rtp.window_attn(self.q_loc, self.k_loc, self.v_loc, self.lens, self.W, self.scale, self.o_loc,
                                self.ws_loc, side)
                for b in range(self.B):
                    h_o[b, RG:].copy_(self.o[b, RG:], non_blocking=True)
        if R:
            with torch.cuda.stream(main):
                rtp.index_project(self.k_ret, self.P, self.k_idx, main)
                rtp.index_project(self.q_ret, self.P, self.q_idx, main)
                rtp.topp_select(self.q_idx, self.k_idx, self.lens, self.p, self.sel, None, main)
                rtp.sparse_attn_prefill(self.q_ret, self.k_ret, self.v_ret, self.q_idx, self.k_idx, self.lens,
                                        self.sel, self.scale, self.o_ret, None, main)
                for b in range(self.B):
                    h_o[b, :RG].copy_(self.o[b, :RG], non_blocking=True)
        if H > R:
            main.wait_stream(side)
        main.synchronize()
        return h_o


class CachedDecodeLayer:
    """Decode over caches the layer keeps itself: every step appends the new
    token's keys and values, then attends with it.

        rtp_kv_append       new K/V -> retrieval heads' full caches and projected
                            keys, local heads' W-row rings (one launch)
        a1  rtp_index_project   queries of the retrieval heads -> q_idx
        a3  rtp_topp_select     top-p over the retrieval heads' caches
        a4  rtp_sparse_attn_decode   attention over the selected keys
        a5  rtp_window_attn     the local heads over their rings

    Retrieval heads (the first R KV heads) keep the full cache, local heads only
    the last W tokens ("RTPurbo: Turning Dense LLMs into Sparse Attention Models
    ...", "Three Key Insights" 1), so a local head's cache is W rows whatever the
    context length.  Sequence lengths live on the device (two buffers used in
    turn: one is an append's ``pos``, the other its ``lens_out``); the host never
    reads them.  Inputs of a step go into ``q`` [B, Hq, 1, D], ``k_new`` and
    ``v_new`` [B, Hkv, 1, D] (in place, or through the arguments of ``step``).
    """

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, R: int, W: int, p: float, P: torch.Tensor,
                 dtype: torch.dtype = torch.bfloat16, out_dtype: torch.dtype = torch.float32,
                 scale: Optional[float] = None, device=None, D: int = 128):
        dev = P.device if device is None else torch.device(device)
        if Hq % Hkv or not 0 <= R <= Hkv or W < 1:
            raise ValueError("need Hkv | Hq, 0 <= R <= Hkv and W >= 1")
        self.B, self.Hq, self.Hkv, self.N, self.D = B, Hq, Hkv, N, D
        self.G = G = Hq // Hkv
        self.R, self.W, self.p = R, W, float(p)
        self.scale = (D ** -0.5) if scale is None else scale
        self.P = P
        L = Hkv - R
        self.k_cache = torch.zeros(B, R, N, D, dtype=dtype, device=dev)
        self.v_cache = torch.zeros(B, R, N, D, dtype=dtype, device=dev)
        self.k_idx = torch.zeros(B, R, N, 16, dtype=dtype, device=dev)
        self.k_ring = torch.zeros(B, L, W, D, dtype=dtype, device=dev)
        self.v_ring = torch.zeros(B, L, W, D, dtype=dtype, device=dev)
        self._lens = [torch.zeros(B, dtype=torch.int32, device=dev) for _ in range(2)]
        self.ring_lens = torch.zeros(B, dtype=torch.int32, device=dev)
        self._cur = 0
        self.q = torch.zeros(B, Hq, 1, D, dtype=dtype, device=dev)
        self.k_new = torch.zeros(B, Hkv, 1, D, dtype=dtype, device=dev)
        self.v_new = torch.zeros(B, Hkv, 1, D, dtype=dtype, device=dev)
        self.q_idx = torch.zeros(B, R * G, 1, 16, dtype=dtype, device=dev)
        self.o = torch.zeros(B, Hq, 1, D, dtype=out_dtype, device=dev)
        self.sel = rtp.Selection.empty(B * R * G, N, dev)
        self.ws_sel = rtp.workspace(rtp.topp_select_workspace_size(B, R * G, 1, R, N), dev)
        self.ws_ret = rtp.workspace(rtp.sparse_attn_decode_workspace_size(B, R * G, R, N), dev) if R else None
        self.ws_loc = (rtp.workspace(rtp.window_attn_workspace_size(B, Hq - R * G, 1, L, W, W), dev)
                       if L else None)
        self._plans = {}

    @property
    def lens(self) -> torch.Tensor:
        """Device lengths of the sequences (tokens appended so far, capped at N)."""
        return self._lens[self._cur]

    def cache_bytes(self) -> int:
        """Device bytes of the K/V caches, rings and projected keys."""
        return sum(t.numel() * t.element_size() for t in (self.k_cache, self.v_cache, self.k_idx,
                                                         self.k_ring, self.v_ring))

    def set_lengths(self, lens: torch.Tensor) -> None:
        """Declare how many tokens each sequence holds (for caches filled by the caller)."""
        self._lens[self._cur].copy_(lens.to(torch.int32))
        self.ring_lens.copy_(torch.clamp(lens.to(torch.int32), 0, self.W))

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        """Append T tokens [B, Hkv, T, D] to every sequence (a chunk of prefill);
        tokens beyond the cache's N rows are dropped."""
        R, L = self.R, self.Hkv - self.R
        cur = self._cur
        rtp.kv_append(k_new, v_new, self._lens[cur], R, self.P if R else None,
                      self.k_cache if R else None, self.v_cache if R else None, self.k_idx if R else None,
                      self.k_ring if L else None, self.v_ring if L else None, self._lens[1 - cur],
                      self.ring_lens if L else None, stream)
        self._cur = 1 - cur

    def _plan(self, cur: int, main: torch.cuda.Stream, side: Optional[torch.cuda.Stream]):
        R, G, L = self.R, self.G, self.Hkv - self.R
        pos, lens = self._lens[cur], self._lens[1 - cur]
        pre, win, chain = [], [], []
        pre.append(rtp.bind_kv_append(self.k_new, self.v_new, pos, R, self.P if R else None,
                                      self.k_cache if R else None, self.v_cache if R else None,
                                      self.k_idx if R else None, self.k_ring if L else None,
                                      self.v_ring if L else None, lens, self.ring_lens if L else None, main))
        if R:
            pre.append(rtp.bind_index_project(self.q[:, : R * G], self.P, self.q_idx, main))
            chain.append(rtp.bind_topp_select(self.q_idx, self.k_idx, lens, self.p, self.sel, self.ws_sel, main))
            chain.append(rtp.bind_sparse_attn_decode(self.q[:, : R * G], self.k_cache, self.v_cache, lens, self.sel,
                                                     self.scale, self.o[:, : R * G], self.ws_ret, main))
        if L:
            win.append(rtp.bind_window_attn(self.q[:, R * G:], self.k_ring, self.v_ring, self.ring_lens, self.W,
                                            self.scale, self.o[:, R * G:], self.ws_loc,
                                            main if side is None else side))
        return pre, win, chain

    def step(self, q: Optional[torch.Tensor] = None, k_new: Optional[torch.Tensor] = None,
             v_new: Optional[torch.Tensor] = None, stream=None,
             side_stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Append the new token of every sequence and decode it; returns o [B, Hq, 1, D].
        With ``side_stream`` the local heads' window attention runs there."""
        for dst, src in ((self.q, q), (self.k_new, k_new), (self.v_new, v_new)):
            if src is not None:
                dst.copy_(src)
        main = torch.cuda.current_stream() if stream is None else stream
        key = (self._cur, main.cuda_stream, None if side_stream is None else side_stream.cuda_stream)
        plan = self._plans.get(key)
        if plan is None:
            plan = self._plans[key] = self._plan(self._cur, main, side_stream)
        pre, win, chain = plan
        for call in pre:
            call()
        if win and side_stream is not None:
            side_stream.wait_stream(main)
            for call in win:
                call()
            for call in chain:
                call()
            main.wait_stream(side_stream)
        else:
            for call in chain:
                call()
            for call in win:
                call()
        self._cur = 1 - self._cur
        return self.o

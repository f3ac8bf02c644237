"""GPU tests of the cache append (rtp_kv_append) and of decoding over the caches
it keeps (CachedDecodeLayer).

  * the append writes exactly the rows it should: retrieval heads' K/V at their
    positions, the projected keys bit-identical to rtp_index_project of the same
    rows, local heads' rings at position mod W (only the last W of a chunk),
    nothing for positions outside [0, N); the lengths it writes;
  * decoding over the caches, step after step, against the oracle on the full
    context (window attention over the ring == window attention over the full
    cache, since attention does not depend on the order of its keys);
  * the same decode over a resident full cache (DecodeLayer): identical bits for
    the retrieval heads, agreement to rounding for the local heads.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_dim_b200 import rtp
from long_context_sparse_dim_b200 import workloads as wl
from long_context_sparse_dim_b200.layer import CachedDecodeLayer, DecodeLayer

from gpu_check import compare_outputs, compare_selection, make_oracle, upload

pytestmark = pytest.mark.gpu


def _chunk(k_full, pos, T):
    """k_new [B, H, T, D]: row t of sequence b is token pos[b] + t of k_full
    (random filler where that position is outside the sequence)."""
    B, H, N, D = k_full.shape
    g = torch.Generator(device="cpu").manual_seed(7)
    out = torch.randn(B, H, T, D, generator=g).to(k_full.dtype).to(k_full.device)
    for b in range(B):
        lo, hi = max(pos[b], 0), min(pos[b] + T, N)
        if hi > lo:
            out[b, :, lo - pos[b]: hi - pos[b]] = k_full[b, :, lo:hi]
    return out


def _expected_ring(x_full, R, W, n):
    """The ring rows [H - R, W, D] the local heads of x_full [H, n', D] hold after
    in-order appends of tokens 0..n-1."""
    ring = torch.zeros(x_full.shape[0] - R, W, x_full.shape[2], dtype=x_full.dtype, device=x_full.device)
    for p in range(max(n - W, 0), n):
        ring[:, p % W] = x_full[R:, p]
    return ring


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_append_rows_projected_keys_rings_and_lengths(dtype):
    torch.manual_seed(0)
    B, H, R, N, W, D = 3, 5, 2, 700, 64, 128
    dev = "cuda"
    k_full = torch.randn(B, H, N + 40, D, device=dev).to(dtype)
    v_full = torch.randn(B, H, N + 40, D, device=dev).to(dtype)
    P = torch.randn(R, 16, D, device=dev) / 8
    k_cache = torch.zeros(B, R, N, D, dtype=dtype, device=dev)
    v_cache = torch.zeros_like(k_cache)
    k_idx = torch.zeros(B, R, N, 16, dtype=dtype, device=dev)
    k_ring = torch.zeros(B, H - R, W, D, dtype=dtype, device=dev)
    v_ring = torch.zeros_like(k_ring)
    lens = [torch.zeros(B, dtype=torch.int32, device=dev) for _ in range(2)]
    ring_lens = torch.full((B,), -7, dtype=torch.int32, device=dev)
    # a left-padded first chunk (sequence 1 starts 37 rows in, sequence 2 with
    # only 20 tokens), a second chunk, single tokens, then a chunk past the end
    lens[0].copy_(torch.tensor([0, -37, -280], dtype=torch.int32))
    cur = 0
    host = [0, -37, -280]
    for T in (300, 129, 1, 1, 1, 300):
        kn, vn = _chunk(k_full, host, T), _chunk(v_full, host, T)
        rtp.kv_append(kn, vn, lens[cur], R, P, k_cache, v_cache, k_idx, k_ring, v_ring, lens[1 - cur], ring_lens)
        host = [min(h + T, N) for h in host]
        torch.cuda.synchronize()
        assert lens[1 - cur].cpu().tolist() == host
        assert ring_lens.cpu().tolist() == [max(min(h, W), 0) for h in host]
        cur = 1 - cur
    assert host == [N, 695, 452]
    ends = [732, 695, 452]   # one past each sequence's last token (the first is cut at N)
    ref_idx = torch.zeros_like(k_idx)
    rtp.index_project(k_full[:, :R, :N].contiguous(), P, ref_idx)
    torch.cuda.synchronize()
    for b in range(B):
        n = min(ends[b], N)
        assert torch.equal(k_cache[b, :, :n], k_full[b, :R, :n])
        assert torch.equal(v_cache[b, :, :n], v_full[b, :R, :n])
        assert not k_cache[b, :, n:].any() and not k_idx[b, :, n:].any()
        assert torch.equal(k_idx[b, :, :n], ref_idx[b, :, :n])   # bit-identical to rtp_index_project
        assert torch.equal(k_ring[b], _expected_ring(k_full[b], R, W, ends[b]))
        assert torch.equal(v_ring[b], _expected_ring(v_full[b], R, W, ends[b]))


def test_append_ring_lengths_and_drop_past_the_end():
    dev = "cuda"
    B, H, R, N, W, D = 2, 2, 1, 50, 8, 128
    k_full = torch.randn(B, H, 60, D, device=dev).to(torch.bfloat16)
    P = torch.randn(R, 16, D, device=dev)
    kc = torch.zeros(B, R, N, D, dtype=torch.bfloat16, device=dev)
    vc, ki = torch.zeros_like(kc), torch.zeros(B, R, N, 16, dtype=torch.bfloat16, device=dev)
    kr = torch.zeros(B, H - R, W, D, dtype=torch.bfloat16, device=dev)
    vr = torch.zeros_like(kr)
    pos = torch.tensor([45, 3], dtype=torch.int32, device=dev)
    out = torch.empty(B, dtype=torch.int32, device=dev)
    rl = torch.empty(B, dtype=torch.int32, device=dev)
    rtp.kv_append(_chunk(k_full, [45, 3], 10), _chunk(k_full, [45, 3], 10), pos, R, P, kc, vc, ki, kr, vr, out, rl)
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [50, 13]                 # clamped to N
    assert rl.cpu().tolist() == [8, 8]
    assert torch.equal(kc[0, 0, 45:], k_full[0, 0, 45:50])
    assert torch.equal(kr[0], _expected_ring(k_full[0], R, W, 55))  # rings keep tokens past N
    # only local heads: no cache, no projection; lengths are not clamped
    out2 = torch.empty(B, dtype=torch.int32, device=dev)
    kr2 = torch.zeros(B, H, W, D, dtype=torch.bfloat16, device=dev)
    vr2 = torch.zeros_like(kr2)
    rtp.kv_append(_chunk(k_full, [45, 3], 10), _chunk(k_full, [45, 3], 10), pos, 0, None, None, None, None, kr2, vr2,
                  out2, None)
    torch.cuda.synchronize()
    assert out2.cpu().tolist() == [55, 13]
    assert torch.equal(kr2[0], _expected_ring(k_full[0], 0, W, 55))
    assert torch.equal(kr2[1], _expected_ring(k_full[1], 0, W, 13))
    # only retrieval heads
    rtp.kv_append(_chunk(k_full, [0, 0], 4), _chunk(k_full, [0, 0], 4), torch.zeros(B, dtype=torch.int32, device=dev),
                  H, torch.randn(H, 16, D, device=dev), torch.zeros(B, H, N, D, dtype=torch.bfloat16, device=dev),
                  torch.zeros(B, H, N, D, dtype=torch.bfloat16, device=dev),
                  torch.zeros(B, H, N, 16, dtype=torch.bfloat16, device=dev), None, None, out2, None)
    torch.cuda.synchronize()
    assert out2.cpu().tolist() == [4, 4]


def _cached_layer_run(inst, n0, steps, side=False):
    """Fill a CachedDecodeLayer with one chunk (sequence b left-padded to hold n0[b]
    tokens), then decode `steps` tokens; yields (lens after the step, o, layer)."""
    w = inst.wl
    q, k, v, P, _ = upload(inst)
    layer = CachedDecodeLayer(w.B, w.Hq, w.Hkv, w.N, w.R, w.W, w.p, P, dtype=k.dtype)
    T0 = max(n0)
    pos = [n - T0 for n in n0]
    layer.set_lengths(torch.tensor(pos, dtype=torch.int32, device="cuda"))
    layer.append(_chunk(k, pos, T0), _chunk(v, pos, T0))
    side_stream = torch.cuda.Stream() if side else None
    for s in range(steps):
        idx = torch.tensor([n + s for n in n0], device="cuda")
        kn = k[torch.arange(w.B, device="cuda"), :, idx].unsqueeze(2)
        vn = v[torch.arange(w.B, device="cuda"), :, idx].unsqueeze(2)
        o = layer.step(q, kn, vn, side_stream=side_stream)
        torch.cuda.synchronize()
        yield np.array([n + s + 1 for n in n0], np.int32), o.float().cpu().numpy(), layer


SMALL = wl.DECODE_B8_N32K.replace(name="cached_small", B=2, N=1000, W=100, needles=0)


@pytest.mark.parametrize("side", [False, True])
def test_cached_decode_steps_match_oracle(side):
    inst = wl.generate(SMALL)
    w = inst.wl
    for lens, o, layer in _cached_layer_run(inst, [900, 851], 4, side):
        assert layer.lens.cpu().numpy().tolist() == lens.tolist()
        inst_s = wl.Instance(wl=w, q=inst.q, k=inst.k, v=inst.v, P=inst.P, lens=lens, needles=[])
        L = make_oracle(inst_s)
        res = L.run()
        compare_outputs(o, res, f"cached decode lens={lens.tolist()}")
        mask = layer.sel.mask.cpu().numpy().view(np.uint32)
        count = layer.sel.count.cpu().numpy()
        Hr = w.R * w.G
        for b in range(w.B):
            for h in range(Hr):
                compare_selection(res[(b, h, 0)], mask[b * Hr + h], int(lens[b]), int(count[b * Hr + h]),
                                  f"cached decode b{b} h{h}")


def test_cached_decode_matches_resident_cache_layer():
    w = wl.DECODE_B8_N32K.replace(name="cached_vs_resident", B=2, N=9000, W=512, needles=0)
    inst = wl.generate(w)
    n0 = [8000, 7333]
    *_, (lens, o, layer) = _cached_layer_run(inst, n0, 2)
    q, k, v, P, _ = upload(inst)
    ref = DecodeLayer(q, k, v, P, R=w.R, W=w.W, p=w.p, lens=torch.from_numpy(lens).cuda())
    ref.build_index()
    o_ref = ref.step().float().cpu().numpy()
    torch.cuda.synchronize()
    Hr = w.R * w.G
    assert np.array_equal(o[:, :Hr], o_ref[:, :Hr])                 # same caches, same kernels
    assert np.abs(o[:, Hr:] - o_ref[:, Hr:]).max() <= 1e-5 * np.abs(o_ref[:, Hr:]).max()
    # memory: the local heads hold W rows instead of N
    ring = 2 * w.B * (w.Hkv - w.R) * w.W * 128 * 2
    full_ret = 2 * w.B * w.R * w.N * 128 * 2 + w.B * w.R * w.N * 16 * 2
    assert layer.cache_bytes() == full_ret + ring


def test_empty_append_and_one_row_ring():
    # T = 0 writes only the lengths; W = 1 keeps the newest token's row
    dev = "cuda"
    B, H, R, N, D = 2, 3, 1, 16, 128
    k_full = torch.randn(B, H, 20, D, device=dev).to(torch.bfloat16)
    P = torch.randn(R, 16, D, device=dev)
    kc = torch.zeros(B, R, N, D, dtype=torch.bfloat16, device=dev)
    vc, ki = torch.zeros_like(kc), torch.zeros(B, R, N, 16, dtype=torch.bfloat16, device=dev)
    kr = torch.zeros(B, H - R, 1, D, dtype=torch.bfloat16, device=dev)
    vr = torch.zeros_like(kr)
    pos = torch.tensor([5, 0], dtype=torch.int32, device=dev)
    out = torch.full((B,), -1, dtype=torch.int32, device=dev)
    rl = torch.full((B,), -1, dtype=torch.int32, device=dev)
    empty = k_full[:, :, :0]  # a zero-length view (its data pointer is valid)
    rtp.kv_append(empty, empty, pos, R, P, kc, vc, ki, kr, vr, out, rl)
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [5, 0] and rl.cpu().tolist() == [1, 0]
    assert not kc.any() and not kr.any()
    rtp.kv_append(_chunk(k_full, [5, 0], 3), _chunk(k_full, [5, 0], 3), pos, R, P, kc, vc, ki, kr, vr, out, rl)
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [8, 3] and rl.cpu().tolist() == [1, 1]
    assert torch.equal(kr[0, :, 0], k_full[0, R:, 7]) and torch.equal(kr[1, :, 0], k_full[1, R:, 2])

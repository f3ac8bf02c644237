"""GPU parity of the decode path (C ABI) against the CPU oracle.

Sizes range from a handful of keys (edge cases, ragged tails) to the full
decode workloads: one fp32 sequence of 4096 keys with one retrieval and one
local head, and a batch of 8 Llama-3-8B-shaped layers at 32768 keys.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_dim_b200 import workloads as wl

from gpu_check import (compare_outputs, compare_selection, device_dtype, make_oracle, upload)

pytestmark = pytest.mark.gpu


def _run(inst, p=None, W=None, out_dtype=torch.float32, ragged=False):
    from long_context_sparse_dim_b200.layer import DecodeLayer
    w = inst.wl
    q, k, v, P, lens = upload(inst)
    layer = DecodeLayer(q, k, v, P, R=w.R, W=w.W if W is None else W, p=w.p if p is None else p,
                        lens=lens if ragged else None, out_dtype=out_dtype)
    layer.build_index()
    o = layer.step()
    torch.cuda.synchronize()
    return layer, o


def _check(inst, layer, o, p=None, W=None, tol=2e-3):
    w = inst.wl
    L = make_oracle(inst, p=p, W=W)
    res = L.run()
    o_np = o.float().cpu().numpy()
    worst = compare_outputs(o_np, res, w.name, tol)
    if w.R:
        mask = layer.sel.mask.cpu().numpy().view(np.uint32)
        count = layer.sel.count.cpu().numpy()
        Hr = w.R * w.G
        for b in range(w.B):
            for h in range(Hr):
                r = b * Hr + h
                compare_selection(res[(b, h, 0)], mask[r], int(inst.lens[b]), int(count[r]), f"{w.name} b{b} h{h}")
    return worst, res


SMALL = wl.DECODE_B8_N32K.replace(name="small_gqa", B=2, N=1000, W=100, needles=8)


@pytest.mark.parametrize("N", [1, 2, 15, 16, 17, 127, 128, 129, 4097])
def test_decode_edge_lengths(N):
    w = SMALL.replace(name=f"edge_n{N}", N=N, W=min(64, N + 5), needles=0 if N < 40 else 4)
    inst = wl.generate(w)
    layer, o = _run(inst)
    _check(inst, layer, o)


@pytest.mark.parametrize("W", [1, 999, 1000, 1005])
def test_decode_window_edges(W):
    inst = wl.generate(SMALL.replace(name=f"win{W}", W=W))
    layer, o = _run(inst, W=W)
    _check(inst, layer, o, W=W)


@pytest.mark.parametrize("p", [1e-6, 0.3, 0.9, 0.999, 1.0])
def test_decode_p_sweep(p):
    inst = wl.generate(SMALL.replace(name=f"p{p}", p=p))
    layer, o = _run(inst, p=p)
    _check(inst, layer, o, p=p)


def test_decode_ragged_batch():
    w = SMALL.replace(name="ragged", B=5, N=3000, ragged=True)
    inst = wl.generate(w)
    assert len(set(inst.lens.tolist())) > 1
    layer, o = _run(inst, ragged=True)
    _check(inst, layer, o)


def test_decode_all_equal_scores_tie_break():
    # zero projected queries -> every indexer score is 0: the lowest positions win
    inst = wl.generate(SMALL.replace(name="ties", N=777))
    P0 = np.zeros_like(inst.P)
    inst.P = P0
    layer, o = _run(inst)
    worst, res = _check(inst, layer, o)
    cnt = layer.sel.count.cpu().numpy()
    want = int(np.ceil(np.float64(np.float32(SMALL.p)) * 777 - 1e-9))
    assert (cnt == want).all()


def test_decode_negative_and_signed_zero_scores():
    # P with a negated coordinate gives negative scores for half the keys, and
    # integer-valued inputs give exact zeros of both signs
    inst = wl.generate(SMALL.replace(name="signs", N=513, dtype="f32"))
    rng = np.random.default_rng(0)
    inst.k = np.round(inst.k * 0.5).astype(np.float32)
    inst.q = np.round(inst.q * 0.5).astype(np.float32)
    inst.P = inst.P.copy()
    inst.P[:, 3] *= -1.0
    layer, o = _run(inst)
    _check(inst, layer, o)


def test_decode_bf16_output():
    inst = wl.generate(SMALL.replace(name="bf16out"))
    layer, o = _run(inst, out_dtype=torch.bfloat16)
    _check(inst, layer, o, tol=6e-3)  # bf16 output rounding adds 2^-9 relative


def test_decode_f32_small_group():
    inst = wl.generate(wl.DECODE_N4K_F32.replace(name="f32_gqa", Hq=8, Hkv=2, R=1, N=900, W=77))
    layer, o = _run(inst)
    _check(inst, layer, o)


def test_decode_deterministic():
    inst = wl.generate(SMALL.replace(name="det", N=5000))
    layer, o1 = _run(inst)
    m1 = layer.sel.mask.clone()
    o1 = o1.clone()
    layer.step()
    torch.cuda.synchronize()
    assert torch.equal(layer.sel.mask, m1)
    assert torch.equal(layer.o, o1)


def test_index_project_general_projection():
    from long_context_sparse_dim_b200 import rtp
    import oracle
    rng = np.random.default_rng(3)
    for dt in (torch.bfloat16, torch.float32):
        x = torch.from_numpy(rng.standard_normal((2, 3, 257, 128)).astype(np.float32)).to("cuda", dt)
        P = torch.from_numpy(rng.standard_normal((3, 16, 128)).astype(np.float32) * 0.1).cuda()
        out = torch.empty(2, 3, 257, 16, dtype=dt, device="cuda")
        rtp.index_project(x, P, out)
        torch.cuda.synchronize()
        xs = [[x[b, h].float().cpu().numpy() for h in range(3)] for b in range(2)]
        Ps = [P[h].cpu().numpy() for h in range(3)]
        ref = np.stack([np.stack([oracle.index_project(xs[b][h], Ps[h], "f64") for h in range(3)])
                        for b in range(2)])
        # forward error bound of an fp32 sum of n=128 products: gamma_n * sum |P_ij x_j|,
        # plus the final rounding to the output type
        absum = np.stack([np.stack([np.abs(xs[b][h]).astype(np.float64) @ np.abs(Ps[h]).T.astype(np.float64)
                                    for h in range(3)]) for b in range(2)])
        u = 2.0 ** -24
        gamma = 128 * u / (1 - 128 * u)
        out_u = 2.0 ** -8 if dt == torch.bfloat16 else 2.0 ** -24
        got = out.float().cpu().numpy()
        assert np.all(np.abs(got - ref) <= gamma * absum + out_u * np.abs(ref) + 1e-30)


def test_decode_n4096_f32_one_retrieval_one_local_head():
    inst = wl.generate(wl.DECODE_N4K_F32)
    layer, o = _run(inst)
    worst, res = _check(inst, layer, o)
    import oracle
    hit, tot = oracle.needle_recall(res, inst.needles)
    assert tot == 16 and hit == tot


def test_decode_b8_n32768_llama8b_layer():
    inst = wl.generate(wl.DECODE_B8_N32K)
    layer, o = _run(inst)
    worst, res = _check(inst, layer, o)
    assert worst <= 2e-3


def test_decode_side_stream_matches_single_stream():
    inst = wl.generate(SMALL.replace(name="side", N=3000))
    layer, o1 = _run(inst)
    o1 = o1.clone()
    side = torch.cuda.Stream()
    layer.o.zero_()
    layer.step(side_stream=side)
    torch.cuda.synchronize()
    assert torch.equal(layer.o, o1)


def test_host_step_matches_device_step():
    # the end-to-end form (pinned host buffers in and out, one captured graph per
    # buffer set) gives the device step's bits, on every replay
    from long_context_sparse_dim_b200.layer import DecodeLayer
    w = SMALL.replace(name="host_step", B=3, N=2000)
    inst = wl.generate(w)
    q, k, v, P, lens = upload(inst)
    layer = DecodeLayer(q, k, v, P, R=w.R, W=w.W, p=w.p)
    layer.build_index()
    o_dev = layer.step().clone()
    n = w.N
    h_q = q.cpu().pin_memory()
    h_k = k[:, :, n - 1: n].cpu().pin_memory()
    h_v = v[:, :, n - 1: n].cpu().pin_memory()
    h_o = torch.empty(o_dev.shape, dtype=o_dev.dtype).pin_memory()
    for _ in range(3):
        h_o.zero_()
        layer.host_step(h_q, h_k, h_v, h_o)
        assert torch.equal(h_o, o_dev.cpu())


def test_host_step_appends_the_new_rows_ragged():
    # host_step writes each sequence's new K/V row (and its projected key) at its last
    # position: over caches that lack those rows it gives the device step's bits over the
    # complete caches; an empty sequence receives nothing
    from long_context_sparse_dim_b200.layer import DecodeLayer
    w = SMALL.replace(name="host_step_ragged", B=3, N=2000)
    inst = wl.generate(w)
    q, k, v, P, _ = upload(inst)
    ln = [2000, 1500, 0]
    lens = torch.tensor(ln, dtype=torch.int32, device=q.device)
    full = DecodeLayer(q, k, v, P, R=w.R, W=w.W, p=w.p, lens=lens)
    full.build_index()
    o_dev = full.step().clone()
    k2, v2 = k.clone(), v.clone()
    for b, n in enumerate(ln):
        if n > 0:
            k2[b, :, n - 1] = 0
            v2[b, :, n - 1] = 0
    layer = DecodeLayer(q, k2, v2, P, R=w.R, W=w.W, p=w.p, lens=lens)
    layer.build_index()
    h_q = q.cpu().pin_memory()
    rows_k = torch.stack([k[b, :, max(n - 1, 0)] for b, n in enumerate(ln)]).unsqueeze(2)
    rows_v = torch.stack([v[b, :, max(n - 1, 0)] for b, n in enumerate(ln)]).unsqueeze(2)
    rows_k[2] = 7.0  # the empty sequence's row is never written
    rows_v[2] = -7.0
    h_k = rows_k.cpu().pin_memory()
    h_v = rows_v.cpu().pin_memory()
    h_o = torch.empty(o_dev.shape, dtype=o_dev.dtype).pin_memory()
    for _ in range(2):
        h_o.zero_()
        layer.host_step(h_q, h_k, h_v, h_o)
        assert torch.equal(h_o, o_dev.cpu())
    assert torch.equal(k2, k) and torch.equal(v2, v)
    assert torch.equal(layer.k_idx, full.k_idx)

"""GPU parity of the prefill path (C ABI) against the CPU oracle: tensor-core
indexer tiles, per-token top-p over the causal prefix, sparse attention over
the selected keys (retrieval heads) and banded attention (local heads)."""
import numpy as np
import pytest
import torch

from long_context_sparse_dim_b200 import rtp
from long_context_sparse_dim_b200 import workloads as wl

from gpu_check import compare_outputs, compare_selection, make_oracle, upload

pytestmark = pytest.mark.gpu

SMALL = wl.PREFILL_N32K.replace(name="prefill_small", N=384, T=384, W=100, needle_fraction=0.1)


def _run(inst, p=None, W=None, ragged=False, out_dtype=torch.float32):
    from long_context_sparse_dim_b200.layer import PrefillLayer
    w = inst.wl
    q, k, v, P, lens = upload(inst)
    layer = PrefillLayer(q, k, v, P, R=w.R, W=w.W if W is None else W, p=w.p if p is None else p,
                         lens=lens if ragged else None, out_dtype=out_dtype, with_mask=True)
    o = layer.step()
    torch.cuda.synchronize()
    assert rtp.poll_device_error() == 0
    return layer, o


def _check(inst, layer, o, p=None, W=None, tol=2e-3, heads=None):
    w = inst.wl
    L = make_oracle(inst, p=p, W=W)
    Hr = w.R * w.G
    qs = [(b, h, t) for b in range(w.B) for h in (range(w.Hq) if heads is None else heads) for t in range(w.T)]
    res = L.run(qs)
    compare_outputs(o.float().cpu().numpy(), res, w.name, tol)
    mask = layer.sel.mask.cpu().numpy().view(np.uint32)
    count = layer.sel.count.cpu().numpy()
    n_diff = 0
    for (b, h, t), r in res.items():
        if h >= Hr:
            continue
        row = (b * Hr + h) * w.T + t
        n = max(L.pos(b, t) + 1, 0)
        n_diff += compare_selection(r, mask[row], n, int(count[row]), f"{w.name} b{b} h{h} t{t}")
    return res, n_diff


def test_prefill_small_causal():
    inst = wl.generate(SMALL)
    layer, o = _run(inst)
    _check(inst, layer, o)


@pytest.mark.parametrize("N,T", [(129, 129), (200, 64), (700, 200), (1000, 3)])
def test_prefill_chunked_and_ragged_tiles(N, T):
    inst = wl.generate(SMALL.replace(name=f"pf_{N}_{T}", N=N, T=T, W=min(77, N)))
    layer, o = _run(inst, W=min(77, N))
    _check(inst, layer, o, W=min(77, N))


@pytest.mark.parametrize("p", [1e-6, 0.5, 0.999, 1.0])
def test_prefill_p_sweep(p):
    inst = wl.generate(SMALL.replace(name=f"pf_p{p}", N=256, T=256))
    layer, o = _run(inst, p=p)
    _check(inst, layer, o, p=p)


@pytest.mark.parametrize("W", [1, 255, 256, 300])
def test_prefill_window_edges(W):
    inst = wl.generate(SMALL.replace(name=f"pf_w{W}", N=256, T=256, R=0, W=W))
    layer, o = _run(inst, W=W)
    _check(inst, layer, o, W=W)


def test_prefill_ragged_batch():
    w = SMALL.replace(name="pf_ragged", B=3, N=500, T=150, ragged=True)
    inst = wl.generate(w)
    assert len(set(inst.lens.tolist())) > 1
    layer, o = _run(inst, ragged=True)
    _check(inst, layer, o)


def test_prefill_all_equal_scores():
    inst = wl.generate(SMALL.replace(name="pf_ties", N=200, T=200))
    inst.P = np.zeros_like(inst.P)
    layer, o = _run(inst)
    _check(inst, layer, o)
    cnt = layer.sel.count.cpu().numpy().reshape(-1, 200)
    pos = np.arange(200)
    want = np.ceil(np.float64(np.float32(SMALL.p)) * (pos + 1) - 1e-9).astype(int)
    assert (cnt == want[None, :]).all()


def test_prefill_bf16_output_and_determinism():
    inst = wl.generate(SMALL.replace(name="pf_det", N=300, T=300))
    layer, o1 = _run(inst, out_dtype=torch.bfloat16)
    o1 = o1.clone()
    m1 = layer.sel.mask.clone()
    layer.step()
    torch.cuda.synchronize()
    assert torch.equal(layer.o, o1) and torch.equal(layer.sel.mask, m1)
    _check(inst, layer, o1, tol=6e-3)


def test_prefill_host_step_matches_step():
    # the end-to-end form (pinned host buffers in and out, copies pipelined with the work on
    # two streams) gives the device step's bits, ragged batch included
    from long_context_sparse_dim_b200.layer import PrefillLayer
    inst = wl.generate(SMALL.replace(name="pf_host", B=2, N=400, T=300))
    w = inst.wl
    q, k, v, P, lens = upload(inst)
    layer = PrefillLayer(q, k, v, P, R=w.R, W=w.W, p=w.p, lens=lens)
    o_dev = layer.step().clone()
    torch.cuda.synchronize()
    h_q, h_k, h_v = (x.cpu().pin_memory() for x in (q, k, v))
    h_o = torch.empty(o_dev.shape, dtype=o_dev.dtype).pin_memory()
    layer.q.zero_()
    layer.k.zero_()
    layer.v.zero_()
    layer.o.zero_()
    for _ in range(2):
        h_o.zero_()
        layer.host_step(h_q, h_k, h_v, h_o)
        assert torch.equal(h_o, o_dev.cpu())
    assert rtp.poll_device_error() == 0

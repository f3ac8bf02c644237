"""rtp_sparse_attn_decode_noalloc against rtp_sparse_attn_decode (GPU, C ABI).

The no-allocation entry point exists for callers that cannot call cudaMalloc
(for instance a plugin inside a host framework that owns every device
allocation, or a runtime that forbids allocation after start-up) and so cannot
hand the library a workspace.  It must give the same results as the
workspace entry point.  Two calls in a row, on two different shapes, also
check that the scratch array left behind by one call does not disturb the
next.  This file runs last so that a failure here leaves every other test
already run; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_dim_b200 import rtp
from long_context_sparse_dim_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 2e-3  # the decode parity tolerance (max |diff| / max |ref| per row)


def _selected(inst):
    w = inst.wl
    dev = torch.device("cuda")
    q = torch.from_numpy(inst.q).to(dev, torch.bfloat16)
    k = torch.from_numpy(inst.k).to(dev, torch.bfloat16)
    v = torch.from_numpy(inst.v).to(dev, torch.bfloat16)
    P = torch.from_numpy(inst.P).to(dev, torch.float32)
    G, R = w.G, w.R
    q_ret, k_ret, v_ret = q[:, : R * G], k[:, :R], v[:, :R]
    k_idx = torch.zeros(w.B, R, w.N, 16, dtype=torch.bfloat16, device=dev)
    q_idx = torch.zeros(w.B, R * G, 1, 16, dtype=torch.bfloat16, device=dev)
    rtp.index_project(k_ret, P, k_idx)
    rtp.index_project(q_ret, P, q_idx)
    sel = rtp.Selection.empty(w.B * R * G, w.N, dev)
    ws = rtp.workspace(rtp.topp_select_workspace_size(w.B, R * G, 1, R, w.N), dev)
    rtp.topp_select(q_idx, k_idx, None, w.p, sel, ws)
    return q_ret, k_ret, v_ret, sel


def _rows_rel_err(a: torch.Tensor, b: torch.Tensor) -> float:
    a = a.double().flatten(0, 2)
    b = b.double().flatten(0, 2)
    den = b.abs().amax(dim=1).clamp_min(1e-30)
    return float(((a - b).abs().amax(dim=1) / den).max())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    shapes = [wl.DECODE_B8_N32K.replace(name="noalloc_a", B=4, N=9000, needles=8),
              wl.DECODE_B8_N32K.replace(name="noalloc_b", B=2, N=20000, needles=8, seed=11)]
    for w in shapes:
        inst = wl.generate(w)
        q, k, v, sel = _selected(inst)
        scale = 128 ** -0.5
        ref = torch.zeros(w.B, w.R * w.G, 1, 128, dtype=torch.float32, device="cuda")
        ws = rtp.workspace(rtp.sparse_attn_decode_workspace_size(w.B, w.R * w.G, w.R, w.N), "cuda")
        rtp.sparse_attn_decode(q, k, v, None, sel, scale, ref, ws)
        out = torch.full_like(ref, float("nan"))
        rtp.sparse_attn_decode_noalloc(q, k, v, None, sel, scale, out)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert _rows_rel_err(out, ref) <= TOL


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # a shape whose split-K scratch exceeds the fixed array is refused before any launch
    B, Hq, Hk, N = 4096, 32, 8, 4096
    assert rtp.sparse_attn_decode_workspace_size(B, Hq, Hk, N) > rtp.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, Hq, 1, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16, device="cuda").expand(B, Hk, N, 128)
    sel = rtp.Selection.empty(B * Hq, N, "cuda")
    o = torch.zeros(B, Hq, 1, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(rtp.RtpError) as e:
        rtp.sparse_attn_decode_noalloc(q, kv, kv, None, sel, 0.088, o)
    assert e.value.status == 7  # RTP_ERR_UNSUPPORTED

"""The give-up path of the prefill kernels' bounded device waits (GPU).

A wait budget of a few clock cycles makes the prefill selection's first
waits on TMA copies and tensor-core commits give up: the kernel records
RTP_DEVICE_ERR_TIMEOUT in the device error word, still waits (with the
default budget) for every copy it issued, frees its tensor memory and exits.
No GPU fault or hang is involved: the copies complete on their own.  The
next launch with the default budget must be correct.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_dim_b200 import rtp
from long_context_sparse_dim_b200 import workloads as wl

from gpu_check import compare_selection, make_oracle, upload

pytestmark = pytest.mark.gpu

RTP_DEVICE_ERR_TIMEOUT = 1


def _select(inst, sel):
    w = inst.wl
    q, k, v, P, lens = upload(inst)
    G, R = w.G, w.R
    k_idx = torch.zeros(w.B, R, w.N, 16, dtype=torch.bfloat16, device="cuda")
    q_idx = torch.zeros(w.B, R * G, w.T, 16, dtype=torch.bfloat16, device="cuda")
    rtp.index_project(k[:, :R], P, k_idx)
    rtp.index_project(q[:, : R * G], P, q_idx)
    rtp.topp_select(q_idx, k_idx, None, w.p, sel)


def test_wait_budget_runs_out_then_next_launch_is_correct():
    w = wl.PREFILL_N32K.replace(name="budget", N=512, T=256, W=64, needle_fraction=0.1)
    inst = wl.generate(w)
    rows = w.B * w.R * w.G * w.T
    assert rtp.poll_device_error() == 0
    sel = rtp.Selection.empty(rows, w.N, "cuda")
    try:
        rtp.set_wait_budget_cycles(4)
        _select(inst, sel)
        torch.cuda.synchronize()
    finally:
        rtp.set_wait_budget_cycles(0)
    assert rtp.poll_device_error() == RTP_DEVICE_ERR_TIMEOUT
    assert rtp.poll_device_error() == 0  # polling cleared it

    sel = rtp.Selection.empty(rows, w.N, "cuda")
    _select(inst, sel)
    torch.cuda.synchronize()
    assert rtp.poll_device_error() == 0
    L = make_oracle(inst)
    mask = sel.mask.cpu().numpy().view(np.uint32)
    count = sel.count.cpu().numpy()
    Hr = w.R * w.G
    for h in range(Hr):
        for t in range(0, w.T, 7):
            r = L.query(0, h, t)
            row = h * w.T + t
            compare_selection(r, mask[row], L.pos(0, t) + 1, int(count[row]), f"after timeout h{h} t{t}")

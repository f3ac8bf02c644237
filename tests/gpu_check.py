"""Helpers shared by the GPU parity tests: upload a drawn workload, run the
decode path through the C ABI, and compare with the CPU oracle.

Comparison rules
  * selected sets: identical, except keys whose oracle indexer score lies
    within the tie band |s - tau| <= 1e-4 * max(|tau|, 1) of the oracle's cut
    score tau (fp32 scores on the GPU vs fp64 in the oracle);
  * counts: the GPU count equals the size of the GPU mask;
  * attention outputs: max |o - o_ref| / max |o_ref| <= 2e-3 per (sequence,
    head) row, o_ref the oracle's output on its own selected set.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TIE_BAND_REL = 1e-4
OUT_TOL = 2e-3


def device_dtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def upload(inst, device="cuda"):
    dt = device_dtype(inst.wl)
    q = torch.from_numpy(inst.q).to(device=device, dtype=dt)
    k = torch.from_numpy(inst.k).to(device=device, dtype=dt)
    v = torch.from_numpy(inst.v).to(device=device, dtype=dt)
    P = torch.from_numpy(np.ascontiguousarray(inst.P)).to(device=device, dtype=torch.float32)
    lens = torch.from_numpy(inst.lens).to(device=device, dtype=torch.int32)
    return q, k, v, P, lens


def make_oracle(inst, p=None, W=None):
    wl = inst.wl
    return oracle.LayerOracle(inst.q, inst.k, inst.v, inst.P, inst.lens, R=wl.R,
                              W=wl.W if W is None else W,
                              p=float(np.float32(wl.p if p is None else p)),
                              storage=wl.dtype)


def mask_to_sets(mask_np: np.ndarray, n: int):
    bits = np.unpackbits(mask_np.view(np.uint8), bitorder="little")
    return np.flatnonzero(bits[:n])


def compare_selection(res, mask_row: np.ndarray, n: int, count_gpu: int, where: str):
    """GPU set (from its mask) against the oracle's selection of one query."""
    got = mask_to_sets(mask_row, mask_row.size * 32)
    assert got.size == 0 or got.max() < n, f"{where}: bits set beyond the sequence"
    assert count_gpu == got.size, f"{where}: count {count_gpu} != mask popcount {got.size}"
    want = res.sel.idx
    diff = np.setxor1d(got, want)
    if diff.size:
        tau = res.sel.tau
        band = TIE_BAND_REL * max(abs(tau), 1.0)
        off = np.abs(res.scores[diff] - tau)
        assert np.all(off <= band), (
            f"{where}: {diff.size} keys differ outside the tie band; worst |s-tau|={off.max():.3g} "
            f"band={band:.3g} count gpu {got.size} oracle {want.size}")
    return diff.size


def rel_err(o, ref):
    den = np.max(np.abs(ref))
    num = np.max(np.abs(o - ref))
    if den == 0.0:
        return float(num)
    return float(num / den)


def compare_outputs(o_gpu: np.ndarray, results, where: str, tol=OUT_TOL):
    worst = 0.0
    for (b, h, t), r in results.items():
        e = rel_err(o_gpu[b, h, t].astype(np.float64), r.o)
        assert e <= tol, f"{where}: (b={b}, h={h}, t={t}) rel err {e:.3g} > {tol}"
        worst = max(worst, e)
    return worst

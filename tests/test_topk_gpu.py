"""GPU parity of rtp_topk_select (decode form): the fixed top-k cut through the
top-p selection's passes, every key weighing 1.

Crafted score sets reach each way the kernel finds the cut (candidates of the
fine cut bin, exact ties at the cut, the tail bin, a fine bin with more
candidates than rank 0 takes); the projected query is (4, 0, ..., 0) in fp32,
so every indexer score is the first coordinate of its projected key exactly.
A bf16 decode workload checks the usual path against the oracle's scores.
"""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_dim_b200 import rtp
from long_context_sparse_dim_b200 import workloads as wl

from gpu_check import compare_selection, make_oracle, upload

pytestmark = pytest.mark.gpu


def _select_k(scores_rows, k, lens=None):
    s = np.asarray(scores_rows, dtype=np.float32)
    B, N = s.shape
    k_idx = np.zeros((B, 1, N, 16), np.float32)
    k_idx[:, 0, :, 0] = s
    q_idx = np.zeros((B, 1, 1, 16), np.float32)
    q_idx[..., 0] = 4.0
    dev = torch.device("cuda")
    sel = rtp.Selection.empty(B, N, dev)
    ld = None if lens is None else torch.tensor(lens, dtype=torch.int32, device=dev)
    rtp.topk_select(torch.from_numpy(q_idx).to(dev), torch.from_numpy(k_idx).to(dev), ld, k, sel)
    torch.cuda.synchronize()
    return (sel.mask.cpu().numpy().view(np.uint32), sel.count.cpu().numpy(),
            sel.tau_bits.cpu().numpy().view(np.uint32), sel.tiepos.cpu().numpy())


def _check(scores_rows, k, where, lens=None):
    s32 = np.asarray(scores_rows, dtype=np.float32)
    mask, count, tau_bits, tiepos = _select_k(s32, k, lens)
    out = []
    for b in range(s32.shape[0]):
        n = s32.shape[1] if lens is None else int(lens[b])
        s = s32[b, :n].astype(np.float64)
        ref = oracle.topk_select(s, k)
        compare_selection(SimpleNamespace(sel=ref, scores=s), mask[b], n, int(count[b]), f"{where} row {b}")
        assert int(count[b]) == ref.count, f"{where} row {b}: count {count[b]} != {ref.count}"
        if ref.count < n:  # the threshold form describes the mask exactly
            tau = np.uint32(tau_bits[b]).view(np.float32)
            bits = np.unpackbits(mask[b].view(np.uint8), bitorder="little")[:n].astype(bool)
            implied = (s32[b, :n] > tau) | ((s32[b, :n] == tau) & (np.arange(n) <= tiepos[b]))
            assert np.array_equal(bits, implied), f"{where} row {b}: mask differs from (tau, tiepos)"
        out.append((ref, mask[b], int(count[b]), int(tiepos[b])))
    return out


@pytest.mark.parametrize("k", [1, 100, 3000, 49999, 50000, 60000])
def test_topk_random_scores(k):
    rng = np.random.default_rng(31)
    _check(rng.standard_normal((3, 50000)).astype(np.float32), k, f"normal k={k}")


def test_topk_exact_ties_at_the_cut():
    # 40 keys share a value no other key has; k cuts through the tie group, whose
    # lowest positions must be the ones taken
    rng = np.random.default_rng(32)
    N = 20000
    s = rng.standard_normal(N).astype(np.float32)
    v = np.float32(0.5)
    s[s == v] = np.float32(0.51)
    tie_pos = np.sort(rng.choice(N, size=40, replace=False))
    s[tie_pos] = v
    n_above = int((s > v).sum())
    (ref, mask, count, tp), = _check(s[None], n_above + 20, "ties")
    assert tp == tie_pos[19] and count == n_above + 20
    bits = np.unpackbits(mask.view(np.uint8), bitorder="little")[:N].astype(bool)
    assert bits[tie_pos[:20]].all() and not bits[tie_pos[20:]].any()


def test_topk_all_equal_and_ragged():
    N = 5000
    lens = [5000, 3333, 17]
    res = _check(np.zeros((3, N), np.float32), 100, "equal", lens=lens)
    for (ref, mask, count, tp), n in zip(res, lens):
        assert count == min(100, n)
        np.testing.assert_array_equal(ref.idx, np.arange(min(100, n)))


def test_topk_cut_in_tail_bin_and_crowded_bin():
    rng = np.random.default_rng(33)
    N = 65536
    a = (0.5 * rng.standard_normal(N)).astype(np.float32)
    a[77] = 30.0                                                   # the rest lie in the tail bin
    b = rng.uniform(0.0, 0.003, N).astype(np.float32)              # one fine bin holds them all
    _check(np.stack([a, b]), 1000, "tail/crowded")


def test_topk_decode_workload_against_oracle():
    w = wl.DECODE_B8_N32K.replace(name="topk_wl", B=2, N=9000, needles=8)
    inst = wl.generate(w)
    q, k, v, P, lens = upload(inst)
    G, R = w.G, w.R
    k_idx = torch.zeros(w.B, R, w.N, 16, dtype=torch.bfloat16, device="cuda")
    q_idx = torch.zeros(w.B, R * G, 1, 16, dtype=torch.bfloat16, device="cuda")
    rtp.index_project(k[:, :R], P, k_idx)
    rtp.index_project(q[:, : R * G], P, q_idx)
    sel = rtp.Selection.empty(w.B * R * G, w.N, "cuda")
    rtp.topk_select(q_idx, k_idx, None, 500, sel)
    torch.cuda.synchronize()
    L = make_oracle(inst)
    mask = sel.mask.cpu().numpy().view(np.uint32)
    count = sel.count.cpu().numpy()
    for b in range(w.B):
        for h in range(R * G):
            s = oracle.indexer_scores(L.q_idx(b, h, 0), L.k_idx(b, h // G))
            ref = oracle.topk_select(s, 500)
            row = b * R * G + h
            compare_selection(SimpleNamespace(sel=ref, scores=s), mask[row], w.N, int(count[row]),
                              f"workload b{b} h{h}")
            assert int(count[row]) == 500

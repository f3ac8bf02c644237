"""GPU parity of rtp_topp_select (decode form) on score sets built to reach
each way the kernel finds the cut: the candidate path (a cut sub-bin with few
keys, exact ties among them included), and the key-window refinement taken
when the cut falls in the tail bin, when one CTA's share of the cut bin
overflows its list, or when the cut sub-bin holds too many keys.

The projected query is (4, 0, ..., 0) in fp32, so every indexer score equals
the first coordinate of its projected key exactly (s = 4 k_0 / 4), and the
oracle's cut is computed on those very fp32 values.
"""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_dim_b200 import rtp

from gpu_check import compare_selection

pytestmark = pytest.mark.gpu


def _select(scores_rows, p):
    """Run the decode select on one query per row of `scores_rows` ([B, N] fp32)."""
    s = np.asarray(scores_rows, dtype=np.float32)
    B, N = s.shape
    k_idx = np.zeros((B, 1, N, 16), np.float32)
    k_idx[:, 0, :, 0] = s
    q_idx = np.zeros((B, 1, 1, 16), np.float32)
    q_idx[..., 0] = 4.0
    dev = torch.device("cuda")
    qd = torch.from_numpy(q_idx).to(dev)
    kd = torch.from_numpy(k_idx).to(dev)
    sel = rtp.Selection.empty(B, N, dev)
    ws = rtp.workspace(rtp.topp_select_workspace_size(B, 1, 1, 1, N), dev)
    rtp.topp_select(qd, kd, None, p, sel, ws)
    torch.cuda.synchronize()
    assert rtp.poll_device_error() == 0
    return (sel.mask.cpu().numpy().view(np.uint32), sel.count.cpu().numpy(),
            sel.tau_bits.cpu().numpy().view(np.uint32), sel.tiepos.cpu().numpy())


def _check_rows(scores_rows, p, where):
    s32 = np.asarray(scores_rows, dtype=np.float32)
    p32 = float(np.float32(p))
    mask, count, tau_bits, tiepos = _select(s32, p)
    out = []
    for b in range(s32.shape[0]):
        s = s32[b].astype(np.float64)
        ref = oracle.topp_select(s, p32)
        compare_selection(SimpleNamespace(sel=ref, scores=s), mask[b], s.size, int(count[b]), f"{where} row {b}")
        # the threshold form describes the mask: s > tau, or s == tau at a position <= tiepos
        tau = np.uint32(tau_bits[b]).view(np.float32)
        bits = np.unpackbits(mask[b].view(np.uint8), bitorder="little")[: s.size].astype(bool)
        pos = np.arange(s.size)
        implied = (s32[b] > tau) | ((s32[b] == tau) & (pos <= tiepos[b]))
        assert np.array_equal(bits, implied), f"{where} row {b}: mask differs from (tau, tiepos)"
        out.append((ref, mask[b], int(count[b]), float(tau), int(tiepos[b])))
    return out


def test_select_candidate_path_random_scores():
    rng = np.random.default_rng(11)
    rows = rng.standard_normal((3, 50000)).astype(np.float32)
    for p in (0.5, 0.9, 0.99):
        _check_rows(rows, p, f"normal p={p}")


def test_select_candidate_path_exact_ties_at_the_cut():
    # 40 keys share one score; p is placed halfway through the mass of the
    # 20th of them (in position order), so the cut falls inside the tie group
    rng = np.random.default_rng(12)
    N = 20000
    s = rng.standard_normal(N).astype(np.float32)
    v = np.float32(np.sort(s)[N // 2])
    tie_pos = np.sort(rng.choice(N, size=40, replace=False))
    s[tie_pos] = v
    s64 = s.astype(np.float64)
    order = np.lexsort((np.arange(N), -s64))
    w = np.exp(s64[order] - s64.max())
    cum = np.cumsum(w)
    k20 = int(np.flatnonzero(order == tie_pos[19])[0])
    p = float(np.float32((cum[k20] - 0.5 * w[k20]) / cum[-1]))
    (ref, mask, count, tau, tp), = _check_rows(s[None], p, "ties")
    assert ref.tiepos == tie_pos[19] and tau == v and tp == tie_pos[19]
    assert count == ref.count
    bits = np.unpackbits(mask.view(np.uint8), bitorder="little")[:N].astype(bool)
    assert bits[tie_pos[:20]].all() and not bits[tie_pos[20:]].any()


def test_select_cut_in_tail_bin():
    # one key 20 nats above the rest: at p close to 1 the cut lies more than
    # 255/16 nats below the maximum, in the tail bin of the first pass
    rng = np.random.default_rng(13)
    N = 100000
    s = (0.5 * rng.standard_normal(N)).astype(np.float32)
    s[12345] = 20.0
    p = 0.99995
    (ref, *_), = _check_rows(s[None], p, "tail")
    assert ref.tau < 20.0 - 255.0 / 16.0


def test_select_cut_bin_overflows_the_list():
    # every key within 0.06 nat of the maximum: the whole sequence is one
    # first-pass bin, far more members per CTA than its list holds
    rng = np.random.default_rng(14)
    s = rng.uniform(0.0, 0.06, size=(1, 65536)).astype(np.float32)
    _check_rows(s, 0.5, "overflow")


def test_select_crowded_sub_bin():
    # 3000 distinct scores within 2e-4 nat: one sub-bin holds them all
    rng = np.random.default_rng(15)
    s = rng.uniform(0.0, 2e-4, size=(1, 3000)).astype(np.float32)
    _check_rows(s, 0.7, "crowded")


def test_select_mixed_rows_in_one_launch():
    # rows taking different paths side by side in one launch
    rng = np.random.default_rng(16)
    N = 30000
    a = rng.standard_normal(N).astype(np.float32)
    b = rng.uniform(0.0, 0.05, N).astype(np.float32)
    c = np.zeros(N, np.float32)
    d = (0.3 * rng.standard_normal(N)).astype(np.float32)
    d[7] = 25.0
    _check_rows(np.stack([a, b, c, d]), 0.9, "mixed p=0.9")
    _check_rows(np.stack([a, b, c, d]), 0.99999, "mixed p=0.99999")


def test_select_scores_streamed_past_the_resident_ones():
    # 700000 keys: 16 CTAs of 43776 keys, of which each keeps 32768 scores in
    # shared memory and recomputes the rest in every pass.  Random rows, a tie
    # group placed inside the recomputed parts with the cut in its middle, and a
    # row whose first-pass bin overflows (key-space passes over both parts)
    rng = np.random.default_rng(17)
    N, chunk = 700000, 43776
    a = rng.standard_normal(N).astype(np.float32)
    streamed = np.concatenate([np.arange(r * chunk + 32768, min((r + 1) * chunk, N)) for r in range(16)])
    tie_pos = np.sort(rng.choice(streamed, size=40, replace=False))
    t = rng.standard_normal(N).astype(np.float32)
    v = np.float32(np.sort(t)[N - 3000])
    t[t == v] = np.float32(v + 1e-3)
    t[tie_pos] = v
    t64 = t.astype(np.float64)
    order = np.lexsort((np.arange(N), -t64))
    w = np.exp(t64[order] - t64.max())
    cum = np.cumsum(w)
    k20 = int(np.flatnonzero(order == tie_pos[19])[0])
    p_tie = float(np.float32((cum[k20] - 0.5 * w[k20]) / cum[-1]))
    _check_rows(a[None], 0.9, "streamed normal")
    (ref, mask, count, tau, tp), = _check_rows(t[None], p_tie, "streamed ties")
    assert tau == v and tp == tie_pos[19] and count == ref.count
    u = rng.uniform(0.0, 0.06, size=(1, N)).astype(np.float32)
    _check_rows(u, 0.5, "streamed overflow")

"""GPU parity of rtp_topp_select (prefill form, tensor-core score tiles) on
score sets built to reach each way the kernel finds a row's cut:

  * the candidate path (a cut bin that ends with <= 32 keys), random scores;
  * exact ties straddling the cut: 20 ties (resolved among the candidates) and
    40 ties (more than a candidate list holds, so the bin is still too full
    after the last linear level and the exact score-key digits and the tie
    sweep finish the cut);
  * the cut in the tail bin of the first level (u >= 31, i.e. more than 7.75
    nat below the row maximum);
  * rows taking different paths side by side in one 128-row block.

Every projected key is (k0, 0, ..., 0) and every projected query (q0, 0, ...,
0) with bf16 values, so the indexer score of key j for query t is
q0_t * k0_j / 4 exactly (a product of two bf16 values is exact in fp32), and
the oracle's cut is computed on those very values.  Query t of the chunk sits
at position N - T + t and ranks keys 0 .. N - T + t.
"""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_dim_b200 import rtp

from gpu_check import compare_selection

pytestmark = pytest.mark.gpu


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _select(q0, k0, p):
    q0 = np.asarray(q0, np.float32)
    k0 = np.asarray(k0, np.float32)
    T, N = q0.size, k0.size
    dev = torch.device("cuda")
    q_idx = torch.zeros(1, 1, T, 16, dtype=torch.bfloat16, device=dev)
    k_idx = torch.zeros(1, 1, N, 16, dtype=torch.bfloat16, device=dev)
    q_idx[0, 0, :, 0] = torch.from_numpy(q0).to(dev, torch.bfloat16)
    k_idx[0, 0, :, 0] = torch.from_numpy(k0).to(dev, torch.bfloat16)
    sel = rtp.Selection.empty(T, N, dev)
    rtp.topp_select(q_idx, k_idx, None, p, sel)
    torch.cuda.synchronize()
    assert rtp.poll_device_error() == 0
    return (sel.mask.cpu().numpy().view(np.uint32), sel.count.cpu().numpy(),
            sel.tau_bits.cpu().numpy().view(np.uint32), sel.tiepos.cpu().numpy())


def _check(q0, k0, p, where, rows=None):
    """Every (or the listed) query row against the oracle; returns per-row results."""
    q0 = _bf16(q0)
    k0 = _bf16(k0)
    T, N = q0.size, k0.size
    p32 = float(np.float32(p))
    mask, count, tau_bits, tiepos = _select(q0, k0, p)
    out = {}
    for t in (range(T) if rows is None else rows):
        pos = N - T + t
        s = q0[t].astype(np.float64) * k0[: pos + 1].astype(np.float64) / 4.0
        ref = oracle.topp_select(s, p32)
        compare_selection(SimpleNamespace(sel=ref, scores=s), mask[t], pos + 1, int(count[t]), f"{where} t={t}")
        # the threshold form describes the mask exactly
        tau = np.uint32(tau_bits[t]).view(np.float32)
        s32 = s.astype(np.float32)
        bits = np.unpackbits(mask[t].view(np.uint8), bitorder="little")[: pos + 1].astype(bool)
        implied = (s32 > tau) | ((s32 == tau) & (np.arange(pos + 1) <= tiepos[t]))
        assert np.array_equal(bits, implied), f"{where} t={t}: mask differs from (tau, tiepos)"
        out[t] = (ref, mask[t], int(count[t]), float(tau), int(tiepos[t]))
    return out


@pytest.mark.parametrize("p", [0.5, 0.9, 0.99])
def test_prefill_select_random_scores_two_blocks(p):
    rng = np.random.default_rng(21)
    N, T = 40000, 256
    _check(np.full(T, 4.0), rng.standard_normal(N), p, f"normal p={p}")


def _ties_case(n_ties, seed):
    """Scores with `n_ties` keys sharing a value no other key has, and the p
    that puts the cut of the last row (which sees every key) halfway through
    the mass of the 20th tie in position order."""
    rng = np.random.default_rng(seed)
    N = 30000
    k0 = _bf16(rng.standard_normal(N))
    v = np.float32(0.3125)                 # exactly representable; clear it from the rest
    k0[k0 == v] = np.float32(0.31640625)   # the next bf16 value up
    tie_pos = np.sort(rng.choice(N, size=n_ties, replace=False))
    k0[tie_pos] = v
    s = k0.astype(np.float64)              # q0 = 4: score = k0
    order = np.lexsort((np.arange(N), -s))
    w = np.exp(s[order] - s.max())
    cum = np.cumsum(w)
    k20 = int(np.flatnonzero(order == tie_pos[19])[0])
    p = float(np.float32((cum[k20] - 0.5 * w[k20]) / cum[-1]))
    return k0, tie_pos, v, p


@pytest.mark.parametrize("n_ties", [20, 40])
def test_prefill_select_exact_ties_at_the_cut(n_ties):
    k0, tie_pos, v, p = _ties_case(n_ties, 22 + n_ties)
    N, T = k0.size, 128
    res = _check(np.full(T, 4.0), k0, p, f"{n_ties} ties")
    ref, mask, count, tau, tp = res[T - 1]
    assert ref.tiepos == tie_pos[19] and tau == v and tp == tie_pos[19]
    assert count == ref.count
    bits = np.unpackbits(mask.view(np.uint8), bitorder="little")[:N].astype(bool)
    assert bits[tie_pos[:20]].all() and not bits[tie_pos[20:]].any()


def test_prefill_select_cut_in_tail_bin():
    # one key 20 nats above the rest, seen by every row: at p close to 1 the
    # cut lies more than 7.75 nats below the maximum, in the first level's tail bin
    rng = np.random.default_rng(23)
    N, T = 20000, 128
    k0 = 0.5 * rng.standard_normal(N)
    k0[5] = 20.0
    res = _check(np.full(T, 4.0), k0, 0.999999, "tail")
    for ref, *_ in res.values():
        assert ref.tau < 20.0 - 7.75


def test_prefill_select_mixed_paths_in_one_block():
    # one 128-row block whose rows reach different paths: ordinary cuts (q0 = 4),
    # a sharp distribution whose cut is in the tail (q0 = 40 with a planted key),
    # reversed order (q0 = -4), all scores equal (q0 = 0: ties everywhere), and a
    # flat distribution whose cut bin is crowded (q0 = 0.015625)
    rng = np.random.default_rng(24)
    N, T = 12000, 128
    k0 = rng.standard_normal(N)
    k0[3] = 6.0
    choices = np.array([4.0, 40.0, -4.0, 0.0, 0.015625])
    q0 = choices[np.arange(T) % choices.size]
    _check(q0, k0, 0.9, "mixed p=0.9")
    _check(q0, k0, 0.9999, "mixed p=0.9999")


def test_prefill_select_long_cache_wide_level0_bins():
    # caches longer than 2^17 keys take level-0 bins of 1/2 nat (a 15.5-nat range
    # before the tail bin): an ordinary cut, and a cut in the (deeper) tail bin
    rng = np.random.default_rng(25)
    N, T = 140000, 128
    k0 = rng.standard_normal(N)
    _check(np.full(T, 4.0), k0, 0.95, "long p=0.95", rows=range(0, T, 9))
    k1 = 0.5 * rng.standard_normal(N)
    k1[11] = 22.0
    res = _check(np.full(T, 4.0), k1, 0.999999, "long tail", rows=range(0, T, 17))
    for ref, *_ in res.values():
        assert ref.tau < 22.0 - 15.5

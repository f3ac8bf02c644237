"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test fixes the oracle against something it does not compute itself: a
hand-derived fixture, a closed form, brute force over all subsets, an
independent library routine (torch's fp64 attention, torch's bf16 cast) or
an invariant.  ``test_mutants_are_caught`` plants plausible mistakes in a
copy of the oracle and checks that these pins reject each one.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import rtp_oracle as ro

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# --------------------------------------------------------------------------
# hand-derived fixtures
# --------------------------------------------------------------------------

def test_topp_hand_fixture():
    s = np.log(np.array([2.0, 4.0, 1.0, 4.0, 2.0]))
    for p, count, tiepos, sel in _read_rows("topp_hand.txt"):
        r = oracle.topp_select(s, float(p))
        assert r.count == int(count)
        assert r.tiepos == int(tiepos)
        assert r.idx.tolist() == [int(x) for x in sel.split(",")]
        assert r.tau == s[int(tiepos)]


def test_attention_hand_fixture():
    q = np.array([1.0, 0.0])
    K = np.array([[0.0, 5.0], [math.log(3.0), 1.0], [math.log(2.0), -7.0]])
    V = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, 2.0]])
    for sel, o0, o1 in _read_rows("attn_hand.txt"):
        idx = np.array([int(x) for x in sel.split(",")])
        o = oracle.attend(q, K, V, idx, 1.0)
        np.testing.assert_allclose(o, [float(o0), float(o1)], rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# storage rounding: independent routine (torch's float32 -> bf16 cast) and hand cases
# --------------------------------------------------------------------------

def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(20000), rng.standard_normal(2000) * 1e-30,
                        rng.standard_normal(2000) * 1e30]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x.astype(np.float64)), ref)


def test_round_bf16_hand_cases():
    h = 2.0 ** -8
    cases = {1.0 + h: 1.0, 1.0 + 3 * h: 1.0 + 4 * h, -(1.0 + h): -1.0, 0.0: 0.0,
             2.0 ** -130: 2.0 ** -130, 3.0: 3.0, 255.5: 256.0, 1.0 + 1.5 * h: 1.0 + 2 * h}
    for x, want in cases.items():
        assert oracle.round_bf16(np.array([x]))[0] == want, x


# --------------------------------------------------------------------------
# indexer: special cases
# --------------------------------------------------------------------------

def test_index_project_coordinate_selection_is_a_gather():
    from long_context_sparse_dim_b200.workloads import lowfreq_dims, lowfreq_projection
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 128))
    P = lowfreq_projection()
    np.testing.assert_array_equal(oracle.index_project(x, P), x[:, lowfreq_dims()])


def test_indexer_score_unit_query_reads_one_coordinate():
    rng = np.random.default_rng(2)
    k_idx = rng.standard_normal((40, 16))
    for i in (0, 7, 15):
        e = np.zeros(16)
        e[i] = 1.0
        np.testing.assert_array_equal(oracle.indexer_scores(e, k_idx), k_idx[:, i] / 4.0)


def test_indexer_score_is_bilinear_and_symmetric():
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal(16), rng.standard_normal(16)
    K = rng.standard_normal((9, 16))
    s_sum = oracle.indexer_scores(a + b, K)
    np.testing.assert_allclose(s_sum, oracle.indexer_scores(a, K) + oracle.indexer_scores(b, K), atol=1e-12)
    # s(a, b) == s(b, a)
    assert abs(oracle.indexer_scores(a, b[None])[0] - oracle.indexer_scores(b, a[None])[0]) < 1e-14
    # |a|^2 / 4 on itself
    assert abs(oracle.indexer_scores(a, a[None])[0] - a @ a / 4) < 1e-12


# --------------------------------------------------------------------------
# top-p: minimality, brute force, closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("p", [0.05, 0.5, 0.9, 0.99])
def test_topp_minimal_prefix(seed, p):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 400))
    s = rng.standard_normal(n) * float(rng.choice([0.3, 1.0, 4.0]))
    if seed % 2:
        s = np.round(s, 1)                       # many exact ties
    r = oracle.topp_select(s, p)
    w = np.exp(s - s.max())
    Z = w.sum()
    # prefix of the (s desc, pos asc) order
    order = sorted(range(n), key=lambda j: (-s[j], j))
    assert sorted(order[: r.count]) == r.idx.tolist()
    # mass reaches p and dropping the last key does not
    assert w[r.idx].sum() >= p * Z * (1 - 1e-12)
    assert w[order[: r.count - 1]].sum() < p * Z
    # the threshold form describes the same set
    pos = np.arange(n)
    thr = (s > r.tau) | ((s == r.tau) & (pos <= r.tiepos))
    assert np.flatnonzero(thr).tolist() == r.idx.tolist()


@pytest.mark.parametrize("seed", range(30))
def test_topp_brute_force_all_subsets(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 13))
    s = np.round(rng.standard_normal(n) * 1.5, 1 if seed % 3 == 0 else 6)
    p = float(rng.uniform(0.05, 0.999))
    r = oracle.topp_select(s, p)
    w = np.exp(s - s.max())
    target = p * w.sum()
    best = None
    for size in range(1, n + 1):
        masses = [w[list(c)].sum() for c in itertools.combinations(range(n), size)]
        if max(masses) >= target:
            best = size
            break
    assert r.count == best
    # no other subset of that size carries more mass
    top_mass = max(w[list(c)].sum() for c in itertools.combinations(range(n), best))
    assert abs(w[r.idx].sum() - top_mass) <= 1e-12 * top_mass


@pytest.mark.parametrize("n", [1, 2, 7, 100, 1001])
@pytest.mark.parametrize("p", [0.013, 0.37, 0.5, 0.81, 0.999])
def test_topp_all_equal_scores(n, p):
    # equal weights: ceil(p n) keys, the lowest positions (pins the tie-break)
    r = oracle.topp_select(np.full(n, 0.7), p)
    k = math.ceil(p * n - 1e-9)
    assert r.count == k
    assert r.idx.tolist() == list(range(k))
    assert r.tiepos == k - 1


def test_topp_single_dominant_key():
    s = np.zeros(50)
    s[17] = 10.0                                  # e^10 / (e^10 + 49) > 0.99
    r = oracle.topp_select(s, 0.99)
    assert r.idx.tolist() == [17]
    rng = np.random.default_rng(4)
    V = rng.standard_normal((50, 8))
    o = oracle.attend(np.zeros(8), rng.standard_normal((50, 8)), V, r.idx, 1.0)
    np.testing.assert_array_equal(o, V[17])


@pytest.mark.parametrize("na,nb,a,b,p", [(3, 40, 2.0, 0.0, 0.3), (3, 40, 2.0, 0.0, 0.9),
                                         (10, 10, 1.0, -1.0, 0.5), (1, 99, 5.0, 0.0, 0.8),
                                         (64, 4000, 1.0, 0.0, 0.95)])
def test_topp_two_level_closed_form(na, nb, a, b, p):
    # n_a keys at score a (> b), n_b at b: k* = ceil(pZ/e^a) if <= n_a, else n_a + ceil((pZ - n_a e^a)/e^b)
    rng = np.random.default_rng(na * 7 + nb)
    s = np.array([a] * na + [b] * nb)
    perm = rng.permutation(na + nb)
    s = s[perm]
    Z = na * math.exp(a) + nb * math.exp(b)
    k_a = math.ceil(p * Z / math.exp(a) - 1e-12)
    k = k_a if k_a <= na else na + math.ceil((p * Z - na * math.exp(a)) / math.exp(b) - 1e-12)
    r = oracle.topp_select(s, p)
    assert r.count == k
    hi = np.flatnonzero(s == a)
    lo = np.flatnonzero(s == b)
    want = sorted(hi[:k].tolist()) if k <= na else sorted(hi.tolist() + lo[: k - na].tolist())
    assert r.idx.tolist() == want


def test_topp_p_one_selects_everything_and_p_invalid():
    s = np.random.default_rng(0).standard_normal(33) * 30.0   # weights underflow to ~0
    assert oracle.topp_select(s, 1.0).count == 33
    for bad in (0.0, -0.5, float("nan")):
        with pytest.raises(ValueError):
            oracle.topp_select(s, bad)


def test_topp_signed_zero_and_negative_scores():
    s = np.array([-0.0, 0.0, -1.5, -0.0, -3.0])
    r = oracle.topp_select(s, 0.5)
    # -0 == +0: the three zero scores tie and are taken by position
    w = np.exp(s - 0.0)
    k = 1
    while w[[0, 1, 3][:k]].sum() < 0.5 * w.sum():
        k += 1
    assert r.idx.tolist() == [0, 1, 3][:k]


# --------------------------------------------------------------------------
# attention: p = 1 and W >= context reduce to full causal attention
# (independent library routine: torch scaled_dot_product_attention in fp64)
# --------------------------------------------------------------------------

def _sdpa_causal(q, k, v, lens_b, T, scale):
    """q [Hq, T, D], k/v [Hkv, n, D] -> [Hq, T, D]; queries are the last T of n positions."""
    Hq, Hkv = q.shape[0], k.shape[0]
    G = Hq // Hkv
    n = lens_b
    kk = torch.from_numpy(np.repeat(k[:, :n], G, axis=0)).double()
    vv = torch.from_numpy(np.repeat(v[:, :n], G, axis=0)).double()
    qq = torch.from_numpy(q).double()
    qpos = torch.arange(T) + n - T
    mask = torch.arange(n)[None, :] <= qpos[:, None]
    return torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale).numpy()


def _layer(seed, B=2, Hq=4, Hkv=2, R=1, N=70, T=70, W=16, p=0.9, storage="f64"):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, T, 32))
    k = rng.standard_normal((B, Hkv, N, 32))
    v = rng.standard_normal((B, Hkv, N, 32))
    P = rng.standard_normal((R, 16, 32))
    lens = np.array([N] * (B - 1) + [max(T, N - 9)])
    return q, k, v, P, lens


@pytest.mark.parametrize("T", [1, 5, 70])
def test_p_one_and_wide_window_equal_full_causal_attention(T):
    q, k, v, P, lens = _layer(7, T=T)
    N = k.shape[2]
    L = oracle.LayerOracle(q, k, v, P, lens, R=1, W=N + 5, p=1.0, storage="f64")
    res = L.run()
    for b in range(q.shape[0]):
        ref = _sdpa_causal(q[b], k[b], v[b], int(lens[b]), T, L.scale)
        got = np.stack([np.stack([res[(b, h, t)].o for t in range(T)]) for h in range(q.shape[1])])
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_window_equals_sdpa_band():
    q, k, v, P, lens = _layer(8, T=70, W=9)
    L = oracle.LayerOracle(q, k, v, P, lens, R=0, W=9, p=0.5, storage="f64")
    b, h = 1, 3
    n = int(lens[b])
    T = q.shape[2]
    qpos = np.arange(T) + n - T
    mask = (np.arange(n)[None, :] <= qpos[:, None]) & (np.arange(n)[None, :] > qpos[:, None] - 9)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[b, h][None]), torch.from_numpy(k[b, h // 2, :n][None]),
        torch.from_numpy(v[b, h // 2, :n][None]), attn_mask=torch.from_numpy(mask)[None], scale=L.scale)[0].numpy()
    got = np.stack([L.query(b, h, t).o for t in range(T)])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_window_one_returns_own_value():
    q, k, v, P, lens = _layer(9, T=4)
    L = oracle.LayerOracle(q, k, v, P, lens, R=0, W=1, p=0.5, storage="f64")
    for t in range(4):
        pos = L.pos(0, t)
        np.testing.assert_array_equal(L.query(0, 1, t).o, v[0, 0, pos])


def test_ragged_length_equals_truncated_cache():
    q, k, v, P, lens = _layer(10, T=1, N=50)
    lens = np.array([50, 31])
    L = oracle.LayerOracle(q, k, v, P, lens, R=1, W=8, p=0.8, storage="f64")
    Lt = oracle.LayerOracle(q[1:], k[1:, :, :31], v[1:, :, :31], P, [31], R=1, W=8, p=0.8, storage="f64")
    for h in range(4):
        np.testing.assert_array_equal(L.query(1, h, 0).o, Lt.query(0, h, 0).o)


def test_empty_candidate_set_gives_zero():
    q, k, v, P, lens = _layer(11, T=6, N=6)
    lens = np.array([6, 6])
    L = oracle.LayerOracle(q, k, v, P, lens, R=1, W=3, p=0.5, storage="f64")
    L.lens = np.array([6, 4])                   # two of the six queries sit before position 0
    assert L.query(1, 0, 0).sel.count == 0
    np.testing.assert_array_equal(L.query(1, 0, 0).o, 0.0)
    np.testing.assert_array_equal(L.query(1, 3, 1).o, 0.0)


# --------------------------------------------------------------------------
# needles: the planted keys are recalled (the pages' ">90% recall")
# --------------------------------------------------------------------------

def test_needle_recall_small_decode():
    from long_context_sparse_dim_b200 import workloads as wl
    inst = wl.generate(wl.DECODE_N4K_F32)
    L = oracle.LayerOracle(inst.q, inst.k, inst.v, inst.P, inst.lens, R=1, W=512, p=0.9, storage="f32")
    res = L.run()
    hit, tot = oracle.needle_recall(res, inst.needles)
    assert tot == 16
    assert hit / tot >= 0.9


# --------------------------------------------------------------------------
# the pins reject planted mistakes
# --------------------------------------------------------------------------

def _mutant_tie_high(s, p):
    s = np.asarray(s, dtype=np.float64)
    n = s.shape[0]
    w = np.exp(s - s.max())
    order = np.lexsort((-np.arange(n), -s))      # wrong: higher position first
    cum = np.cumsum(w[order])
    k = n if p >= 1 else int(np.searchsorted(cum, p * w.sum())) + 1
    return ro.Selection(np.sort(order[:k]), k, s[order[k - 1]], int(order[k - 1]), w.sum(), 0.0, order)


_TRUE_TOPP = ro.topp_select


def _mutant_off_by_one(s, p):
    r = _TRUE_TOPP(s, p)
    n = len(s)
    k = min(n, r.count + 1)
    return ro.Selection(np.sort(r.order[:k]), k, s[r.order[k - 1]], int(r.order[k - 1]), r.Z, 0.0, r.order)


def _mutant_no_temperature_shift(s, p):
    # wrong: weights exp(2 s) (a dropped /2 somewhere in the exponent)
    return _TRUE_TOPP(2.0 * np.asarray(s, dtype=np.float64), p)


@pytest.mark.parametrize("mutant", [_mutant_tie_high, _mutant_off_by_one, _mutant_no_temperature_shift])
def test_mutants_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(ro, "topp_select", mutant)
    monkeypatch.setattr(oracle, "topp_select", mutant)
    failures = 0
    for fn in (test_topp_hand_fixture,
               lambda: test_topp_all_equal_scores(7, 0.37),
               lambda: test_topp_two_level_closed_form(3, 40, 2.0, 0.0, 0.3)):
        try:
            fn()
        except AssertionError:
            failures += 1
    assert failures >= 1


# --------------------------------------------------------------------------
# head layout: grouped-query mapping and which heads are retrieval heads
# --------------------------------------------------------------------------

def test_gqa_mapping_and_head_roles():
    # V carries (position, KV head) in its first two coordinates.  Every query
    # head must read KV head h // G; local heads (KV head >= R) with W = 1 see
    # only their own position, retrieval heads with p = 1 see every key.
    rng = np.random.default_rng(7)
    B, Hq, Hkv, N, D, R = 2, 8, 4, 50, 16, 2
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, 1, D))
    k = rng.standard_normal((B, Hkv, N, D))
    v = np.zeros((B, Hkv, N, D))
    v[:, :, :, 0] = np.arange(N)[None, None, :]
    v[:, :, :, 1] = np.arange(Hkv)[None, :, None]
    lens = np.array([N, 37])
    P = np.zeros((R, 16, D))
    P[:, np.arange(16), np.arange(16)] = 1.0
    L = oracle.LayerOracle(q, k, v, P, lens, R=R, W=1, p=1.0, storage="f64")
    for b in range(B):
        pos = int(lens[b]) - 1
        for h in range(Hq):
            o = L.query(b, h, 0).o
            assert o[1] == pytest.approx(h // G)          # the KV head of the group
            if h // G >= R:
                assert o[0] == pytest.approx(pos)         # window of one key: the token itself
            else:
                assert 0.0 < o[0] < pos                   # an average over keys 0 .. pos


# --------------------------------------------------------------------------
# the fixed top-k variant (the budget the pages set dynamic top-p against)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_topk_k_one_is_the_first_argmax(seed):
    # k = 1 keeps the first occurrence of the maximum (numpy's argmax), ties included
    rng = np.random.default_rng(100 + seed)
    s = np.round(rng.standard_normal(40), 1)       # rounded: repeated values
    r = oracle.topk_select(s, 1)
    assert r.count == 1 and int(r.idx[0]) == int(np.argmax(s))


@pytest.mark.parametrize("seed,k", [(0, 3), (1, 10), (2, 39), (3, 40), (4, 55), (5, 17)])
def test_topk_invariants(seed, k):
    # |S| = min(k, n); every selected score >= every unselected one; among equal
    # scores at the boundary the selected positions precede the unselected ones
    rng = np.random.default_rng(200 + seed)
    s = np.round(rng.standard_normal(40), 1)
    r = oracle.topk_select(s, k)
    n = s.size
    assert r.count == min(k, n) == r.idx.size
    sel = np.zeros(n, bool)
    sel[r.idx] = True
    if sel.all():
        return
    assert s[sel].min() >= s[~sel].max()
    tau = s[sel].min()
    assert np.flatnonzero(sel & (s == tau)).max() < np.flatnonzero(~sel & (s == tau)).min() \
        if (~sel & (s == tau)).any() else True
    # the k largest values, as a multiset, are numpy's partition
    np.testing.assert_array_equal(np.sort(s[sel]), np.sort(np.partition(s, n - r.count)[n - r.count:]))


def test_topk_all_equal_keeps_the_lowest_positions():
    r = oracle.topk_select(np.zeros(30), 7)
    np.testing.assert_array_equal(r.idx, np.arange(7))
    assert r.tiepos == 6 and r.tau == 0.0


def test_topk_rejects_k_below_one():
    with pytest.raises(ValueError):
        oracle.topk_select(np.zeros(3), 0)


# --------------------------------------------------------------------------
# needle recall counts needles inside their query's SELECTED set only
# --------------------------------------------------------------------------

def test_needle_recall_hand_case():
    # query (0, 0, 0) selected keys {1, 4} out of candidates 0..5; its needles sit
    # at key 4 (selected) and key 2 (a candidate that was NOT selected); a needle
    # of a local head (no selection) is not counted
    sel = oracle.Selection(idx=np.array([1, 4]), count=2, tau=0.0, tiepos=4, Z=1.0, mass=1.0,
                           order=np.arange(6))
    res = {(0, 0, 0): oracle.QueryResult(np.zeros(4), sel, np.zeros(6)),
           (0, 5, 0): oracle.QueryResult(np.zeros(4), None, None)}
    needles = [(0, 0, 0, 0, 4), (0, 0, 0, 0, 2), (0, 1, 5, 0, 3)]
    assert oracle.needle_recall(res, needles) == (1, 2)


# --------------------------------------------------------------------------
# keys split by position over devices: per-range results and their merge
# --------------------------------------------------------------------------

def test_lse_closed_forms():
    rng = np.random.default_rng(40)
    q = rng.standard_normal(128)
    K = np.tile(rng.standard_normal(128), (5, 1))          # five identical keys
    V = rng.standard_normal((5, 128))
    scale = 1 / math.sqrt(128)
    a = float(K[0] @ q) * scale
    o, lse = oracle.attend_lse(q, K, V, np.arange(5), scale)
    assert lse == pytest.approx(a + math.log(5), rel=0, abs=1e-12)      # n equal logits: a + ln n
    np.testing.assert_allclose(o, V.mean(axis=0), rtol=1e-12, atol=1e-12)
    o1, lse1 = oracle.attend_lse(q, K, V, np.array([3]), scale)
    assert lse1 == pytest.approx(a, abs=1e-12)
    np.testing.assert_array_equal(o1, V[3])
    o0, lse0 = oracle.attend_lse(q, K, V, np.array([], dtype=np.int64), scale)
    assert lse0 == -np.inf and not o0.any()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_range_partials_merge_to_attention_over_the_union(seed):
    # softmax over a union of disjoint sets: independent check with torch's fp64
    # attention over the union, the set split into ranges (one of them empty)
    rng = np.random.default_rng(50 + seed)
    n = 300
    q = rng.standard_normal(128)
    K = 2.0 * rng.standard_normal((n, 128))
    V = rng.standard_normal((n, 128))
    idx = np.sort(rng.choice(n, size=170, replace=False))
    scale = 1 / math.sqrt(128)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[None, None]), torch.from_numpy(K[idx][None]), torch.from_numpy(V[idx][None]),
        scale=scale)[0, 0].numpy()
    bounds = [0, 64, 64, 192, n]                           # [64, 64) is empty
    parts = [oracle.attend_lse(q, K, V, idx[(idx >= lo) & (idx < hi)], scale) for lo, hi in zip(bounds, bounds[1:])]
    assert parts[1][1] == -np.inf
    np.testing.assert_allclose(oracle.combine_partials(parts), ref, rtol=1e-12, atol=1e-12)
    # a lone partial with lse 0 passes through unchanged
    np.testing.assert_array_equal(oracle.combine_partials([(parts[0][0], 0.0), (parts[2][0], -np.inf)]), parts[0][0])
    assert not oracle.combine_partials([(parts[1][0], -np.inf), (parts[1][0], -np.inf)]).any()

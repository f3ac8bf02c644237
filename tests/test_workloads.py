"""The seeded input generator (no GPU): rotary conventions, projection, needles."""
import numpy as np

from long_context_sparse_dim_b200 import workloads as wl


def test_lowfreq_dims_are_the_slowest_rotary_pairs():
    inv = wl.rope_inv_freq()
    dims = wl.lowfreq_dims()
    slow_pairs = np.argsort(inv)[:8]
    assert sorted(dims[:8].tolist()) == sorted(slow_pairs.tolist())
    assert (dims[8:] == dims[:8] + 64).all()
    P = wl.lowfreq_projection()
    assert P.shape == (16, 128) and P.sum() == 16 and (P.sum(axis=1) == 1).all()


def test_rope_is_a_rotation_with_relative_phase():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 128)).astype(np.float32)
    k = rng.standard_normal((1, 128)).astype(np.float32)
    a = wl.apply_rope(q, [1000])[0].astype(np.float64) @ wl.apply_rope(k, [990])[0].astype(np.float64)
    b = wl.apply_rope(q, [20])[0].astype(np.float64) @ wl.apply_rope(k, [10])[0].astype(np.float64)
    assert abs(a - b) < 1e-3
    assert abs(np.linalg.norm(wl.apply_rope(q, [12345])) - np.linalg.norm(q)) < 1e-3


def test_bf16_rounding_and_bits_roundtrip():
    x = np.random.default_rng(1).standard_normal(1000).astype(np.float32)
    r = wl.round_to_bf16(x)
    assert np.array_equal(wl.bits_to_f32(wl.bf16_bits(r)), r)
    assert np.max(np.abs(r - x) / np.abs(x)) <= 2.0 ** -8


def test_generate_is_deterministic_and_per_head_independent():
    w = wl.DECODE_B8_N32K.replace(B=2, N=512, needles=8, W=64)
    a = wl.generate(w)
    b = wl.generate(w, heads_kv=[1])
    assert np.array_equal(a.k[:, 1], b.k[:, 1]) and np.array_equal(a.q[:, 4:8], b.q[:, 4:8])
    assert not b.k[:, 0].any()
    assert len(a.needles) == 2 * 2 * 4 * 8
    pos = {(n[0], n[1], n[4]) for n in a.needles}
    assert len(pos) == len(a.needles)                       # distinct per (b, kv head)
    assert all(n[4] < 511 for n in a.needles)
    assert np.array_equal(wl.round_to_bf16(a.k), a.k)      # bf16 workload holds bf16 values


def test_prefill_needles_point_backwards():
    w = wl.PREFILL_N32K.replace(N=600, T=600, W=64)
    inst = wl.generate(w)
    assert len(inst.needles) == 2 * round(0.1 * 599)
    for b, kvh, h, t, j in inst.needles:
        assert j < inst.q_positions(b)[t] and h // w.G == kvh
    w5 = wl.PREFILL_CHUNK_1M.replace(N=4096, T=256, W=128, needle_count=32)
    inst5 = wl.generate(w5)
    assert len(inst5.needles) == 2 * 32
    assert all(j < 4096 - 256 for *_, j in inst5.needles)

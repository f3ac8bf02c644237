"""The key-range split of long-sequence decode (KeyRangeDecodeLayer) on CPU:
2 and 3 ranks over gloo, the library calls replaced by oracle stand-ins
(split_cpu_ops), against the oracle's unsplit layer.  What this checks is the
host logic of the split: the ranges and their padding, which rank computes
which local heads and the lse it reports for the others, the layout of the
all-gathered rows, and that the merge of the per-rank rows is the layer's
output on every rank.  The GPU kernels of the range attention and of the merge
are checked against the oracle on one GPU (emulated ranks) by
test_split_range_gpu.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from long_context_sparse_dim_b200 import workloads as wl
from long_context_sparse_dim_b200.split import key_ranges, local_head_block

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

WL = wl.DECODE_N4K_F32.replace(name="split_cpu", B=2, Hq=8, Hkv=4, R=2, N=300, W=40, p=0.9, needles=0,
                               ragged=True, seed=11)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_key_ranges_cover_the_sequence():
    for N, world in [(1, 1), (300, 2), (300, 3), (4096, 8), (1 << 20, 8), (65, 2)]:
        rs = key_ranges(N, world)
        rows = rs[0][1]
        assert rows % 64 == 0 and all(r == rows for _, r in rs)
        assert [lo for lo, _ in rs] == [r * rows for r in range(world)]
        assert rs[-1][0] < N <= rs[-1][0] + rows or world * rows - rows < N   # the last range reaches N
        assert world * rows >= N and (world - 1) * rows < N + rows
    blocks = [local_head_block(6, 8, r) for r in range(8)]
    assert blocks[0][0] == 0 and blocks[-1][1] == 6
    assert all(a[1] == b[0] for a, b in zip(blocks, blocks[1:]))
    assert sum(b - a for a, b in blocks) == 6


def _rank(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    sys.path.insert(0, TESTS)
    import torch.distributed as dist
    import split_cpu_ops
    from long_context_sparse_dim_b200.split import KeyRangeDecodeLayer
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inst = wl.generate(WL)
        q = torch.from_numpy(inst.q)
        k = torch.from_numpy(inst.k)
        v = torch.from_numpy(inst.v)
        P = torch.from_numpy(np.ascontiguousarray(inst.P)).float()
        lens = torch.from_numpy(inst.lens).int()
        B, R, N, W, D = WL.B, WL.R, WL.N, WL.W, 128
        key_lo, rows = key_ranges(N, world)[rank]
        k_range = torch.zeros(B, R, rows, D)
        v_range = torch.zeros(B, R, rows, D)
        hi = min(key_lo + rows, N)
        if hi > key_lo:
            k_range[:, :, : hi - key_lo] = k[:, :R, key_lo:hi]
            v_range[:, :, : hi - key_lo] = v[:, :R, key_lo:hi]
        k_idx = torch.zeros(B, R, N, 16)
        split_cpu_ops.index_project(k[:, :R], P, k_idx)
        # the local heads' windows: the last min(n, W) rows, in ring order
        L = WL.Hkv - R
        k_win = torch.zeros(B, L, W, D)
        v_win = torch.zeros(B, L, W, D)
        for b, n in enumerate(inst.lens.tolist()):
            for pos in range(max(0, n - W), n):
                k_win[b, :, pos % W] = k[b, R:, pos]
                v_win[b, :, pos % W] = v[b, R:, pos]
        win_lens = torch.clamp(lens, max=W)
        layer = KeyRangeDecodeLayer(q, k_range, v_range, k_idx, P, key_lo, k_win, v_win, win_lens, lens, R=R, W=W,
                                    p=WL.p, ops=split_cpu_ops)
        o = layer.step()
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o.double().numpy())
        np.save(os.path.join(out_dir, f"lse{rank}.npy"), layer.lse_part.double().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("world", [2, 3, 4])
def test_split_decode_matches_the_unsplit_oracle(world, tmp_path):
    import oracle
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    inst = wl.generate(WL)
    L = oracle.LayerOracle(inst.q, inst.k, inst.v, inst.P, inst.lens, R=WL.R, W=WL.W,
                           p=float(np.float32(WL.p)), storage="f32")
    ref = L.run()
    Hr = WL.R * WL.G
    outs = [np.load(tmp_path / f"o{r}.npy") for r in range(world)]
    for r in range(world):
        np.testing.assert_array_equal(outs[r], outs[0])          # the same output on every rank
        lse = np.load(tmp_path / f"lse{r}.npy")
        l0, l1 = local_head_block(WL.Hkv - WL.R, world, r)
        own = np.zeros(WL.Hq - Hr, bool)
        own[l0 * WL.G: l1 * WL.G] = True
        assert np.all(lse[:, Hr:][:, own] == 0.0) and np.all(np.isneginf(lse[:, Hr:][:, ~own]))
    for (b, h, t), res in ref.items():
        got = outs[0][b, h, t]
        np.testing.assert_allclose(got, res.o, rtol=0, atol=2e-6 * max(1.0, np.abs(res.o).max()),
                                   err_msg=f"b={b} h={h}")

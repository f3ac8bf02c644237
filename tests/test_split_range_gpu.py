"""GPU parity of the key-range split's kernels: rtp_sparse_attn_decode_range
(attention over the selected keys inside one range of positions, with its
log-sum-exp) and rtp_attn_combine (the merge), on one GPU with the ranks
emulated one after another (no kernel waits on another), against the oracle;
and KeyRangeDecodeLayer in a one-rank NCCL group against DecodeLayer."""
import math
import socket

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_dim_b200 import rtp
from long_context_sparse_dim_b200 import workloads as wl
from long_context_sparse_dim_b200.layer import DecodeLayer
from long_context_sparse_dim_b200.split import key_ranges

from gpu_check import make_oracle, mask_to_sets, rel_err, upload

pytestmark = pytest.mark.gpu

WL = wl.DECODE_B8_N32K.replace(name="split_gpu", B=2, N=9000, W=512, needles=0, ragged=True, seed=12)


def _selection(inst, q, k, P, lens):
    w = inst.wl
    R, G = w.R, w.G
    k_idx = torch.zeros(w.B, R, w.N, 16, dtype=torch.bfloat16, device="cuda")
    q_idx = torch.zeros(w.B, R * G, 1, 16, dtype=torch.bfloat16, device="cuda")
    rtp.index_project(k[:, :R], P, k_idx)
    rtp.index_project(q[:, : R * G], P, q_idx)
    sel = rtp.Selection.empty(w.B * R * G, w.N, "cuda")
    rtp.topp_select(q_idx, k_idx, lens, w.p, sel)
    return k_idx, sel


def _range_rows(x, lo, rows):
    out = torch.zeros(x.shape[0], x.shape[1], rows, x.shape[3], dtype=x.dtype, device=x.device)
    hi = min(lo + rows, x.shape[2])
    if hi > lo:
        out[:, :, : hi - lo] = x[:, :, lo:hi]
    return out


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_range_attention_and_merge_against_oracle(world):
    inst = wl.generate(WL)
    w = inst.wl
    q, k, v, P, lens = upload(inst)
    R, G = w.R, w.G
    Hr = R * G
    k_idx, sel = _selection(inst, q, k, P, lens)
    o_parts = torch.zeros(world, w.B, Hr, 128, dtype=torch.float32, device="cuda")
    lse_parts = torch.zeros(world, w.B, Hr, dtype=torch.float32, device="cuda")
    ranges = key_ranges(w.N, world)
    for r, (lo, rows) in enumerate(ranges):
        kr, vr = _range_rows(k[:, :R], lo, rows), _range_rows(v[:, :R], lo, rows)
        ws = rtp.workspace(rtp.sparse_attn_decode_workspace_size(w.B, Hr, R, rows), "cuda")
        rtp.sparse_attn_decode_range(q[:, :Hr], kr, vr, lens, sel, lo, 1 / math.sqrt(128),
                                     o_parts[r].unsqueeze(2), lse_parts[r], ws)
    o = torch.zeros(w.B, Hr, 1, 128, dtype=torch.float32, device="cuda")
    rtp.attn_combine(o_parts, lse_parts, o)
    # the unsplit kernel on the same selection
    o_full = torch.zeros_like(o)
    rtp.sparse_attn_decode(q[:, :Hr], k[:, :R], v[:, :R], lens, sel, 1 / math.sqrt(128), o_full,
                           rtp.workspace(rtp.sparse_attn_decode_workspace_size(w.B, Hr, R, w.N), "cuda"))
    torch.cuda.synchronize()
    mask = sel.mask.cpu().numpy().view(np.uint32)
    op, lp = o_parts.cpu().double().numpy(), lse_parts.cpu().double().numpy()
    L = make_oracle(inst)
    for b in range(w.B):
        n = int(inst.lens[b])
        for h in range(Hr):
            idx = mask_to_sets(mask[b * Hr + h], n)       # the GPU's own selection
            parts = []
            for r, (lo, rows) in enumerate(ranges):
                j = idx[(idx >= lo) & (idx < lo + rows)]
                ref_o, ref_lse = oracle.attend_lse(inst.q[b, h, 0], inst.k[b, h // G], inst.v[b, h // G], j,
                                                   L.scale)
                parts.append((ref_o, ref_lse))
                if j.size == 0:
                    assert np.isneginf(lp[r, b, h]) and not op[r, b, h].any(), f"empty range {r} b{b} h{h}"
                else:
                    assert abs(lp[r, b, h] - ref_lse) <= 1e-4 * max(1.0, abs(ref_lse)), f"lse r{r} b{b} h{h}"
                    assert rel_err(op[r, b, h], ref_o) <= 2e-3, f"o r{r} b{b} h{h}"
            ref = oracle.combine_partials(parts)
            got = o[b, h, 0].cpu().double().numpy()
            assert rel_err(got, ref) <= 2e-3, f"merged b{b} h{h}"
            assert rel_err(got, o_full[b, h, 0].cpu().double().numpy()) <= 1e-5, f"vs unsplit b{b} h{h}"


def test_combine_pass_through_and_empty_rows():
    rng = np.random.default_rng(3)
    S, B, Hq = 3, 2, 5
    x = torch.from_numpy(rng.standard_normal((S, B, Hq, 128)).astype(np.float32)).cuda()
    lse = torch.full((S, B, Hq), float("-inf"), device="cuda")
    lse[1, 0] = 0.0
    lse[2, 1, :3] = 0.0            # rows (1, 3), (1, 4) have no partial at all
    o = torch.full((B, Hq, 1, 128), 7.0, device="cuda")
    rtp.attn_combine(x, lse, o)
    torch.cuda.synchronize()
    assert torch.equal(o[0, :, 0], x[1, 0])                  # weight exactly 1: bit-identical
    assert torch.equal(o[1, :3, 0], x[2, 1, :3])
    assert not o[1, 3:].any()
    # two partials with equal lse: the mean; strided lse rows (a slice of a wider buffer)
    wide = torch.zeros(2, B, Hq + 3, device="cuda")
    ob = torch.empty(B, Hq, 1, 128, dtype=torch.bfloat16, device="cuda")
    rtp.attn_combine(x[:2], wide[:, :, :Hq], ob)
    torch.cuda.synchronize()
    ref = ((x[0] + x[1]) / 2).to(torch.bfloat16)
    assert (ob[:, :, 0].float() - ref.float()).abs().max() <= 1e-2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_key_range_layer_one_rank_nccl_matches_decode_layer():
    import torch.distributed as dist
    from long_context_sparse_dim_b200.split import KeyRangeDecodeLayer
    inst = wl.generate(WL)
    w = inst.wl
    q, k, v, P, lens = upload(inst)
    R = w.R
    ref = DecodeLayer(q, k, v, P, R=R, W=w.W, p=w.p, lens=lens)
    ref.build_index()
    o_ref = ref.step().clone()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        lo, rows = key_ranges(w.N, 1)[0]
        L = w.Hkv - R
        k_win = torch.zeros(w.B, L, w.W, 128, dtype=k.dtype, device="cuda")
        v_win = torch.zeros_like(k_win)
        for b, n in enumerate(inst.lens.tolist()):
            pos = torch.arange(max(0, n - w.W), n, device="cuda")
            k_win[b, :, pos % w.W] = k[b, R:, pos]
            v_win[b, :, pos % w.W] = v[b, R:, pos]
        win_lens = torch.clamp(lens, max=w.W)
        layer = KeyRangeDecodeLayer(q, _range_rows(k[:, :R], lo, rows), _range_rows(v[:, :R], lo, rows), ref.k_idx,
                                    P, lo, k_win, v_win, win_lens, lens, R=R, W=w.W, p=w.p)
        o = layer.step()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    Hr = R * w.G
    assert torch.equal(layer.sel.mask, ref.sel.mask)                 # the same selection bits
    assert rel_err(o[:, :Hr].cpu().double().numpy(), o_ref[:, :Hr].cpu().double().numpy()) <= 1e-5
    assert rel_err(o[:, Hr:].cpu().double().numpy(), o_ref[:, Hr:].cpu().double().numpy()) <= 1e-5
    res = make_oracle(inst).run([(b, h, 0) for b in range(w.B) for h in range(0, w.Hq, 5)])
    for (b, h, t), r in res.items():
        assert rel_err(o[b, h, 0].cpu().double().numpy(), r.o) <= 2e-3

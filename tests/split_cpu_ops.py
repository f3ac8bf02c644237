"""CPU stand-ins for the library calls KeyRangeDecodeLayer makes, written on
the oracle (test infrastructure): they let the multi-rank host logic of the
key-range split run over gloo on machines without a GPU.  Same signatures and
tensor layouts as long_context_sparse_dim_b200.rtp; every value is fp64
oracle arithmetic, stored into the caller's tensors."""
import numpy as np
import torch

import oracle
from long_context_sparse_dim_b200.rtp import Selection  # noqa: F401  (a plain dataclass of tensors)


def _storage(t):
    return "bf16" if t.dtype == torch.bfloat16 else "f32"


def workspace(nbytes, device):
    return None


def topp_select_workspace_size(*a):
    return 0


def sparse_attn_decode_workspace_size(*a):
    return 0


def window_attn_workspace_size(*a):
    return 0


def index_project(x, P, out, stream=None):
    H, HP = x.shape[1], P.shape[0]
    xs, Ps = x.double().numpy(), P.double().numpy()
    for h in range(H):
        out[:, h] = torch.from_numpy(oracle.index_project(xs[:, h], Ps[h // (H // HP)], _storage(out))).to(out.dtype)


def _lens(lens, B, N):
    return [N] * B if lens is None else [int(x) for x in lens.tolist()]


def topp_select(q_idx, k_idx, lens, p, sel, ws=None, stream=None):
    B, Hr = q_idx.shape[:2]
    G = Hr // k_idx.shape[1]
    N = k_idx.shape[2]
    mask = np.zeros((B * Hr, sel.mask.shape[1] * 32), dtype=bool)
    for b, n in enumerate(_lens(lens, B, N)):
        for h in range(Hr):
            s = oracle.indexer_scores(q_idx[b, h, 0].double().numpy(), k_idx[b, h // G, :n].double().numpy())
            r = oracle.topp_select(s, float(np.float32(p)))
            mask[b * Hr + h, r.idx] = True
            sel.count[b * Hr + h] = r.count
    sel.mask.copy_(torch.from_numpy(np.packbits(mask, axis=1, bitorder="little").view(np.int32)))


def sparse_attn_decode_range(q, k, v, lens, sel, key_lo, scale, o, lse, ws=None, stream=None):
    B, Hq = q.shape[:2]
    G = Hq // k.shape[1]
    rows = k.shape[2]
    bits = np.unpackbits(sel.mask.numpy().view(np.uint8), axis=1, bitorder="little").astype(bool)
    for b, n in enumerate(_lens(lens, B, key_lo + rows)):
        for h in range(Hq):
            j = np.flatnonzero(bits[b * Hq + h])
            j = j[(j >= key_lo) & (j < min(n, key_lo + rows))] - key_lo
            ob, lb = oracle.attend_lse(q[b, h, 0].double().numpy(), k[b, h // G].double().numpy(),
                                       v[b, h // G].double().numpy(), j, scale)
            o[b, h, 0] = torch.from_numpy(ob).to(o.dtype)
            lse[b, h] = lb


def window_attn(q, k, v, lens, W, scale, o, ws=None, stream=None):
    B, Hq = q.shape[:2]
    G = Hq // k.shape[1]
    for b, n in enumerate(_lens(lens, B, k.shape[2])):
        for h in range(Hq):
            r = oracle.local_query(q[b, h, 0].double().numpy(), k[b, h // G].double().numpy(),
                                   v[b, h // G].double().numpy(), n - 1, W, scale)
            o[b, h, 0] = torch.from_numpy(r.o).to(o.dtype)


def attn_combine(o_parts, lse_parts, o, stream=None):
    S, B, Hq = lse_parts.shape
    for b in range(B):
        for h in range(Hq):
            parts = [(o_parts[s, b, h].double().numpy(), float(lse_parts[s, b, h])) for s in range(S)]
            o[b, h, 0] = torch.from_numpy(oracle.combine_partials(parts)).to(o.dtype)

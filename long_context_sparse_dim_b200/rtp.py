"""ctypes binding of librtp.so (include/rtp.h): argument marshalling only.

Every function here has the C name without the ``rtp_`` prefix, takes torch
tensors that already live on the GPU, turns them into ``rtp_tensor``
descriptors and calls the library on the current torch stream (or the given
one).  A non-OK status raises :class:`RtpError`.  There is no fallback: if
the shared library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librtp.so")

RTP_OK = 0
RTP_F32, RTP_BF16 = 0, 1
STATUS_NAMES = {0: "RTP_OK", 1: "RTP_ERR_INVALID_ARG", 2: "RTP_ERR_SHAPE", 3: "RTP_ERR_DTYPE",
                4: "RTP_ERR_ALIGNMENT", 5: "RTP_ERR_WORKSPACE", 6: "RTP_ERR_CUDA", 7: "RTP_ERR_UNSUPPORTED"}

EXPORTED = ("rtp_index_project", "rtp_topp_select", "rtp_topp_select_workspace_size", "rtp_topk_select",
            "rtp_sparse_attn_decode", "rtp_sparse_attn_decode_workspace_size", "rtp_sparse_attn_decode_noalloc",
            "rtp_sparse_attn_prefill", "rtp_sparse_attn_prefill_workspace_size",
            "rtp_window_attn", "rtp_window_attn_workspace_size",
            "rtp_kv_append", "rtp_sparse_attn_decode_range", "rtp_attn_combine", "rtp_poll_device_error", "rtp_set_wait_budget_cycles", "rtp_status_string", "rtp_last_cuda_error",
            "rtp_version")


class RtpTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class RtpSelection(ctypes.Structure):
    _fields_ = [("tau_bits", ctypes.c_void_p), ("tiepos", ctypes.c_void_p), ("count", ctypes.c_void_p),
                ("mask", ctypes.c_void_p), ("mask_words", ctypes.c_int64)]


class RtpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS_NAMES.get(status, status)} ({_lib.rtp_status_string(status).decode()})"
        if status == 6:
            msg += f", cudaError {_lib.rtp_last_cuda_error()}"
        super().__init__(msg)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run python -m long_context_sparse_dim_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    T, S = P(RtpTensor), P(RtpSelection)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "rtp_index_project": ([T, T, T, vp], i32),
        "rtp_topp_select": ([T, T, vp, f32, S, vp, sz, vp], i32),
        "rtp_topp_select_workspace_size": ([i64, i64, i64, i64, i64], sz),
        "rtp_topk_select": ([T, T, vp, i32, S, vp, sz, vp], i32),
        "rtp_sparse_attn_decode": ([T, T, T, vp, S, f32, T, vp, sz, vp], i32),
        "rtp_sparse_attn_decode_workspace_size": ([i64, i64, i64, i64], sz),
        "rtp_sparse_attn_decode_noalloc": ([T, T, T, vp, S, f32, T, vp], i32),
        "rtp_sparse_attn_prefill": ([T, T, T, T, T, vp, S, f32, T, vp, sz, vp], i32),
        "rtp_sparse_attn_prefill_workspace_size": ([i64, i64, i64, i64, i64], sz),
        "rtp_window_attn": ([T, T, T, vp, i32, f32, T, vp, sz, vp], i32),
        "rtp_window_attn_workspace_size": ([i64, i64, i64, i64, i64, i32], sz),
        "rtp_sparse_attn_decode_range": ([T, T, T, vp, S, i64, f32, T, T, vp, sz, vp], i32),
        "rtp_attn_combine": ([T, T, T, vp], i32),
        "rtp_kv_append": ([T, T, vp, i32, T, T, T, T, T, T, vp, vp, vp], i32),
        "rtp_poll_device_error": ([P(i32)], i32),
        "rtp_set_wait_budget_cycles": ([i64], i32),
        "rtp_status_string": ([i32], ctypes.c_char_p),
        "rtp_last_cuda_error": ([], i32),
        "rtp_version": ([], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


# --------------------------------------------------------------------------
# marshalling
# --------------------------------------------------------------------------

def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RTP_F32
    if t.dtype == torch.bfloat16:
        return RTP_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def tensor_desc(t: torch.Tensor, ndim: int = 4) -> RtpTensor:
    if t.dim() != ndim:
        raise ValueError(f"expected a {ndim}-D tensor, got {tuple(t.shape)}")
    d = RtpTensor()
    d.data = t.data_ptr()
    d.dtype = _dt(t)
    d.ndim = ndim
    for i in range(ndim):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(status: int, where: str):
    if status != RTP_OK:
        raise RtpError(status, where)


@dataclass
class Selection:
    """Device arrays of rtp_selection for ``rows`` queries and ``N`` keys."""

    tau_bits: torch.Tensor
    tiepos: torch.Tensor
    count: torch.Tensor
    mask: Optional[torch.Tensor]

    @staticmethod
    def empty(rows: int, N: int, device, with_mask: bool = True) -> "Selection":
        words = max((N + 31) // 32, 1)
        return Selection(
            tau_bits=torch.empty(rows, dtype=torch.int32, device=device),
            tiepos=torch.empty(rows, dtype=torch.int32, device=device),
            count=torch.empty(rows, dtype=torch.int32, device=device),
            mask=torch.empty(rows, words, dtype=torch.int32, device=device) if with_mask else None)

    def desc(self) -> RtpSelection:
        s = RtpSelection()
        s.tau_bits = self.tau_bits.data_ptr()
        s.tiepos = self.tiepos.data_ptr()
        s.count = self.count.data_ptr()
        s.mask = self.mask.data_ptr() if self.mask is not None else None
        s.mask_words = self.mask.shape[1] if self.mask is not None else 0
        return s


def workspace(nbytes: int, device) -> Optional[torch.Tensor]:
    """A zero-filled workspace (256-byte aligned by the caching allocator)."""
    if nbytes == 0:
        return None
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def _ws(ws: Optional[torch.Tensor]):
    return (None, 0) if ws is None else (ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size())


# --------------------------------------------------------------------------
# the calls
# --------------------------------------------------------------------------

def index_project(x: torch.Tensor, P: torch.Tensor, x_idx: torch.Tensor, stream=None) -> None:
    _check(_lib.rtp_index_project(ctypes.byref(tensor_desc(x)), ctypes.byref(tensor_desc(P, 3)),
                                  ctypes.byref(tensor_desc(x_idx)), _stream(stream)), "rtp_index_project")


def _opt_desc(t: Optional[torch.Tensor], ndim: int = 4, keep=None):
    if t is None:
        return None
    d = tensor_desc(t, ndim)
    if keep is not None:
        keep.append(d)
    return ctypes.byref(d)


def _kv_append_args(k_new, v_new, pos, R, P, k_cache, v_cache, k_idx, k_ring, v_ring, lens_out, ring_lens,
                    stream, keep):
    return [_opt_desc(k_new, keep=keep), _opt_desc(v_new, keep=keep), _ptr(pos), ctypes.c_int32(int(R)),
            _opt_desc(P, 3, keep), _opt_desc(k_cache, keep=keep), _opt_desc(v_cache, keep=keep),
            _opt_desc(k_idx, keep=keep), _opt_desc(k_ring, keep=keep), _opt_desc(v_ring, keep=keep),
            _ptr(lens_out), _ptr(ring_lens), _stream(stream)]


def kv_append(k_new, v_new, pos, R: int, P=None, k_cache=None, v_cache=None, k_idx=None, k_ring=None,
              v_ring=None, lens_out=None, ring_lens=None, stream=None) -> None:
    """Append T new tokens per sequence: retrieval heads (the first R KV heads)
    to the full caches and the projected-key cache, local heads to W-row rings."""
    keep = []
    _check(_lib.rtp_kv_append(*_kv_append_args(k_new, v_new, pos, R, P, k_cache, v_cache, k_idx, k_ring, v_ring,
                                               lens_out, ring_lens, stream, keep)), "rtp_kv_append")


def topp_select_workspace_size(B, Hq, T, Hk, N) -> int:
    return int(_lib.rtp_topp_select_workspace_size(B, Hq, T, Hk, N))


def topp_select(q_idx: torch.Tensor, k_idx: torch.Tensor, lens: Optional[torch.Tensor], p: float,
                sel: Selection, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    w, nb = _ws(ws)
    _check(_lib.rtp_topp_select(ctypes.byref(tensor_desc(q_idx)), ctypes.byref(tensor_desc(k_idx)),
                                _ptr(lens), float(p), ctypes.byref(sel.desc()), w, nb, _stream(stream)),
           "rtp_topp_select")


def topk_select(q_idx: torch.Tensor, k_idx: torch.Tensor, lens: Optional[torch.Tensor], k: int,
                sel: Selection, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    w, nb = _ws(ws)
    _check(_lib.rtp_topk_select(ctypes.byref(tensor_desc(q_idx)), ctypes.byref(tensor_desc(k_idx)),
                                _ptr(lens), int(k), ctypes.byref(sel.desc()), w, nb, _stream(stream)),
           "rtp_topk_select")


def sparse_attn_decode_workspace_size(B, Hq, Hk, N) -> int:
    return int(_lib.rtp_sparse_attn_decode_workspace_size(B, Hq, Hk, N))


def sparse_attn_decode(q, k, v, lens, sel: Selection, scale: float, o, ws=None, stream=None) -> None:
    w, nb = _ws(ws)
    _check(_lib.rtp_sparse_attn_decode(ctypes.byref(tensor_desc(q)), ctypes.byref(tensor_desc(k)),
                                       ctypes.byref(tensor_desc(v)), _ptr(lens), ctypes.byref(sel.desc()),
                                       float(scale), ctypes.byref(tensor_desc(o)), w, nb, _stream(stream)),
           "rtp_sparse_attn_decode")


NOALLOC_SCRATCH_BYTES = 4 << 20


def sparse_attn_decode_range(q, k, v, lens, sel: Selection, key_lo: int, scale: float, o, lse, ws=None,
                            stream=None) -> None:
    """Attention over the selected keys among rows key_lo .. key_lo + N - 1 of
    each sequence (k, v hold just those rows); lse [B, Hq] f32 (last dim
    contiguous) receives the log-sum-exp for rtp_attn_combine."""
    w, nb = _ws(ws)
    _check(_lib.rtp_sparse_attn_decode_range(ctypes.byref(tensor_desc(q)), ctypes.byref(tensor_desc(k)),
                                             ctypes.byref(tensor_desc(v)), _ptr(lens), ctypes.byref(sel.desc()),
                                             int(key_lo), float(scale), ctypes.byref(tensor_desc(o)),
                                             ctypes.byref(tensor_desc(lse, 2)), w, nb, _stream(stream)),
           "rtp_sparse_attn_decode_range")


def attn_combine(o_parts, lse_parts, o, stream=None) -> None:
    """o [B, Hq, 1, 128] from S partials o_parts [S, B, Hq, 128] f32 and lse_parts [S, B, Hq] f32."""
    _check(_lib.rtp_attn_combine(ctypes.byref(tensor_desc(o_parts)), ctypes.byref(tensor_desc(lse_parts, 3)),
                                 ctypes.byref(tensor_desc(o)), _stream(stream)), "rtp_attn_combine")


def sparse_attn_decode_noalloc(q, k, v, lens, sel: Selection, scale: float, o, stream=None) -> None:
    """rtp_sparse_attn_decode without a workspace, for callers that cannot
    allocate device memory: the scratch is a fixed array inside the library
    (NOALLOC_SCRATCH_BYTES per device, shared by all calls; keep calls ordered
    on one stream, and make the first call on a device outside stream capture)."""
    _check(_lib.rtp_sparse_attn_decode_noalloc(ctypes.byref(tensor_desc(q)), ctypes.byref(tensor_desc(k)),
                                               ctypes.byref(tensor_desc(v)), _ptr(lens), ctypes.byref(sel.desc()),
                                               float(scale), ctypes.byref(tensor_desc(o)), _stream(stream)),
           "rtp_sparse_attn_decode_noalloc")


def sparse_attn_prefill_workspace_size(B, Hq, T, Hk, N) -> int:
    return int(_lib.rtp_sparse_attn_prefill_workspace_size(B, Hq, T, Hk, N))


def sparse_attn_prefill(q, k, v, q_idx, k_idx, lens, sel: Selection, scale: float, o, ws=None,
                        stream=None) -> None:
    w, nb = _ws(ws)
    _check(_lib.rtp_sparse_attn_prefill(ctypes.byref(tensor_desc(q)), ctypes.byref(tensor_desc(k)),
                                        ctypes.byref(tensor_desc(v)), ctypes.byref(tensor_desc(q_idx)),
                                        ctypes.byref(tensor_desc(k_idx)), _ptr(lens), ctypes.byref(sel.desc()),
                                        float(scale), ctypes.byref(tensor_desc(o)), w, nb, _stream(stream)),
           "rtp_sparse_attn_prefill")


def window_attn_workspace_size(B, Hq, T, Hk, N, W) -> int:
    return int(_lib.rtp_window_attn_workspace_size(B, Hq, T, Hk, N, W))


def window_attn(q, k, v, lens, W: int, scale: float, o, ws=None, stream=None) -> None:
    w, nb = _ws(ws)
    _check(_lib.rtp_window_attn(ctypes.byref(tensor_desc(q)), ctypes.byref(tensor_desc(k)),
                                ctypes.byref(tensor_desc(v)), _ptr(lens), int(W), float(scale),
                                ctypes.byref(tensor_desc(o)), w, nb, _stream(stream)), "rtp_window_attn")


# --------------------------------------------------------------------------
# bound calls: arguments marshalled once for buffers that do not change
# --------------------------------------------------------------------------

class Bound:
    """One C-ABI call whose arguments (descriptors, pointers, scalars, stream)
    were marshalled once; calling it re-issues the call with them.  Valid while
    the tensors it was built from keep their storage and shapes."""

    __slots__ = ("_fn", "_args", "_name", "_keep")

    def __init__(self, name: str, args, keep):
        self._fn = getattr(_lib, name)
        self._args = tuple(args)
        self._name = name
        self._keep = keep

    def __call__(self) -> None:
        status = self._fn(*self._args)
        if status != RTP_OK:
            raise RtpError(status, self._name)


def _ref(struct, keep):
    keep.append(struct)
    return ctypes.byref(struct)


def bind_index_project(x, P, x_idx, stream=None) -> Bound:
    keep = [x, P, x_idx]
    return Bound("rtp_index_project", [_ref(tensor_desc(x), keep), _ref(tensor_desc(P, 3), keep),
                                       _ref(tensor_desc(x_idx), keep), _stream(stream)], keep)


def bind_topp_select(q_idx, k_idx, lens, p: float, sel: Selection, ws=None, stream=None) -> Bound:
    keep = [q_idx, k_idx, lens, sel, ws]
    w, nb = _ws(ws)
    return Bound("rtp_topp_select", [_ref(tensor_desc(q_idx), keep), _ref(tensor_desc(k_idx), keep), _ptr(lens),
                                     ctypes.c_float(p), _ref(sel.desc(), keep), w, ctypes.c_size_t(nb),
                                     _stream(stream)], keep)


def bind_sparse_attn_decode(q, k, v, lens, sel: Selection, scale: float, o, ws=None, stream=None) -> Bound:
    keep = [q, k, v, lens, sel, o, ws]
    w, nb = _ws(ws)
    return Bound("rtp_sparse_attn_decode",
                 [_ref(tensor_desc(q), keep), _ref(tensor_desc(k), keep), _ref(tensor_desc(v), keep), _ptr(lens),
                  _ref(sel.desc(), keep), ctypes.c_float(scale), _ref(tensor_desc(o), keep), w,
                  ctypes.c_size_t(nb), _stream(stream)], keep)


def bind_window_attn(q, k, v, lens, W: int, scale: float, o, ws=None, stream=None) -> Bound:
    keep = [q, k, v, lens, o, ws]
    w, nb = _ws(ws)
    return Bound("rtp_window_attn",
                 [_ref(tensor_desc(q), keep), _ref(tensor_desc(k), keep), _ref(tensor_desc(v), keep), _ptr(lens),
                  ctypes.c_int32(W), ctypes.c_float(scale), _ref(tensor_desc(o), keep), w, ctypes.c_size_t(nb),
                  _stream(stream)], keep)


def bind_kv_append(k_new, v_new, pos, R: int, P=None, k_cache=None, v_cache=None, k_idx=None, k_ring=None,
                   v_ring=None, lens_out=None, ring_lens=None, stream=None) -> Bound:
    keep = [k_new, v_new, pos, P, k_cache, v_cache, k_idx, k_ring, v_ring, lens_out, ring_lens]
    return Bound("rtp_kv_append", _kv_append_args(k_new, v_new, pos, R, P, k_cache, v_cache, k_idx, k_ring,
                                                  v_ring, lens_out, ring_lens, stream, keep), keep)


def bind_sparse_attn_decode_range(q, k, v, lens, sel: Selection, key_lo: int, scale: float, o, lse, ws=None,
                                  stream=None) -> Bound:
    keep = [q, k, v, lens, sel, o, lse, ws]
    w, nb = _ws(ws)
    return Bound("rtp_sparse_attn_decode_range",
                 [_ref(tensor_desc(q), keep), _ref(tensor_desc(k), keep), _ref(tensor_desc(v), keep), _ptr(lens),
                  _ref(sel.desc(), keep), ctypes.c_int64(key_lo), ctypes.c_float(scale), _ref(tensor_desc(o), keep),
                  _ref(tensor_desc(lse, 2), keep), w, ctypes.c_size_t(nb), _stream(stream)], keep)


def bind_attn_combine(o_parts, lse_parts, o, stream=None) -> Bound:
    keep = [o_parts, lse_parts, o]
    return Bound("rtp_attn_combine", [_ref(tensor_desc(o_parts), keep), _ref(tensor_desc(lse_parts, 3), keep),
                                      _ref(tensor_desc(o), keep), _stream(stream)], keep)


def poll_device_error() -> int:
    """Synchronise, return and clear the device error word (0 = no error)."""
    code = ctypes.c_int32(0)
    _check(_lib.rtp_poll_device_error(ctypes.byref(code)), "rtp_poll_device_error")
    return int(code.value)


def set_wait_budget_cycles(cycles: int) -> None:
    """Budget of each bounded device wait in later prefill launches (0 = default)."""
    _check(_lib.rtp_set_wait_budget_cycles(int(cycles)), "rtp_set_wait_budget_cycles")


def version() -> int:
    return int(_lib.rtp_version())

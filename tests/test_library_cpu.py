"""librtp.so without a GPU: it loads, exports every declared symbol, and its
host-side validation rejects bad arguments before touching the device.

Every call below is built to FAIL validation (the pointers are fake), so
nothing here ever reaches a CUDA call.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from long_context_sparse_dim_b200 import build
    if not os.path.exists(build.LIB):
        build.build()
    from long_context_sparse_dim_b200 import rtp
    return rtp


def _declared():
    with open(os.path.join(ROOT, "include", "rtp.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"RTP_API\s+[\w\s\*]+?\b(rtp_\w+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = _declared()
    for n in ("rtp_index_project", "rtp_topp_select", "rtp_sparse_attn_decode", "rtp_sparse_attn_prefill",
              "rtp_window_attn"):
        assert n in names


def test_library_exports_every_declared_symbol():
    rtp = _lib()
    lib = rtp.lib()
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(rtp.EXPORTED)
    assert rtp.version() >= 100


def test_exports_only_the_c_abi():
    from long_context_sparse_dim_b200 import build
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True).stdout
    syms = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    ours = {s for s in syms if s.startswith("rtp_")}
    assert ours == set(_declared())


def _desc(rtp, shape, dtype=1, data=0x10000, strides=None):
    d = rtp.RtpTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, s in enumerate(shape):
        d.shape[i] = s
        d.stride[i] = strides[i]
    return d


def test_status_strings():
    rtp = _lib()
    for s in range(0, 8):
        assert rtp.lib().rtp_status_string(s)
    assert rtp.lib().rtp_status_string(99) == b"unknown status"


def test_index_project_validation():
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    x = _desc(rtp, [2, 2, 64, 128])
    P = _desc(rtp, [2, 16, 128], dtype=0)
    xi = _desc(rtp, [2, 2, 64, 16])
    assert L.rtp_index_project(None, by(P), by(xi), None) == 1
    assert L.rtp_index_project(by(_desc(rtp, [2, 2, 64, 128], data=0)), by(P), by(xi), None) == 1
    assert L.rtp_index_project(by(_desc(rtp, [2, 2, 64, 64])), by(P), by(xi), None) == 2          # D != 128
    assert L.rtp_index_project(by(x), by(P), by(_desc(rtp, [2, 2, 64, 8])), None) == 2          # d != 16
    assert L.rtp_index_project(by(x), by(P), by(_desc(rtp, [2, 2, 63, 16])), None) == 2         # N mismatch
    assert L.rtp_index_project(by(x), by(_desc(rtp, [3, 16, 128], dtype=0)), by(xi), None) == 2  # H % HP
    assert L.rtp_index_project(by(x), by(_desc(rtp, [2, 16, 128], dtype=1)), by(xi), None) == 3  # P not f32
    assert L.rtp_index_project(by(_desc(rtp, [2, 2, 64, 128], dtype=7)), by(P), by(xi), None) == 3
    assert L.rtp_index_project(by(_desc(rtp, [2, 2, 64, 128], data=0x10008)), by(P), by(xi), None) == 4
    bad_stride = _desc(rtp, [2, 2, 64, 128], strides=[2 * 64 * 130, 64 * 130, 130, 1])  # 260 B rows
    assert L.rtp_index_project(by(bad_stride), by(P), by(xi), None) == 4
    non_contig = _desc(rtp, [2, 2, 64, 128], strides=[2 * 64 * 256, 64 * 256, 256, 2])
    assert L.rtp_index_project(by(non_contig), by(P), by(xi), None) == 4


def _sel(rtp, mask=True, words=2):
    s = rtp.RtpSelection()
    s.tau_bits = 0x20000
    s.tiepos = 0x30000
    s.count = 0x40000
    s.mask = 0x50000 if mask else None
    s.mask_words = words
    return s


def test_topp_select_validation():
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    qi = _desc(rtp, [2, 8, 1, 16])
    ki = _desc(rtp, [2, 2, 64, 16])
    s = _sel(rtp)
    assert L.rtp_topp_select(by(qi), by(ki), None, 0.0, by(s), None, 0, None) == 1      # p <= 0
    assert L.rtp_topp_select(by(qi), by(ki), None, -1.0, by(s), None, 0, None) == 1
    assert L.rtp_topp_select(by(qi), by(ki), None, float("nan"), by(s), None, 0, None) == 1
    assert L.rtp_topp_select(by(qi), by(ki), None, 0.9, None, None, 0, None) == 1
    assert L.rtp_topp_select(by(qi), by(ki), None, 0.9, by(_sel(rtp, words=1)), None, 0, None) == 2
    assert L.rtp_topp_select(by(_desc(rtp, [2, 7, 1, 16])), by(ki), None, 0.9, by(s), None, 0, None) == 2
    assert L.rtp_topp_select(by(_desc(rtp, [3, 8, 1, 16])), by(ki), None, 0.9, by(s), None, 0, None) == 2
    assert L.rtp_topp_select(by(_desc(rtp, [2, 8, 1, 16], dtype=0)), by(ki), None, 0.9, by(s), None, 0,
                             None) == 3


def test_attention_validation():
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    q = _desc(rtp, [2, 8, 1, 128])
    k = _desc(rtp, [2, 2, 64, 128])
    o = _desc(rtp, [2, 8, 1, 128], dtype=0)
    s = _sel(rtp)
    # no workspace
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(k), None, by(s), 0.088, by(o), None, 0, None) == 5
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(k), None, by(s), 0.088, by(o), 0x100000, 16, None) == 5
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(k), None, by(s), 0.088, by(o), 0x100010, 1 << 30, None) == 4
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(k), None, by(_sel(rtp, mask=False)), 0.088, by(o), None, 0,
                                    None) == 1
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(k), None, by(s), float("inf"), by(o), None, 0, None) == 1
    assert L.rtp_sparse_attn_decode(by(_desc(rtp, [2, 18, 1, 128])), by(_desc(rtp, [2, 2, 64, 128])),
                                    by(_desc(rtp, [2, 2, 64, 128])), None, by(s), 0.088,
                                    by(_desc(rtp, [2, 18, 1, 128], dtype=0)), None, 0, None) == 2   # G = 9 > 8
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(_desc(rtp, [2, 2, 65, 128])), None, by(s), 0.088, by(o),
                                    None, 0, None) == 2
    assert L.rtp_sparse_attn_decode(by(q), by(k), by(_desc(rtp, [2, 2, 64, 128], dtype=0)), None, by(s), 0.088,
                                    by(o), None, 0, None) == 3
    assert L.rtp_window_attn(by(q), by(k), by(k), None, 0, 0.088, by(o), None, 0, None) == 1       # W < 1
    assert L.rtp_window_attn(by(q), by(k), by(k), None, 16, 0.088, by(o), None, 0, None) == 5
    assert L.rtp_window_attn(by(q), by(k), by(k), None, 16, 0.088, by(_desc(rtp, [2, 8, 2, 128], dtype=0)),
                             None, 0, None) == 2


def test_workspace_sizes_are_monotone():
    rtp = _lib()
    a = rtp.sparse_attn_decode_workspace_size(8, 8, 2, 32768)
    b = rtp.sparse_attn_decode_workspace_size(8, 8, 2, 131072)
    assert 0 < a <= b
    assert rtp.window_attn_workspace_size(8, 24, 1, 6, 32768, 4096) > 0
    assert rtp.topp_select_workspace_size(8, 8, 1, 2, 32768) == 0


def test_bench_traffic_record_follows_the_kernels_device_code(tmp_path, monkeypatch):
    # the DRAM-traffic figure is reported while the kernel's device code (the
    # source up to its host-side section) is the one the counters were taken on
    import hashlib
    import json
    import bench
    src = tmp_path / "k.cu"
    device = "__global__ void k() {}\n"
    src.write_text(device + bench.HOST_SIDE_MARKER + " ----\nint host() { return 1; }\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"kern": {"dram_bytes_retrieval_launch": 123, "source": "k.cu",
                    "device_code_sha1": hashlib.sha1(device.encode()).hexdigest()}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic_record("kern")["dram_bytes_retrieval_launch"] == 123
    src.write_text(device + bench.HOST_SIDE_MARKER + " ----\nint host() { return 2; }\n")  # host side only
    assert bench._traffic_record("kern") is not None
    src.write_text("__global__ void k() { int x; }\n" + bench.HOST_SIDE_MARKER + "\n")   # device code changed
    assert bench._traffic_record("kern") is None
    assert bench._traffic_record("other") is None


class _FakeStream:
    """Stands in for a CUDA stream handle when only the marshalling is checked."""

    def __init__(self, handle):
        self.cuda_stream = handle

    def __int__(self):
        return self.cuda_stream


def _descs(bound, rtp):
    return [x for x in bound._keep if isinstance(x, rtp.RtpTensor)]


def test_decode_layer_marshals_each_call_of_the_step():
    # the calls of one decode step, marshalled once: which calls, in which
    # order, on which stream, and the exact views they are given
    import torch
    rtp = _lib()
    from long_context_sparse_dim_b200.layer import DecodeLayer
    B, Hq, Hkv, N, D, R, W = 2, 8, 2, 300, 128, 1, 64
    G = Hq // Hkv
    q = torch.zeros(B, Hq, 1, D, dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, N, D, dtype=torch.bfloat16)
    v = torch.zeros(B, Hkv, N, D, dtype=torch.bfloat16)
    P = torch.zeros(R, 16, D)
    layer = DecodeLayer(q, k, v, P, R=R, W=W, p=0.9)
    main, side = _FakeStream(11), _FakeStream(22)
    pre, win, chain = layer._plan(main, side)
    assert [c._name for c in pre] == ["rtp_index_project", "rtp_index_project"]
    assert [c._name for c in win] == ["rtp_window_attn"]
    assert [c._name for c in chain] == ["rtp_topp_select", "rtp_sparse_attn_decode"]
    for c in pre + chain:
        assert c._args[-1].value == 11
    assert win[0]._args[-1].value == 22
    # the newest key row of the retrieval heads, a strided view of the cache
    kx, kp, ko = _descs(pre[0], rtp)
    assert list(kx.shape) == [B, R, 1, D] and list(kx.stride) == [Hkv * N * D, N * D, D, 1]
    assert kx.data == k.data_ptr() + (N - 1) * D * 2
    assert list(kp.shape)[:3] == [R, 16, D] and kp.ndim == 3
    assert list(ko.shape) == [B, R, 1, 16] and ko.data == layer.k_idx.data_ptr() + (N - 1) * 16 * 2
    # queries of the retrieval heads -> q_idx
    qx, _, qo = _descs(pre[1], rtp)
    assert list(qx.shape) == [B, R * G, 1, D] and qx.data == q.data_ptr()
    assert list(qo.shape) == [B, R * G, 1, 16]
    # window attention over the local heads: views starting at KV head R
    wq, wk, wv, wo = _descs(win[0], rtp)
    assert list(wq.shape) == [B, Hq - R * G, 1, D] and wq.data == q.data_ptr() + R * G * D * 2
    assert list(wk.shape) == [B, Hkv - R, N, D] and wk.data == k.data_ptr() + R * N * D * 2
    assert wv.data == v.data_ptr() + R * N * D * 2
    assert list(wo.shape) == [B, Hq - R * G, 1, D]
    # the selection's descriptors, then the sparse attention's
    sq, sk = _descs(chain[0], rtp)[:2]
    assert sq.data == layer.q_idx.data_ptr() and sk.data == layer.k_idx.data_ptr()
    aq, ak, av, ao = _descs(chain[1], rtp)
    assert list(ak.shape) == [B, R, N, D] and ak.data == k.data_ptr()
    assert list(ao.shape) == [B, R * G, 1, D] and ao.data == layer.o.data_ptr()


def test_decode_layer_host_plan_appends_the_new_rows():
    # the host-buffer step appends the staged new rows with rtp_kv_append (retrieval
    # heads to their caches and projected keys, local heads to their full caches used
    # as rings of N rows) and then projects only the queries
    import torch
    rtp = _lib()
    from long_context_sparse_dim_b200.layer import DecodeLayer
    B, Hq, Hkv, N, D, R, W = 2, 8, 2, 300, 128, 1, 64
    G = Hq // Hkv
    q = torch.zeros(B, Hq, 1, D, dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, N, D, dtype=torch.bfloat16)
    v = torch.zeros(B, Hkv, N, D, dtype=torch.bfloat16)
    P = torch.zeros(R, 16, D)
    layer = DecodeLayer(q, k, v, P, R=R, W=W, p=0.9)
    k_new = torch.zeros(B, Hkv, 1, D, dtype=torch.bfloat16)
    v_new = torch.zeros_like(k_new)
    pos = torch.tensor([N - 1, N - 1], dtype=torch.int32)
    main, side = _FakeStream(11), _FakeStream(22)
    pre, win, chain = layer._plan(main, side, new_rows=(k_new, v_new, pos))
    assert [c._name for c in pre] == ["rtp_kv_append", "rtp_index_project"]
    assert [c._name for c in win] == ["rtp_window_attn"]
    assert [c._name for c in chain] == ["rtp_topp_select", "rtp_sparse_attn_decode"]
    app = pre[0]._args
    assert app[2].value == pos.data_ptr() and app[3].value == R
    assert app[10] is None and app[11] is None and app[-1].value == 11  # no lengths written
    kn, vn, Pd, kc, vc, ki, kr, vr = _descs(pre[0], rtp)
    assert kn.data == k_new.data_ptr() and vn.data == v_new.data_ptr()
    assert kc.data == k.data_ptr() and list(kc.shape) == [B, R, N, D]
    assert ki.data == layer.k_idx.data_ptr() and list(ki.shape) == [B, R, N, 16]
    assert kr.data == k.data_ptr() + R * N * D * 2 and list(kr.shape) == [B, Hkv - R, N, D]
    assert vr.data == v.data_ptr() + R * N * D * 2
    qx, _, qo = _descs(pre[1], rtp)
    assert list(qx.shape) == [B, R * G, 1, D] and qo.data == layer.q_idx.data_ptr()
    # every head a retrieval head: no rings
    layer2 = DecodeLayer(q, k, v, torch.zeros(Hkv, 16, D), R=Hkv, W=W, p=0.9)
    pre2, win2, _ = layer2._plan(main, side, new_rows=(k_new, v_new, pos))
    assert win2 == [] and pre2[0]._args[8] is None and pre2[0]._args[9] is None


def test_host_steps_take_pinned_buffers_only():
    import torch
    _lib()
    from long_context_sparse_dim_b200.layer import DecodeLayer, PrefillLayer
    B, Hq, Hkv, N, T, D = 1, 8, 2, 256, 256, 128
    q = torch.zeros(B, Hq, T, D, dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, N, D, dtype=torch.bfloat16)
    v = torch.zeros(B, Hkv, N, D, dtype=torch.bfloat16)
    P = torch.zeros(1, 16, D)
    pl = PrefillLayer(q, k, v, P, R=1, W=64, p=0.9)
    with pytest.raises(ValueError):
        pl.host_step(q, k, v, torch.zeros(B, Hq, T, D))  # not pinned
    dl = DecodeLayer(q[:, :, :1], k, v, P, R=1, W=64, p=0.9)
    with pytest.raises(ValueError):
        dl.host_step(q[:, :, :1], k[:, :, :1], v[:, :, :1], torch.zeros(B, Hq, 1, D))


def test_header_is_plain_c_and_links_against_the_library(tmp_path):
    # include/rtp.h is a C header (C99, no C++), and a C program links
    # against librtp.so by the names it declares
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    rtp = _lib()
    src = tmp_path / "use.c"
    src.write_text(
        '#include "rtp.h"\n'
        "int main(void) {\n"
        "  size_t ws = rtp_topp_select_workspace_size(1, 8, 1, 2, 4096)\n"
        "            + rtp_sparse_attn_decode_workspace_size(1, 8, 2, 4096)\n"
        "            + rtp_window_attn_workspace_size(1, 24, 1, 6, 4096, 512);\n"
        "  return (rtp_version() > 0 && ws > 0 && rtp_status_string(RTP_OK) != 0) ? 0 : 1;\n"
        "}\n")
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(rtp.LIB_PATH)
    exe = tmp_path / "use"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", str(src), "-I", inc,
                        "-L", libdir, "-lrtp", "-Wl,-rpath," + libdir, "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0


def test_noalloc_scratch_size_matches_the_header():
    # the Python wrapper's copy of RTP_NOALLOC_SCRATCH_BYTES is the header's value
    rtp = _lib()
    with open(os.path.join(ROOT, "include", "rtp.h")) as f:
        m = re.search(r"#define\s+RTP_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    assert m, "RTP_NOALLOC_SCRATCH_BYTES not found in rtp.h"
    assert int(m.group(1)) << int(m.group(2)) == rtp.NOALLOC_SCRATCH_BYTES


def test_noalloc_validates_before_touching_the_device():
    # on a machine without a GPU any CUDA call would fail with RTP_ERR_CUDA (6):
    # an invalid call must be refused by the argument checks alone
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    q = _desc(rtp, [2, 8, 1, 128])
    k = _desc(rtp, [2, 2, 64, 128])
    o = _desc(rtp, [2, 8, 1, 128], dtype=0)
    s = _sel(rtp)
    fn = L.rtp_sparse_attn_decode_noalloc
    assert fn(by(q), by(k), by(k), None, None, 0.088, by(o), None) == 1                       # no selection
    assert fn(by(q), by(k), by(k), None, by(_sel(rtp, mask=False)), 0.088, by(o), None) == 1  # no mask
    assert fn(by(q), by(k), by(k), None, by(s), float("nan"), by(o), None) == 1               # bad scale
    assert fn(by(_desc(rtp, [2, 8, 2, 128])), by(k), by(k), None, by(s), 0.088,
              by(_desc(rtp, [2, 8, 2, 128], dtype=0)), None) == 2                             # T != 1
    assert fn(by(q), by(k), by(_desc(rtp, [2, 2, 64, 128], dtype=0)), None, by(s), 0.088, by(o), None) == 3
    big = _desc(rtp, [4096, 32, 1, 128])
    kv = _desc(rtp, [4096, 8, 4096, 128])
    assert fn(by(big), by(kv), by(kv), None, by(_sel(rtp, words=128)), 0.088,
              by(_desc(rtp, [4096, 32, 1, 128], dtype=0)), None) == 7                         # beyond the scratch


def test_wait_budget_setter_validates():
    rtp = _lib()
    with pytest.raises(rtp.RtpError):
        rtp.set_wait_budget_cycles(-1)
    rtp.set_wait_budget_cycles(0)  # restores the default


def test_topk_select_validation():
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    qi = _desc(rtp, [2, 8, 1, 16])
    ki = _desc(rtp, [2, 2, 64, 16])
    s = _sel(rtp)
    assert L.rtp_topk_select(by(qi), by(ki), None, 0, by(s), None, 0, None) == 1          # k < 1
    assert L.rtp_topk_select(by(qi), by(ki), None, 5, None, None, 0, None) == 1           # no selection
    assert L.rtp_topk_select(by(_desc(rtp, [2, 8, 3, 16])), by(ki), None, 5, by(s), None, 0, None) == 7  # T != 1
    assert L.rtp_topk_select(by(_desc(rtp, [2, 7, 1, 16])), by(ki), None, 5, by(s), None, 0, None) == 2


def test_kv_append_validation():
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    B, H, R, T, N, W = 2, 4, 1, 3, 64, 16
    kn = _desc(rtp, [B, H, T, 128])
    P = _desc(rtp, [R, 16, 128], dtype=0)
    kc = _desc(rtp, [B, R, N, 128])
    ki = _desc(rtp, [B, R, N, 16])
    kr = _desc(rtp, [B, H - R, W, 128])
    pos, out, rl = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), ctypes.c_void_p(0x40000)
    fn = L.rtp_kv_append

    def call(pos=pos, R=R, P=by(P), kc=by(kc), ki=by(ki), kr=by(kr), out=out, rl=rl, kn=by(kn)):
        return fn(kn, kn, pos, R, P, kc, kc, ki, kr, kr, out, rl, None)

    assert call(pos=None) == 1                                    # no positions
    assert call(R=5) == 1 and call(R=-1) == 1                     # R outside [0, H]
    assert call(out=pos) == 1 and call(rl=pos) == 1 and call(out=rl) == 1   # aliased length buffers
    assert call(P=None) == 1                                      # retrieval heads need P
    assert call(kr=None) == 1                                     # local heads need a ring
    assert call(P=by(_desc(rtp, [2, 16, 128], dtype=0))) == 2     # one P per retrieval head
    assert call(P=by(_desc(rtp, [R, 16, 128]))) == 3              # P is f32
    assert call(kc=by(_desc(rtp, [B, 2, N, 128]))) == 2           # cache heads != R
    assert call(ki=by(_desc(rtp, [B, R, N + 1, 16]))) == 2        # projected rows != cache rows
    assert call(kc=by(_desc(rtp, [B, R, N, 128], dtype=0))) == 3  # cache dtype != new rows
    assert call(kr=by(_desc(rtp, [B, H - R, 0, 128]))) == 2       # an empty ring
    assert call(kr=by(_desc(rtp, [B + 1, H - R, W, 128]))) == 2   # ring batch != B
    assert call(kn=by(_desc(rtp, [B, H, T, 64]))) == 2            # head dim 128
    # all heads retrieval heads: no ring, and no ring lengths
    assert fn(by(kn), by(kn), pos, H, by(_desc(rtp, [H, 16, 128], dtype=0)), by(_desc(rtp, [B, H, N, 128])),
              by(_desc(rtp, [B, H, N, 128])), by(_desc(rtp, [B, H, N, 16])), None, None, out, rl, None) == 1


def test_cached_decode_layer_marshals_append_then_the_step():
    import torch
    rtp = _lib()
    from long_context_sparse_dim_b200.layer import CachedDecodeLayer
    B, Hq, Hkv, N, D, R, W = 2, 8, 2, 300, 128, 1, 64
    G = Hq // Hkv
    P = torch.zeros(R, 16, D)
    layer = CachedDecodeLayer(B, Hq, Hkv, N, R, W, 0.9, P, device="cpu")
    main, side = _FakeStream(11), _FakeStream(22)
    for cur in (0, 1):
        pre, win, chain = layer._plan(cur, main, side)
        assert [c._name for c in pre] == ["rtp_kv_append", "rtp_index_project"]
        assert [c._name for c in win] == ["rtp_window_attn"]
        assert [c._name for c in chain] == ["rtp_topp_select", "rtp_sparse_attn_decode"]
        app = pre[0]._args
        pos, lens = layer._lens[cur], layer._lens[1 - cur]
        assert app[2].value == pos.data_ptr() and app[10].value == lens.data_ptr()
        assert app[11].value == layer.ring_lens.data_ptr() and app[3].value == R
        kn, vn, Pd, kc, vc, ki, kr, vr = _descs(pre[0], rtp)
        assert list(kn.shape) == [B, Hkv, 1, D] and kn.data == layer.k_new.data_ptr()
        assert list(kc.shape) == [B, R, N, D] and list(kr.shape) == [B, Hkv - R, W, D]
        assert list(ki.shape) == [B, R, N, 16] and Pd.ndim == 3
        # the selection and sparse attention read the lengths the append writes
        assert chain[0]._args[2].value == lens.data_ptr() and chain[1]._args[3].value == lens.data_ptr()
        # the window attention reads the ring with its lengths, window W
        wq, wk, wv, wo = _descs(win[0], rtp)
        assert wk.data == layer.k_ring.data_ptr() and list(wk.shape) == [B, Hkv - R, W, D]
        assert win[0]._args[3].value == layer.ring_lens.data_ptr() and win[0]._args[4].value == W
        assert wq.data == layer.q.data_ptr() + R * G * D * 2 and win[0]._args[-1].value == 22
    assert layer.cache_bytes() == 2 * B * R * N * D * 2 + B * R * N * 16 * 2 + 2 * B * (Hkv - R) * W * D * 2


def test_decode_selection_workspace_for_long_caches():
    # up to 16 x 32768 keys the decode cut lives on chip; past that the workspace holds the
    # scores each of a query's 16 CTAs cannot keep (4 bytes per key beyond 16 x 32768)
    rtp = _lib()
    assert rtp.topp_select_workspace_size(8, 32, 1, 8, 32768) == 0
    assert rtp.topp_select_workspace_size(1, 8, 1, 2, 524288) == 0
    assert rtp.topp_select_workspace_size(1, 8, 1, 2, 1 << 20) == 8 * 16 * (65536 - 32768) * 4
    assert rtp.topp_select_workspace_size(1, 8, 4096, 2, 1 << 20) == 0      # prefill
    L = rtp.lib()
    by = ctypes.byref
    qi = _desc(rtp, [1, 8, 1, 16])
    ki = _desc(rtp, [1, 2, 1 << 20, 16])
    s = _sel(rtp, words=(1 << 20) // 32)
    assert L.rtp_topp_select(by(qi), by(ki), None, 0.9, by(s), None, 0, None) == 5          # no workspace
    assert L.rtp_topk_select(by(qi), by(ki), None, 10, by(s), None, 0, None) == 5


def test_empty_tensors_may_have_a_null_base():
    # a zero among the first three dimensions: nothing is read or written, no launch
    rtp = _lib()
    L = rtp.lib()
    by = ctypes.byref
    x = _desc(rtp, [2, 4, 0, 128], data=0)
    xi = _desc(rtp, [2, 4, 0, 16], data=0)
    P = _desc(rtp, [4, 16, 128], dtype=0)
    assert L.rtp_index_project(by(x), by(P), by(xi), None) == 0
    assert L.rtp_index_project(by(_desc(rtp, [2, 4, 3, 128], data=0)), by(P), by(xi), None) == 1  # not empty

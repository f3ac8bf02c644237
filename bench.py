"""Benchmark of the RTPurbo decode path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one decode step of one attention layer for the whole batch:
project the newest key row and the queries (a1), score every cached key with
the 16-dim indexer and cut at top-p (a2+a3), attend the selected keys
(retrieval heads, a4) and the last W keys (local heads, a5).  All inputs are
seeded synthetic tensors resident in HBM before the timed region; the timed
region replays CUDA graphs of exactly K steps, bracketed by a barrier and a
device synchronisation, and the step time is the max over ranks.  Each rank
runs its own replica of the workload (weak scaling, no data-path collective).

``value`` is decode tokens/s (sequences advanced by one token per second,
summed over ranks).  ``e2e`` is the same metric through the public API with
host buffers (``DecodeLayer.host_step``): each step copies the new token's
q/k/v from pinned host memory, appends the new K/V rows (rtp_kv_append),
makes the other C-ABI calls and reads the output back, replayed as one CUDA
graph, with the host waiting for every token; the prefill object's ``e2e``
uses ``PrefillLayer.host_step``, whose copies run pipelined with the work on
two streams.  ``--impl reference`` times the CPU oracle on the same workload
instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_dim_b200 import workloads as wls  # noqa: E402

DECODE_WORKLOADS = {w.name: w for w in (wls.DECODE_B8_N32K, wls.DECODE_N4K_F32, wls.DECODE_B4_N128K)}
PREFILL_WORKLOADS = {w.name: w for w in (wls.PREFILL_N32K, wls.PREFILL_N8K, wls.PREFILL_CHUNK_1M)}
ALL_WORKLOADS = {**DECODE_WORKLOADS, **PREFILL_WORKLOADS}
DEFAULT_WORKLOAD = wls.DECODE_B8_N32K.name
EVENT_EVERY = 8  # decode: timing events around the sparse attention of one step in 8
METRIC = "decode sparse-attn tokens/s"
METRIC_PREFILL = "prefill queries/s"
ROW_BYTES = {"bf16": 2 * 128 * 2, "f32": 2 * 128 * 4}  # one K row + one V row
L2_BYTES = 126 * 2 ** 20
E2E_MIN_STEPS = 200  # end-to-end decode steps timed, whatever --steps is
PREFILL_STEPS = 10   # timed steps of the prefill object on the default decode line


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _tensor_peaks():
    """(burst, sustained) dense bf16 TFLOP/s, and where they come from."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return 0, 1, 0
    import torch.distributed as dist
    import datetime
    backend = os.environ.get("RTP_BENCH_BACKEND", "nccl")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist.get_rank(), ws, int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# reference arm: the CPU oracle
# --------------------------------------------------------------------------

class _OneThread:
    """The oracle evaluates one query at a time in NumPy; its BLAS calls are
    pinned to one thread so that the reported core count is the parallelism used."""

    def __enter__(self):
        from threadpoolctl import threadpool_limits
        self._lim = threadpool_limits(limits=1)
        return self

    def __exit__(self, *exc):
        self._lim.unregister()
        return False


ORACLE_CORES = 1


def oracle_step_runner(inst, wl):
    """Returns run(b) that computes every head of sequence b with the CPU oracle."""
    import oracle
    L = oracle.LayerOracle(inst.q, inst.k, inst.v, inst.P, inst.lens, R=wl.R, W=wl.W,
                           p=float(np.float32(wl.p)), storage=wl.dtype)
    for b in range(wl.B):            # the projected-key cache exists before decoding starts
        for kvh in range(wl.R):
            L.k_idx(b, kvh)

    def run(b):
        for h in range(wl.Hq):
            L.query(b, h, 0)
    return run


def cpu_baseline(inst, wl, budget_s=10.0):
    with _OneThread():
        return _cpu_baseline(inst, wl, budget_s)


def _cpu_baseline(inst, wl, budget_s):
    run = oracle_step_runner(inst, wl)
    t0 = time.perf_counter()
    done = 0
    while True:
        run(done % wl.B)
        done += 1
        if time.perf_counter() - t0 >= budget_s or done >= 4 * wl.B:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tokens/s", "cores": ORACLE_CORES, "kind": "oracle",
            "sample": f"{done} sequences x all {wl.Hq} heads of {wl.name} (one token each), "
                      f"projected-key cache prebuilt, {dt:.1f} s"}


REFERENCE_BUDGET_S = 120.0  # the oracle arm's whole warm-up + timed run, on the host's cores


def run_reference(args, wl, rank):
    """The oracle arm: the CPU oracle on this workload.  A step is a bounded
    sample of it -- a number of (sequence, head[, token]) queries sized so that
    warm-up plus timed steps take about REFERENCE_BUDGET_S -- and the rate is
    reported in the same unit as our arm (tokens or query tokens per second,
    a token counting all of its heads)."""
    if rank != 0:
        return 0
    with _OneThread():
        return _run_reference(args, wl)


def _run_reference(args, wl):
    import oracle
    inst = wls.generate(wl)
    L = oracle.LayerOracle(inst.q, inst.k, inst.v, inst.P, inst.lens, R=wl.R, W=wl.W,
                           p=float(np.float32(wl.p)), storage=wl.dtype)
    T = inst.q.shape[2]
    for b in range(wl.B):            # the projected-key cache exists before the step starts
        for kvh in range(wl.R):
            L.k_idx(b, kvh)
    rng = np.random.default_rng(12345)
    order = [(b, h) for b in range(wl.B) for h in range(wl.Hq)]
    cursor = [0]

    def one_query():
        b, h = order[cursor[0] % len(order)]
        cursor[0] += 1
        t = 0 if T == 1 else int(rng.integers(T))
        L.query(b, h, t)

    # calibrate the cost of one query (untimed), then size the step
    t0 = time.perf_counter()
    for _ in range(min(wl.Hq, 8)):
        one_query()
    per_query = (time.perf_counter() - t0) / min(wl.Hq, 8)
    per_step = REFERENCE_BUDGET_S / max(args.steps + args.warmup, 1)
    q_per_step = int(min(max(per_step / max(per_query, 1e-9), 1), wl.Hq))
    for _ in range(args.warmup):
        for _ in range(q_per_step):
            one_query()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(q_per_step):
            one_query()
    dt = time.perf_counter() - t0
    tokens = args.steps * q_per_step / wl.Hq
    v = tokens / dt
    decode = wl.mode != "prefill"
    metric, unit = (METRIC, "tokens/s") if decode else (METRIC_PREFILL, "queries/s")
    sample = (f"each step = {q_per_step} of the {wl.Hq} head queries of one "
              f"{'decode token' if decode else 'uniformly drawn query token'} of {wl.name} "
              f"(cycling over sequences and heads), projected-key cache prebuilt; a token counts all {wl.Hq} heads")
    config = {"workload": wl.name, "B": wl.B, "N": wl.N, "Hq": wl.Hq, "Hkv": wl.Hkv,
              "retrieval_kv_heads": wl.R, "W": wl.W, "p": wl.p}
    if not decode:
        config["T"] = T
    line = {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": v, "unit": unit, "cores": ORACLE_CORES, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

HOST_SIDE_MARKER = "// ---- host side"


def _traffic_record(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's device
    code (the source file up to its host-side section) is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        with open(os.path.join(ROOT, rec["source"]), encoding="utf-8") as f:
            text = f.read()
        if HOST_SIDE_MARKER in text:
            text = text[:text.index(HOST_SIDE_MARKER)]
        if hashlib.sha1(text.encode("utf-8")).hexdigest() != rec["device_code_sha1"]:
            return None
        return rec
    except Exception:
        return None


def run_ours(args, wl, rank, world, local_rank):
    import torch
    from long_context_sparse_dim_b200 import rtp  # noqa: F401  (fails loudly without librtp.so)
    from long_context_sparse_dim_b200.layer import DecodeLayer

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    inst = wls.generate(wl)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    q = torch.from_numpy(inst.q).to(dev, dt)
    k = torch.from_numpy(inst.k).to(dev, dt)
    v = torch.from_numpy(inst.v).to(dev, dt)
    P = torch.from_numpy(inst.P).to(dev, torch.float32)
    layer = DecodeLayer(q, k, v, P, R=wl.R, W=wl.W, p=wl.p)
    layer.build_index()
    torch.cuda.synchronize()

    # warm-up (also loads every kernel)
    for _ in range(max(args.warmup, 1)):
        layer.step()
    torch.cuda.synchronize()

    # graphs of the timed steps, events around the dominant kernel (sparse attention)
    chunk = 500
    graphs, ev = [], []
    s = torch.cuda.Stream(dev)
    side = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    remaining = args.steps
    with torch.cuda.stream(s):
        while remaining > 0:
            n = min(chunk, remaining)
            g = torch.cuda.CUDAGraph()
            # events around the sparse attention of every EVENT_EVERY-th step
            pairs = [tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(4))
                     if i % EVENT_EVERY == 0 else None for i in range(n)]
            with torch.cuda.graph(g, stream=s):
                for i in range(n):
                    _step_with_events(layer, pairs[i], side)
            graphs.append(g)
            ev.extend(pr for pr in pairs if pr is not None)
            remaining -= n
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    for g in graphs[:1]:
        g.replay()                     # graph upload / first-launch costs stay untimed
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.2)
    barrier(world, dev)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for g in graphs:
        g.replay()
    t_end.record()
    torch.cuda.synchronize()
    barrier(world, dev)
    clock_info = clocks.stop()
    step_ms_local = t_start.elapsed_time(t_end) / args.steps
    step_ms = max_over_ranks(step_ms_local, world, dev)
    # durations of the two attention launches (the window's overlaps the selection)
    attn_ms = statistics.mean(e3.elapsed_time(e1) for _, e1, _, e3 in ev)
    win_ms = statistics.mean(e0.elapsed_time(e2) for e0, _, e2, _ in ev)

    # realised selection: union of the GQA group's masks per (sequence, KV head)
    m = layer.sel.mask.view(torch.int32).cpu().numpy().view(np.uint32)
    G, R = wl.G, wl.R
    union_rows = 0
    sel_rows = 0
    for b in range(wl.B):
        for kh in range(R):
            rows = m[(b * R * G + kh * G):(b * R * G + (kh + 1) * G)]
            u = np.bitwise_or.reduce(rows, axis=0)
            union_rows += int(np.unpackbits(u.view(np.uint8)).sum())
            sel_rows += int(np.unpackbits(rows.view(np.uint8)).sum())
    row_b = ROW_BYTES[wl.dtype]
    attn_bytes = union_rows * row_b
    peak, peak_kind = _peaks()
    idx_bytes = wl.B * R * wl.N * 16 * (2 if wl.dtype == "bf16" else 4)
    win_rows = wl.B * (wl.Hkv - R) * min(wl.W, wl.N)
    win_bytes = win_rows * row_b
    step_bytes = idx_bytes + attn_bytes + win_bytes
    achieved = attn_bytes / (attn_ms * 1e-3) / 1e9
    tr = _traffic_record("attn_decode_bf16_kernel" if wl.dtype == "bf16" else "attn_decode_f32_kernel")

    # end to end through the public API with host buffers
    e2e = _e2e(layer, inst, wl, dev, max(args.steps, E2E_MIN_STEPS))
    dense = _dense_decode(layer, wl, dev, step_ms)
    budget = _budget_decode(layer, wl)
    cache = _cache_maintenance(inst, wl, dev, step_ms) if wl.Hkv > wl.R and wl.N > 4096 else None
    split = _key_range_split(dev) if wl.name == DEFAULT_WORKLOAD else None

    line = {
        "metric": METRIC, "value": world * wl.B / (step_ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "N": wl.N, "Hq": wl.Hq, "Hkv": wl.Hkv,
                   "retrieval_kv_heads": R, "W": wl.W, "p": wl.p,
                   "l2": f"inputs larger than L2: {step_bytes / 1e6:.0f} MB touched per step vs 126 MB L2, no flush",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "attn_decode_bf16_kernel" if wl.dtype == "bf16" else "attn_decode_f32_kernel",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": tr["dram_bytes_retrieval_launch"] if tr else None,
                     "launch": "retrieval heads: the union of each GQA group's selected rows",
                     "algorithmic_bytes": attn_bytes, "units": union_rows, "bytes_per_unit": row_b,
                     "ms_per_launch": attn_ms,
                     "local_heads_launch": {"algorithmic_bytes": win_bytes, "units": win_rows, "ms_per_launch": win_ms,
                                            "achieved": win_bytes / (win_ms * 1e-3) / 1e9,
                                            "note": "runs concurrently with the selection, sharing its SMs"}},
        "step_roofline": {"bytes": step_bytes, "achieved_gbs": step_bytes / (step_ms * 1e-3) / 1e9,
                          "frac": step_bytes / (step_ms * 1e-3) / 1e9 / peak},
        "selection": {"mean_selected_fraction": sel_rows / (wl.B * R * G * wl.N),
                      "mean_group_union_fraction": union_rows / (wl.B * R * wl.N)},
        "e2e": e2e,
        "dense_comparator": dense,
        "budget": budget,
        "cache_maintenance": cache,
        "key_range_split": split,
        "gpu_launches": 5 * args.steps,
        "streams": "window attention (local heads) forked onto a second stream after the projections",
        "timing_events": f"around both attention launches of every {EVENT_EVERY}th timed step",
        "clocks": clock_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inst, wl, args.cpu_budget)
    del graphs, layer, q, k, v
    torch.cuda.empty_cache()
    if not args.no_prefill and wl.name == DEFAULT_WORKLOAD:
        # the metric's second half: the 32768-token causal prefill of the same layer shape
        line["prefill"] = measure_prefill(args, wls.PREFILL_N32K, dev, world, PREFILL_STEPS, 3,
                                          rank == 0 and world == 1 and not args.no_cpu_baseline)
        line["gpu_launches"] += line["prefill"]["gpu_launches"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


PAGES_SPEEDUP = "the pages report up to 9.36x prefill at 1M context and ~2.01x decode over full attention " \
                "(hardware, precision and baseline not stated; context only)"


def _timed(fn, reps):
    import torch
    fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / reps


def _dense_decode(layer, wl, dev, step_ms, reps=200):
    """Our own dense comparator: every query head attends all n cached keys
    (rtp_window_attn with W = N over all heads), against the sparse step."""
    import torch
    from long_context_sparse_dim_b200 import rtp
    o = torch.empty(layer.q.shape, dtype=torch.float32, device=dev)
    ws = rtp.workspace(rtp.window_attn_workspace_size(wl.B, wl.Hq, 1, wl.Hkv, wl.N, wl.N), dev)
    ms = _timed(lambda: rtp.window_attn(layer.q, layer.k, layer.v, layer.lens, wl.N, layer.scale, o, ws), reps)
    return {"kernel": "rtp_window_attn with W = N over all query heads (full attention, same kernel as the "
                      "local heads)", "ms": ms, "sparse_step_ms": step_ms, "speedup": ms / step_ms,
            "bytes": wl.B * wl.Hkv * wl.N * ROW_BYTES[wl.dtype], "pages": PAGES_SPEEDUP}


def _budget_decode(layer, wl, reps=200):
    """Dynamic top-p against a fixed top-k budget of the same mean size: the
    spread of the per-query counts, and the cost of both selections."""
    import torch
    from long_context_sparse_dim_b200 import rtp
    cnt = layer.sel.count.cpu().numpy().astype(np.float64)
    k = max(int(round(cnt.mean())), 1)
    sel_k = rtp.Selection.empty(layer.sel.count.numel(), wl.N, layer.q.device)
    topp_ms = _timed(lambda: rtp.topp_select(layer.q_idx, layer.k_idx, layer.lens, layer.p, layer.sel,
                                             layer.ws_sel), reps)
    topk_ms = _timed(lambda: rtp.topk_select(layer.q_idx, layer.k_idx, layer.lens, k, sel_k, layer.ws_sel), reps)
    return {"topp_p": wl.p, "topp_count": {"min": int(cnt.min()), "mean": float(cnt.mean()),
                                            "max": int(cnt.max()), "std": float(cnt.std())},
            "topk_k": k, "topp_select_ms": topp_ms, "topk_select_ms": topk_ms,
            "queries": int(cnt.size)}


def _cache_maintenance(inst, wl, dev, resident_step_ms, reps=200):
    """Decode over caches the path keeps itself (CachedDecodeLayer): each step
    appends the new token (rtp_kv_append: full cache + projected key for the
    retrieval heads, a W-row ring for the local heads) before attending.
    Reports the cache memory against a full cache of every head, the chunk
    append of the prompt (HBM-bound copy + projection), the one-token append,
    and the whole appending step against the resident-cache step."""
    import torch
    from long_context_sparse_dim_b200 import rtp
    from long_context_sparse_dim_b200.layer import CachedDecodeLayer
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    es = 2 if wl.dtype == "bf16" else 4
    B, Hkv, R, N, W, D = wl.B, wl.Hkv, wl.R, wl.N, wl.W, 128
    L = Hkv - R
    k = torch.from_numpy(inst.k).to(dev, dt)
    v = torch.from_numpy(inst.v).to(dev, dt)
    P = torch.from_numpy(inst.P).to(dev, torch.float32)
    layer = CachedDecodeLayer(B, wl.Hq, Hkv, N, R, W, wl.p, P, dtype=dt, device=dev)
    T0 = N - 2 * reps - 16          # the prompt; the steps below append real rows up to N
    kc, vc = k[:, :, :T0], v[:, :, :T0]
    zeros = torch.zeros(B, dtype=torch.int32, device=dev)
    lens_o = torch.empty(B, dtype=torch.int32, device=dev)
    rl = torch.empty(B, dtype=torch.int32, device=dev)
    args = (kc, vc, zeros, R, P, layer.k_cache, layer.v_cache, layer.k_idx, layer.k_ring, layer.v_ring, lens_o, rl)
    chunk_ms = _timed(lambda: rtp.kv_append(*args), 10)
    chunk_bytes = (2 * B * Hkv * T0 * D * es             # read every new K and V row
                   + 2 * B * R * T0 * D * es + B * R * T0 * 16 * es   # full caches + projected keys
                   + 2 * B * L * min(T0, W) * D * es)    # the rings keep the last W
    peak, peak_kind = _peaks()
    layer.set_lengths(zeros)
    layer.append(kc, vc)
    q = torch.from_numpy(inst.q).to(dev, dt)
    layer.q.copy_(q)
    side = torch.cuda.Stream(dev)

    def feed(i):
        layer.k_new.copy_(k[:, :, T0 + i: T0 + i + 1])
        layer.v_new.copy_(v[:, :, T0 + i: T0 + i + 1])

    for i in range(4):                      # warm-up, marshals both plans
        feed(i)
        layer.step(side_stream=side)
    torch.cuda.synchronize()
    # one-token append alone (positions of the next step; idempotent rewrites)
    one = rtp.bind_kv_append(layer.k_new, layer.v_new, layer._lens[layer._cur], R, P, layer.k_cache, layer.v_cache,
                             layer.k_idx, layer.k_ring, layer.v_ring, lens_o, rl)
    append_ms = _timed(one, reps)
    # the whole appending step, graph-replayed like the resident step
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):           # even: the host's plan choice comes back to the start
                layer.step(side_stream=side)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    g.replay()                              # appends tokens T0+4 .. T0+4+reps-1 (upload untimed)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()                              # the next reps tokens, all below N
    b.record()
    b.synchronize()
    step_ms = a.elapsed_time(b) / reps
    ok = bool((layer.lens == T0 + 4 + 2 * reps).all().item())
    full_bytes = 2 * B * Hkv * N * D * es + B * R * N * 16 * es
    del g
    return {"layer": "CachedDecodeLayer (rtp_kv_append + the decode calls)",
            "cache_bytes": layer.cache_bytes(), "full_cache_bytes": full_bytes,
            "cache_fraction": layer.cache_bytes() / full_bytes,
            "prompt_append": {"tokens": T0, "ms": chunk_ms, "algorithmic_bytes": chunk_bytes,
                              "achieved_gbs": chunk_bytes / (chunk_ms * 1e-3) / 1e9,
                              "frac": chunk_bytes / (chunk_ms * 1e-3) / 1e9 / peak, "peak_kind": peak_kind},
            "one_token_append_ms": append_ms,
            "step_ms": step_ms, "resident_step_ms": resident_step_ms,
            "tokens_per_s": B / (step_ms * 1e-3), "lengths_advanced": ok}


def _key_range_split(dev, N=1 << 20, worlds=(1, 2, 4, 8), reps=50):
    """One sequence of 2^20 keys (the layer shape of the decode workloads, W =
    8192) decoded with its keys split by position over S ranks
    (KeyRangeDecodeLayer), each rank's share of a step emulated on this one GPU:
    the replicated query projection + top-p selection over all N keys, the
    range attention over N / S rows, its block of local heads and the merge of
    S partials.  The all-gather between the ranks (one row of 129 floats per
    query head and rank) is not part of the emulation.  Inputs are random
    device tensors; S = 1 is the unsplit step."""
    import math
    import torch
    from long_context_sparse_dim_b200 import rtp
    from long_context_sparse_dim_b200.split import key_ranges
    B, Hq, Hkv, R, W, D, p = 1, 32, 8, 2, 8192, 128, 0.95
    G, L = Hq // Hkv, Hkv - R
    Hr = R * G
    g = torch.Generator(device=dev).manual_seed(5)
    k = torch.randn(B, R, N, D, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(B, R, N, D, generator=g, device=dev).to(torch.bfloat16)
    q = torch.randn(B, Hq, 1, D, generator=g, device=dev).to(torch.bfloat16)
    kw = torch.randn(B, L, W, D, generator=g, device=dev).to(torch.bfloat16)
    vw = torch.randn(B, L, W, D, generator=g, device=dev).to(torch.bfloat16)
    P = torch.from_numpy(np.ascontiguousarray(np.broadcast_to(wls.lowfreq_projection(), (R, 16, D)))).to(dev)
    lens = torch.full((B,), N, dtype=torch.int32, device=dev)
    wl_ = torch.full((B,), W, dtype=torch.int32, device=dev)
    k_idx = torch.zeros(B, R, N, 16, dtype=torch.bfloat16, device=dev)
    rtp.index_project(k, P, k_idx)
    q_idx = torch.zeros(B, Hr, 1, 16, dtype=torch.bfloat16, device=dev)
    sel = rtp.Selection.empty(B * Hr, N, dev)
    scale = 1 / math.sqrt(D)

    ws_sel = rtp.workspace(rtp.topp_select_workspace_size(B, Hr, 1, R, N), dev)

    def select():
        rtp.index_project(q[:, :Hr], P, q_idx)
        rtp.topp_select(q_idx, k_idx, lens, p, sel, ws_sel)

    sel_ms = _timed(select, reps)
    out = {"N": N, "B": B, "W": W, "p": p, "selection_ms": sel_ms,
           "selected_fraction": float(sel.count.float().mean().item()) / N, "ranks": {}}
    for S in worlds:
        lo, rows = key_ranges(N, S)[0]
        l0, l1 = 0, -(-L // S)          # the busiest rank's block of local heads (ceil(L / S) of them)
        o = torch.zeros(B, Hq, 1, D, device=dev)
        lse = torch.zeros(B, Hq, device=dev)
        ws = rtp.workspace(rtp.sparse_attn_decode_workspace_size(B, Hr, R, rows), dev)
        kr, vr = k[:, :, lo:lo + rows], v[:, :, lo:lo + rows]
        wsw = rtp.workspace(rtp.window_attn_workspace_size(B, (l1 - l0) * G, 1, l1 - l0, W, W), dev)
        parts = torch.zeros(S, B, Hq, D, device=dev)
        lses = torch.zeros(S, B, Hq, device=dev)
        o_final = torch.zeros(B, Hq, 1, D, device=dev)

        def share():
            rtp.sparse_attn_decode_range(q[:, :Hr], kr, vr, lens, sel, lo, scale, o[:, :Hr], lse[:, :Hr], ws)
            if l1 > l0:
                rtp.window_attn(q[:, Hr + l0 * G: Hr + l1 * G], kw[:, l0:l1], vw[:, l0:l1], wl_, W, scale,
                                o[:, Hr + l0 * G: Hr + l1 * G], wsw)
            rtp.attn_combine(parts, lses, o_final)

        share_ms = _timed(share, reps)
        step_ms = sel_ms + share_ms
        out["ranks"][str(S)] = {"rows_per_rank": rows, "local_kv_heads_per_rank": l1 - l0,
                                "rank_step_ms": step_ms, "range_and_merge_ms": share_ms,
                                "tokens_per_s_projected": B / (step_ms * 1e-3)}
    out["note"] = ("per-rank shares emulated one at a time on one GPU; the all-gather of the partial rows "
                   "(129 floats per query head and rank) is not included: unmeasured on more than one GPU")
    del k, v, k_idx, kw, vw
    torch.cuda.empty_cache()
    return out


def _step_with_events(layer, ev, side):
    """One decode step (the sequence of DecodeLayer.step with a side stream:
    the window attention forked after the projections).  With ``ev`` =
    (e0, e1, e2, e3): e0/e2 around the window attention on the side stream,
    e3/e1 around the sparse attention on the main stream."""
    import torch
    from long_context_sparse_dim_b200 import rtp
    main = torch.cuda.current_stream()
    local = layer.Hkv > layer.R
    if layer.R:
        n = layer.N
        rtp.index_project(layer.k_ret[:, :, n - 1: n], layer.P, layer.k_idx[:, :, n - 1: n])
        rtp.index_project(layer.q_ret, layer.P, layer.q_idx)
    side.wait_stream(main)
    with torch.cuda.stream(side):
        if ev is not None:
            ev[0].record()
        if local:
            rtp.window_attn(layer.q_loc, layer.k_loc, layer.v_loc, layer.lens, layer.W, layer.scale, layer.o_loc,
                            layer.ws_loc)
        if ev is not None:
            ev[2].record()
    if layer.R:
        rtp.topp_select(layer.q_idx, layer.k_idx, layer.lens, layer.p, layer.sel, layer.ws_sel)
        if ev is not None:
            ev[3].record()
        rtp.sparse_attn_decode(layer.q_ret, layer.k_ret, layer.v_ret, layer.lens, layer.sel, layer.scale,
                               layer.o_ret, layer.ws_ret)
        if ev is not None:
            ev[1].record()
    main.wait_stream(side)


def _e2e(layer, inst, wl, dev, steps):
    import torch
    dt = layer.q.dtype
    n = wl.N
    h_q = torch.from_numpy(inst.q).to(dt).pin_memory()
    h_k = torch.from_numpy(np.ascontiguousarray(inst.k[:, :, n - 1: n])).to(dt).pin_memory()
    h_v = torch.from_numpy(np.ascontiguousarray(inst.v[:, :, n - 1: n])).to(dt).pin_memory()
    h_o = torch.empty(layer.o.shape, dtype=layer.o.dtype).pin_memory()
    h2d = h_q.numel() * h_q.element_size() + 2 * h_k.numel() * h_k.element_size()
    d2h = h_o.numel() * h_o.element_size()
    layer.host_step(h_q, h_k, h_v, h_o)      # captures the step's graph for these buffers (untimed)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        layer.host_step(h_q, h_k, h_v, h_o)  # copies in, the step, copy out, host waits for the output
    t1.record()
    t1.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return {"value": wl.B / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps}


# --------------------------------------------------------------------------
# prefill
# --------------------------------------------------------------------------

def _prefill_calls(layer, side):
    """The calls of one prefill step; returns (name, fn) pairs in launch order."""
    from long_context_sparse_dim_b200 import rtp
    L = layer
    calls = []
    if L.R:
        calls += [("index_project_k", lambda: rtp.index_project(L.k_ret, L.P, L.k_idx)),
                  ("index_project_q", lambda: rtp.index_project(L.q_ret, L.P, L.q_idx)),
                  ("topp_select", lambda: rtp.topp_select(L.q_idx, L.k_idx, L.lens, L.p, L.sel)),
                  ("sparse_attn_prefill", lambda: rtp.sparse_attn_prefill(
                      L.q_ret, L.k_ret, L.v_ret, L.q_idx, L.k_idx, L.lens, L.sel, L.scale, L.o_ret))]
    if L.Hkv > L.R:
        calls += [("window_attn", lambda: rtp.window_attn(L.q_loc, L.k_loc, L.v_loc, L.lens, L.W, L.scale,
                                                          L.o_loc, L.ws_loc))]
    return calls


def cpu_baseline_prefill(inst, wl, budget_s=10.0):
    with _OneThread():
        return _cpu_baseline_prefill(inst, wl, budget_s)


def _cpu_baseline_prefill(inst, wl, budget_s):
    import oracle
    L = oracle.LayerOracle(inst.q, inst.k, inst.v, inst.P, inst.lens, R=wl.R, W=wl.W,
                           p=float(np.float32(wl.p)), storage=wl.dtype)
    for kvh in range(wl.R):
        L.k_idx(0, kvh)
    rng = np.random.default_rng(0)
    t0 = time.perf_counter()
    done = 0
    while time.perf_counter() - t0 < budget_s:
        t = int(rng.integers(0, wl.T))
        for h in range(wl.Hq):
            L.query(0, h, t)
        done += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "queries/s", "cores": ORACLE_CORES, "kind": "oracle",
            "sample": f"{done} uniformly drawn query tokens x all {wl.Hq} heads of {wl.name}, "
                      f"projected-key cache prebuilt, {dt:.1f} s"}


def _needle_recall(layer, inst, wl):
    """Planted needles whose key is in their query's selected set, read from the
    selection's threshold form (score > tau, or == tau at a position <= tiepos);
    scores recomputed from the stored projected vectors in fp64 (a tie-band
    difference from the GPU's fp32 score can only move needles at the cut)."""
    if not inst.needles:
        return None
    import torch
    nd = np.array(inst.needles, dtype=np.int64)                 # (b, kv head, q head, t, key position)
    b, kvh, h, t, j = nd.T
    Hr = wl.R * wl.G
    qi = layer.q_idx[torch.from_numpy(b), torch.from_numpy(h), torch.from_numpy(t)].double().cpu().numpy()
    ki = layer.k_idx[torch.from_numpy(b), torch.from_numpy(kvh), torch.from_numpy(j)].double().cpu().numpy()
    s = (qi * ki).sum(axis=1) / 4.0
    rows = torch.from_numpy((b * Hr + h) * wl.T + t)
    tau = layer.sel.tau_bits[rows].cpu().numpy().view(np.float32).astype(np.float64)
    tp = layer.sel.tiepos[rows].cpu().numpy()
    hit = (s > tau) | ((s == tau) & (j <= tp))
    return {"recalled": int(hit.sum()), "needles": int(hit.size), "fraction": float(hit.mean())}


def measure_prefill(args, wl, dev, world, steps, warmup, with_cpu):
    """One prefill workload measured on this rank: the JSON fields of its line."""
    import torch
    from long_context_sparse_dim_b200 import rtp  # noqa: F401
    from long_context_sparse_dim_b200.layer import PrefillLayer

    inst = wls.generate(wl)
    q = torch.from_numpy(inst.q).to(dev, torch.bfloat16)
    k = torch.from_numpy(inst.k).to(dev, torch.bfloat16)
    v = torch.from_numpy(inst.v).to(dev, torch.bfloat16)
    P = torch.from_numpy(inst.P).to(dev, torch.float32)
    layer = PrefillLayer(q, k, v, P, R=wl.R, W=wl.W, p=wl.p)
    side = torch.cuda.Stream(dev)
    for _ in range(warmup):
        layer.step(side_stream=side)
    torch.cuda.synchronize()

    # per-kernel times, serialised on one stream (events on the launching stream)
    calls = _prefill_calls(layer, side)
    reps = max(1, min(steps, 3))
    times = {n: [] for n, _ in calls}
    for _ in range(reps):
        for n, fn in calls:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            times[n].append(a.elapsed_time(b))
    kernels_ms = {n: statistics.mean(v) for n, v in times.items()}

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.2)
    barrier(world, dev)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(steps):
        layer.step(side_stream=side)
    t_end.record()
    torch.cuda.synchronize()
    barrier(world, dev)
    clock_info = clocks.stop()
    assert rtp.poll_device_error() == 0, "a device wait timed out"
    step_ms = max_over_ranks(t_start.elapsed_time(t_end) / steps, world, dev)

    G, R = wl.G, wl.R
    T, N = wl.T, wl.N
    needle = _needle_recall(layer, inst, wl)
    counts = layer.sel.count.cpu().numpy().astype(np.int64)
    admitted = int(counts.sum())                       # (query, key) pairs the sparse attention runs
    pos = np.arange(T) + N - T
    causal = int((pos + 1).sum()) * R * G              # indexer (query, key) pairs
    win = int(np.minimum(pos + 1, wl.W).sum()) * (wl.Hq - R * G)
    burst, sustained, pk = _tensor_peaks()
    attn_flop = 4.0 * 128 * admitted                   # QK^T + PV, 2 FLOP per MAC
    win_flop = 4.0 * 128 * win
    gemm_flop = 2.0 * 16 * causal                      # one pass of the depth-16 score GEMM
    flop = {"sparse_attn_prefill": attn_flop, "window_attn": win_flop, "topp_select": gemm_flop}
    dom = max((n for n in flop if n in kernels_ms), key=lambda n: kernels_ms[n])
    dom_ach = flop[dom] / (kernels_ms[dom] * 1e-3) / 1e12
    out = {
        "metric": METRIC_PREFILL, "value": world * wl.B * T / (step_ms * 1e-3), "unit": "queries/s",
        "ms_per_step": step_ms, "steps": steps, "warmup": warmup, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "T": T, "N": N, "Hq": wl.Hq, "Hkv": wl.Hkv,
                   "retrieval_kv_heads": R, "W": wl.W, "p": wl.p,
                   "l2": "inputs larger than L2 (K/V cache and score sweeps), no flush",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": dom_ach, "peak": sustained,
                     "unit": "TFLOP/s", "frac": dom_ach / sustained, "peak_kind": pk + " sustained",
                     "traffic": None, "algorithmic_flop": flop[dom], "ms_per_launch": kernels_ms[dom],
                     "flop_per_unit": {"sparse_attn_prefill": "512 per admitted (query, key) pair",
                                       "window_attn": "512 per (query, key) pair in the band",
                                       "topp_select": "32 per causal (query, key) pair, one pass of the "
                                                      "score GEMM"}[dom]},
        "score_gemm": {"kernel": "topp_select", "algorithmic_flop_one_pass": gemm_flop,
                       "causal_pairs": causal,
                       "achieved_tflops_one_pass": gemm_flop / (kernels_ms["topp_select"] * 1e-3) / 1e12,
                       "frac_of_burst": gemm_flop / (kernels_ms["topp_select"] * 1e-3) / 1e12 / burst,
                       "pairs_per_s": causal / (kernels_ms["topp_select"] * 1e-3)},
        "kernels_ms": kernels_ms,
        "kernels_tflops": {n: flop[n] / (kernels_ms[n] * 1e-3) / 1e12 for n in flop if n in kernels_ms},
        "selection": {"mean_selected_fraction": admitted / max(causal, 1), "needle_recall": needle},
        "gpu_launches": len(calls) * steps,
        "streams": "window attention (local heads) forked onto a second stream inside each step",
        "clocks": clock_info,
    }
    # our own dense comparator: causal full attention of every query head (W = N)
    o_dense = torch.empty(layer.o.shape, dtype=layer.o.dtype, device=dev)
    dense_ms = _timed(lambda: rtp.window_attn(layer.q, layer.k, layer.v, layer.lens, N, layer.scale, o_dense,
                                              None), max(1, min(steps, 3)))
    out["dense_comparator"] = {"kernel": "rtp_window_attn with W = N over all query heads (causal full "
                                         "attention, same tcgen05 kernel as the local heads)",
                               "ms": dense_ms, "sparse_step_ms": step_ms, "speedup": dense_ms / step_ms,
                               "flop": 4.0 * 128 * int((pos + 1).sum()) * wl.Hq,
                               "pages": PAGES_SPEEDUP}
    del o_dense
    out["e2e"] = _e2e_prefill(layer, inst, max(1, min(steps, 3)))
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline_prefill(inst, wl, args.cpu_budget)
    del layer, q, k, v
    torch.cuda.empty_cache()
    return out


def run_prefill(args, wl, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    m = measure_prefill(args, wl, dev, world, args.steps, args.warmup,
                        rank == 0 and world == 1 and not args.no_cpu_baseline)
    line = {"metric": m.pop("metric"), "value": m.pop("value"), "unit": m.pop("unit"), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": m.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None}
    m.pop("steps")
    m.pop("warmup")
    line.update(m)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def _e2e_prefill(layer, inst, steps):
    import torch
    h_q = torch.from_numpy(inst.q).to(torch.bfloat16).pin_memory()
    h_k = torch.from_numpy(inst.k).to(torch.bfloat16).pin_memory()
    h_v = torch.from_numpy(inst.v).to(torch.bfloat16).pin_memory()
    h_o = torch.empty(layer.o.shape, dtype=layer.o.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (h_q, h_k, h_v))
    d2h = h_o.numel() * h_o.element_size()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    layer.host_step(h_q, h_k, h_v, h_o)  # untimed: first use of the host streams
    torch.cuda.synchronize()
    t0.record()
    for _ in range(steps):
        layer.host_step(h_q, h_k, h_v, h_o)  # copies in, the step, copy out (pipelined), host waits
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return {"value": inst.wl.B * inst.wl.T / (ms * 1e-3), "unit": "queries/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(ALL_WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="leave the prefill object out of the decode line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    wl = ALL_WORKLOADS[args.workload]
    rank, world, local_rank = _dist()
    try:
        if args.impl == "reference":
            return run_reference(args, wl, rank)
        if wl.mode == "prefill":
            return run_prefill(args, wl, rank, world, local_rank)
        return run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

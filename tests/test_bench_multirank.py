"""bench.py's multi-rank harness on CPU: two ranks over gloo.

The helpers the timed region relies on (process-group set-up from the
launcher's environment, barrier, max over ranks) and the oracle arm launched
the way the multi-GPU run launches it (torch.distributed.run, one process per
rank; rank 0 alone measures and prints one JSON line, the others exit 0).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _helpers_rank(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank), "RTP_BENCH_BACKEND": "gloo"})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, ws, lr = bench._dist()
    try:
        bench.barrier(ws)
        mx = bench.max_over_ranks(float(10 * (r + 1)), ws)
        bench.barrier(ws)
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"rank": r, "world": ws, "local_rank": lr, "max": mx}, f)
    finally:
        dist.destroy_process_group()


def test_dist_helpers_two_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_helpers_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [g["rank"] for g in got] == [0, 1]
    assert all(g["world"] == world for g in got)
    assert all(g["local_rank"] == g["rank"] for g in got)
    assert all(g["max"] == 10.0 * world for g in got)  # the max over ranks, on every rank


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    env = dict(os.environ, RTP_BENCH_BACKEND="gloo", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "3", "--workload", "decode_b1_n4096_f32_1ret1loc"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1

"""The multi-process path of bench.py on CPU: world size 2 over gloo.

* the plumbing each rank runs around the timed region — barrier, maximum of
  the per-rank times over the ranks, whole-job weak-scaling throughput;
* the reference arm launched as a multi-GPU run is launched
  (torch.distributed.run, 2 processes, 127.0.0.1): rank 0 alone runs and
  prints one JSON line, the other rank exits 0 without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    my_ms = 10.0 + 5.0 * r                       # rank 1 is the slow one
    mx = bench.allmax(w, my_ms)
    value = bench.weak_scaling_value(w, 1000, mx)
    bench.barrier(w)
    dist.destroy_process_group()
    out_q.put((r, w, mx, value))


def test_allmax_barrier_and_value_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, mx, value in res:
        assert w == 2
        assert mx == 15.0                          # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 1000 / 0.015)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                          # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"

"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The hot path shards by independent (batch, head) slices with no data-path collective; the
benchmark's only cross-rank steps are the barrier around the timed region and the max over
ranks of the measured time.  These run here as two gloo processes.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    assert torch.distributed.get_backend() == "gloo"
    bench.barrier(w)
    # every rank times its own shard; the job's time is the slowest rank's
    t = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    results[rank] = t
    torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    mgr = mp.Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(2, port, results), nprocs=2, join=True, start_method="spawn")
    assert results[0] == results[1] == 15.0


def test_reference_arm_prints_one_line_on_rank0_only():
    # the oracle arm of bench.py: rank 0 runs it and prints one JSON line; other ranks exit 0
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
           "tiny_fp32", "--steps", "1"]
    r1 = subprocess.run(cmd, env=dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1"),
                        capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"),
                        capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr
    lines = [l for l in r0.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0

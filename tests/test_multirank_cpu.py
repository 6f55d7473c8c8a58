"""The N > 1 path of bench.py on the CPU: two ranks over gloo.

The method's chunks are independent, so ranks share no data: each draws its
own batch (shard_seed) and the only collectives are the timing barrier and the
max-over-ranks all-reduce.  These tests run that host logic in two real
processes (rendezvous on 127.0.0.1) and the reference arm under torchrun,
where rank 0 alone works and prints.
"""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def cpu_env(**extra):
    env = dict(os.environ)
    env.update({"CUDA_VISIBLE_DEVICES": "", "MASTER_ADDR": "127.0.0.1",
                "PYTHONPATH": ROOT + os.pathsep + env.get("PYTHONPATH", "")})
    env.update({k: str(v) for k, v in extra.items()})
    return env


WORKER = textwrap.dedent("""
    import json, os, sys
    import torch
    import bench
    world, rank, local = bench.dist_setup()
    assert world == 2
    import torch.distributed as dist
    assert dist.get_backend() == "gloo"
    bench.barrier(world)
    # the time that counts is the slowest rank's
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
    out = {"rank": rank, "ms": ms,
           "seeds": [bench.shard_seed(rank, r) for r in range(3)],
           "value": bench.aggregate_throughput(4096, world, ms, 10)}
    bench.barrier(world)
    dist.destroy_process_group()
    print("RESULT " + json.dumps(out), flush=True)
""")


def test_two_rank_timing_collectives_gloo():
    port = free_port()
    procs = [subprocess.Popen([sys.executable, "-c", WORKER], cwd=ROOT,
                              env=cpu_env(RANK=r, LOCAL_RANK=r, WORLD_SIZE=2, MASTER_PORT=port),
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for r in range(2)]
    results = {}
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        line = [l for l in out.splitlines() if l.startswith("RESULT ")][-1]
        d = json.loads(line[len("RESULT "):])
        results[d["rank"]] = d
    assert set(results) == {0, 1}
    # max over ranks, identical on both
    assert results[0]["ms"] == results[1]["ms"] == 15.0
    # each rank its own batch: no seed shared between ranks
    assert not set(results[0]["seeds"]) & set(results[1]["seeds"])
    # whole-job throughput: both ranks' chunks over the slowest rank's time per step
    assert results[0]["value"] == pytest.approx(2 * 4096 / (15.0e-3 / 10))


def test_reference_arm_under_torchrun_two_ranks():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--sample-chunks", "4"]
    r = subprocess.run(cmd, cwd=ROOT, env=cpu_env(), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                                  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["unit"] == "chunks/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_bounds_its_work():
    """However many steps are asked for, the reference arm's windows shrink so
    that warm-up and timed steps together stay within its chunk budget."""
    import bench

    for steps in (1, 10, 100, 500, 5000, 100000):
        n = bench.reference_window(steps, 5, 512)
        assert 1 <= n <= 512
        assert n * (steps + 5) <= max(bench.REFERENCE_CHUNK_BUDGET, steps + 5)
    assert bench.reference_window(1, 3, 512) == 512
    # the windows wrap around the workload's chunks
    w = dict(bench.WORKLOAD)
    data = bench.OracleInputs(w)
    K, V, b, g = data.window(data.nc - 2, 5)
    assert K.shape[0] == 5 and (K[2] == data.K[0]).all() and (g[4] == data.g[2]).all()

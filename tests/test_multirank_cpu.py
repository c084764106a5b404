"""The benchmark's multi-process path, on the CPU with gloo and two ranks.

The hot path shards by independent sequences, so the only cross-rank steps are the
timing plumbing: a barrier around the timed region, the max of the per-rank times and
the sum of the per-rank token counts.  These run here exactly as they do under
torchrun on GPUs, with the gloo backend; and the oracle ("reference") arm is checked to
run on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, l = bench.dist_env()
    assert (w, r, l) == (world, rank, rank)
    dist = bench.init_dist(w, l, backend="gloo")
    dev = torch.device("cpu")
    bench.barrier(dist, dev)
    t_max = bench.max_over_ranks(dist, 1.5 + rank, dev)       # per-rank "ms"
    n_sum = bench.sum_over_ranks(dist, 1000.0 * (rank + 1), dev)
    bench.barrier(dist, dev)
    out.put((rank, t_max, n_sum))
    dist.destroy_process_group()


def test_timing_reductions_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t_max, n_sum in res:
        assert t_max == 2.5          # max over ranks of 1.5 + rank
        assert n_sum == 3000.0       # all ranks' units


def test_reference_arm_runs_on_rank_zero_only(tmp_path):
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                        timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r0 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--steps", "1", "--warmup", "3", "--workload", "elu1_f32_small"],
                        env=env, capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0

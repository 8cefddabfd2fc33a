"""The benchmark's multi-rank plumbing on the CPU: world size 2 over gloo.

The path shards into independent (sequence, kv head) units with no exchange,
so ranks meet only for the barrier around the timed region and the max over
ranks of the timings; the reference arm runs on rank 0 alone."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    got_world, got_rank, _ = bench.dist_setup()
    try:
        assert (got_world, got_rank) == (world, rank)
        bench.barrier(world)
        out[rank] = bench.max_over_ranks(values[rank], world)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    world = 2
    values = [3.25, 7.5]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), values, out), nprocs=world, join=True)
        assert dict(out) == {0: 7.5, 1: 7.5}


def test_ranks_draw_distinct_inputs():
    from bit_kv_cache_tq_b200 import inputs
    seeds = [bench.rank_seed(r) for r in range(8)]
    assert len(set(seeds)) == 8
    a = inputs.queries(1, 4, 128, seeds[0])
    b = inputs.queries(1, 4, 128, seeds[1])
    assert not torch.equal(a, b)


def test_reference_arm_prints_once_under_torchrun():
    """`--impl reference` under torchrun with two ranks: rank 0 prints one
    JSON line, rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", "--master-port=%d" % _free_port(), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"

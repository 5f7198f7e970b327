"""Multi-rank host logic of bench.py, run as two gloo ranks on the CPU.

The forward shards into independent (batch, head) recurrences, so N GPUs run
N replicas with no collective on the data path; the only cross-rank steps are
the barrier around the timed region and the max-over-ranks of the step time.
These tests check those steps, the per-rank input shards and the reference
arm's rank-0-only rule without a GPU.
"""
import io
import json
import os
import socket
from contextlib import redirect_stdout
from types import SimpleNamespace

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from gated_delta_rule_wy_b200 import inputs as I


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    w, r, _ = bench.dist_env()
    assert (w, r) == (world, rank)
    bench.init_dist(w, "gloo")
    try:
        dev = torch.device("cpu")
        bench.barrier(w)
        # rank r took 10 (r + 1) ms over 5 steps: the job is as slow as the slowest rank
        value, ms_per_step = bench.job_throughput(10.0 * (rank + 1), 5, 1000, w, dev)
        # each rank draws its own shard of independent recurrences
        cfg = dict(B=1, H=2, T=8, dk=4, dv=4, seed=bench.shard_seed(3, rank))
        x = I.make_forward_inputs(**cfg)
        shard = torch.cat([x.q.flatten(), x.k.flatten(), x.v.flatten()])
        shards = [torch.empty_like(shard) for _ in range(w)]
        dist.all_gather(shards, shard)
        distinct = not torch.equal(shards[0], shards[1])
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"value": value, "ms_per_step": ms_per_step, "distinct": distinct}, f)
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r in res:
        # slowest rank: 20 ms / 5 steps = 4 ms per step; 2 ranks x 1000 units per step
        assert r["ms_per_step"] == pytest.approx(4.0)
        assert r["value"] == pytest.approx(2 * 1000 / 4e-3)
        assert r["distinct"]


def test_single_rank_needs_no_process_group():
    value, ms = bench.job_throughput(12.0, 4, 300, 1, torch.device("cpu"))
    assert ms == pytest.approx(3.0) and value == pytest.approx(1e5)
    assert not dist.is_initialized()


def test_shard_seeds_are_distinct():
    seeds = {bench.shard_seed(11, r) for r in range(8)}
    assert len(seeds) == 8


def test_reference_arm_prints_on_rank_zero_only():
    args = SimpleNamespace(gpus=2, steps=1, warmup=3)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, world=2, rank=1)
    assert buf.getvalue() == ""

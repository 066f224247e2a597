"""The multi-rank (N > 1) host logic of bench.py, on CPU with two gloo ranks.

Under torchrun every rank times its own independent problem, and rank 0
reports the whole job: the slowest rank's time and the units of all ranks.
These tests run that logic on two CPU processes (gloo, 127.0.0.1): the max
over ranks, the whole-job rate, distinct per-rank inputs, the order of the
collectives, and the reference arm's rank-0-only rule.
"""
import datetime
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # the slowest rank's time, seen by every rank
        local_ms = [10.0, 12.5][rank]
        res["max_ms"] = bench.max_over_ranks(local_ms, WORLD, device="cpu")
        # stage times reduced in one order on every rank (same keys, same order)
        stages = {"select": 0.5 + rank, "attn": 3.0 - rank}
        res["stages"] = {k: bench.max_over_ranks(v, WORLD, device="cpu") for k, v in stages.items()}
        # each rank draws its own problem
        wl = WORKLOADS["tiny"].with_(seqlen_q=64, seqlen_kv=64)
        x = make_inputs(wl, device="cpu", seed=bench.rank_seed(rank))
        digest = float(x["q"].float().sum())
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, digest)
        res["digests"] = gathered
        bench.barrier(WORLD)
        torch.save(res, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_draw_distinct_inputs(tmp_path):
    mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(WORLD)]
    for r in res:
        assert r["max_ms"] == 12.5
        assert r["stages"] == {"select": 1.5, "attn": 3.0}
        assert r["digests"] == res[0]["digests"]
    a, b = res[0]["digests"]
    assert a != b, "the two ranks drew the same inputs"


def test_job_rate_is_all_units_over_the_slowest_rank():
    # 2 ranks x 1e12 FLOP each in 12.5 ms (the slower rank) = 160 TFLOP/s
    assert bench.job_rate(1e12, 2, 12.5) == pytest.approx(1.6e14)
    assert bench.job_rate(1e12, 1, 12.5) == pytest.approx(8e13)
    assert bench.rank_seed(0) != bench.rank_seed(1)
    assert bench.rank_seed(0, decode=True) != bench.rank_seed(0)


def test_single_rank_reduction_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"workload": "tiny", "steps": 1, "warmup": 0})()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""

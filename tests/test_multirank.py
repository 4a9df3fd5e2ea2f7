"""The multi-rank bench path on the host: world_size-2 gloo process groups on CPU.

`bench.py --gpus N` runs one independent replica of the workload per rank (units are
independent, so there is no collective on the data path) and reports the slowest rank's time.
These tests cover that host logic without a GPU: the max-over-ranks reduction, the per-rank
workload replicas, the whole-job throughput, and the reference arm's rank-0-only rule.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import kda_workloads as W  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_path):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        got = bench._max_over_ranks(times[rank], dist, torch.device("cpu"))
        # the replica of this rank: same shapes, distinct seed
        w = bench.rank_workload(2, rank, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, w.seed)
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(f"{got!r} {seeds[0]} {seeds[1]}\n")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_seeds_gloo(tmp_path):
    world, port = 2, _free_port()
    times = [3.25, 7.5]
    out = str(tmp_path / "r")
    mp.spawn(_worker, args=(world, port, times, out), nprocs=world, join=True)
    for r in range(world):
        got, s0, s1 = open(f"{out}.{r}").read().split()
        assert float(got) == max(times)  # every rank reports the slowest rank's time
        assert int(s0) != int(s1)        # ranks run distinct replicas


def test_single_rank_needs_no_process_group():
    assert bench._max_over_ranks(4.0, None, None) == 4.0


def test_rank_workload_replicas_share_shapes():
    base = W.workload(5)
    for rank in range(4):
        w = bench.rank_workload(5, rank, 4)
        assert (w.layout, w.B, w.Nqk, w.Nv, w.S, w.lengths) == (base.layout, base.B, base.Nqk,
                                                                base.Nv, base.S, base.lengths)
        assert w.seed == base.seed + 1000 * rank
    assert bench.rank_workload(5, 0, 1).seed == base.seed


def test_replica_inputs_differ_by_rank():
    a = W.generate(bench.rank_workload(1, 0, 2))
    b = W.generate(bench.rank_workload(1, 1, 2))
    assert a["q"].shape == b["q"].shape
    assert not np.array_equal(a["q"], b["q"])


def test_job_throughput_is_weak_scaling_aggregate():
    th = W.workload(5).token_heads
    one = bench.job_throughput(th, 1, 20, 70.0)
    eight = bench.job_throughput(th, 8, 20, 70.0)
    assert eight == pytest.approx(8 * one)
    assert one == pytest.approx(th * 20 / 0.070)


def test_config_names_the_replicas():
    w = W.workload(5)
    assert bench._config(w, 1)["parallelism"] == "single GPU"
    assert "4 replicas" in bench._config(w, 4)["parallelism"]


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""

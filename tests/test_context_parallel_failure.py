"""Failure detection in the context-parallel schedule, on the host (gloo ranks on CPU, no GPU).

One rank of three fails before the exchange: its summary raises, as a failed library call would
(the rank then exits), or it stalls for longer than the process group's timeout before raising.
The other ranks must not hang in the all-gather: they get an error from
``flash_kda_context_parallel`` within a bounded time (at once when the peer's connection closes,
after the group's 5 s timeout when the peer stalls), and the failing rank's own exception
reaches its caller unchanged.
"""
import datetime
import os
import sys
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import chunked_kda_prefill_b200 as kda  # noqa: E402
from test_context_parallel_host import S_LOC, OracleOps, _free_port, _span, _workload  # noqa: E402
import kda_workloads as W  # noqa: E402

STALL_S = 20


class FailingSummary(OracleOps):
    stall = False

    @classmethod
    def summary(cls, *args, **kwargs):
        if cls.stall:
            time.sleep(STALL_S)
        raise RuntimeError("summary failed on this rank")


def _worker(rank, world, port, path, stall):
    outcome = "ok"
    t0 = time.time()
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=5))
        w = _workload(world, "BNSD")
        inp = W.generate(w)
        sp = _span(inp, "BNSD", rank)
        t = {n: torch.from_numpy(a.view(np.int16)) for n, a in sp.items()}
        shape = kda.KdaShape(kda.LAYOUTS["BNSD"], w.B, w.Nqk, w.Nv, S_LOC, w.D)
        plan = kda.make_plan(shape, "BNSD")
        FailingSummary.stall = stall
        ops = FailingSummary if rank == 1 else OracleOps
        ops.layout, ops.Nqk, ops.calls = "BNSD", w.Nqk, []
        kda.flash_kda_context_parallel(
            t["q"], t["k"], t["v"], t["g"], t["beta"], w.scale,
            torch.from_numpy(inp["initial_state"]), torch.from_numpy(inp["A_log"]),
            torch.from_numpy(inp["dt_bias"]), w.lower_bound, "BNSD", plan, ops=ops)
    except Exception as e:  # noqa: BLE001 - the outcome is the test's subject
        outcome = f"error: {type(e).__name__}: {e}"
    with open(f"{path}.{rank}", "w") as f:
        f.write(f"{time.time() - t0:.1f}\n{outcome}\n")
    # no destroy_process_group: the group may be broken; the process exits


@pytest.mark.parametrize("stall", [False, True], ids=["raises", "stalls"])
def test_a_failing_rank_does_not_hang_the_others(stall, tmp_path):
    world, path = 3, str(tmp_path / "fail")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, path, stall))
             for r in range(world)]
    for p in procs:
        p.start()
    deadline = time.time() + 120
    for p in procs:
        p.join(max(1.0, deadline - time.time()))
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung in the exchange"
    results = {}
    for r in range(world):
        secs, outcome = open(f"{path}.{r}").read().split("\n", 1)
        results[r] = (float(secs), outcome.strip())
    assert results[1][1].startswith("error: RuntimeError: summary failed"), results
    for r in (0, 2):  # both wait on the exchange that rank 1 never joins
        assert results[r][1].startswith("error:"), results
        # a stalled peer is detected by the group timeout, before the peer itself gives up
        assert results[r][0] < (STALL_S if stall else 60), results

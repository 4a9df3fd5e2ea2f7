#!/usr/bin/env python
"""Throughput of chunked KDA prefill on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 5]

A step is one kda_forward over the large prefill (B=4, Nqk=Nv=32, S=16384, D=128, BNSD; seeded
synthetic bf16 inputs ~ N(0,1)).  Units (sequence, value head) are independent, so N > 1 runs one
replica of the workload per GPU with no collective on the data path (weak scaling); torchrun
supplies RANK / LOCAL_RANK / WORLD_SIZE.  ``--impl reference`` times the fp64 CPU oracle on a
bounded sample of the same workload (rank 0 only).  ``--mode decode`` times the single-token
decode step, ``--mode cp`` context parallelism (one sequence split over the ranks; with one
process ``--cp-emulate E`` runs E ranks' work one after another).
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_workloads as W  # noqa: E402

METRIC = "KDA prefill tokens/s per B200 (B·Nv·S/s) and % of tensor/HBM roofline"
UNIT = "token-heads/s"
FALLBACK_HBM_GBS = 6650.0


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML)
# ----------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period, self.ok = period_s, False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks rather than guess
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in _REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# roofline bookkeeping
# ----------------------------------------------------------------------------

def algorithmic_bytes(w: W.Workload, with_initial_state: bool) -> int:
    """Unique HBM bytes of one forward: q, k (per qk head), v, g and beta of the valid rows
    (rows past a valid length are never read), out over every storage row (those rows are written
    as zeros), the initial and final states, A_log and dt_bias."""
    valid = sum(w.lengths)
    stored = w.S if w.layout == "TND" else w.B * w.S
    qk = 2 * valid * w.Nqk * w.D * 2
    vg = 2 * valid * w.Nv * w.D * 2
    beta = valid * w.Nv * 2
    out = stored * w.Nv * w.D * 2
    states = (2 if with_initial_state else 1) * w.B * w.Nv * w.D * w.D * 4
    params = w.Nv * 4 + w.Nv * w.D * 4
    return qk + vg + beta + out + states + params


def algorithmic_flops(w: W.Workload) -> float:
    """Dense matrix-product flops of the chunked method: per chunk-head (C = 64) five 64x64xD
    products (K K^T, Q K^T, W, U, Aqk Delta) and three 64xDxD ones (W S^T, Q~ S^T, Delta^T K^):
    11.53 MFLOP at D = 128.  The triangular solve (about 0.09 MFLOP, CUDA cores) is not counted."""
    per_chunk = 5 * 2 * 64 * 64 * w.D + 3 * 2 * 64 * w.D * w.D
    chunks = sum(math.ceil(L / 64) for L in w.lengths) * w.Nv
    return float(per_chunk * chunks)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def schedule_name(plan, w: W.Workload, one_cta: str = "") -> str:
    """How the forward runs the workload: segments (the chunk-parallel scan), or whole units,
    claimed dynamically, longest first, when their lengths differ (the library's rule)."""
    if plan.segment_chunks > 0:
        return f"segments of {plan.segment_chunks} chunks"
    if len(set(int(L) for L in w.lengths)) > 1:
        return "whole units, claimed longest first by the CTA that frees up first"
    return "whole units" + one_cta


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "chunked_kda_prefill_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernels."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload_name}.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("kernel_source_sha") == kernel_source_hash():
            return float(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ----------------------------------------------------------------------------

def cpu_oracle_sample(w: W.Workload, inp: dict, budget_s: float = 10.0, tokens: int | None = None,
                      form: str = "recurrent"):
    """Time the fp64 oracle (``form``: the recurrence, or the chunked form) on batches of whole
    units until ``budget_s`` elapses.

    One batch is one unit per host thread.  ``tokens`` keeps only the first ``tokens`` rows of
    every sequence (BNSD/BSND), a bounded sample with the same per-token work.
    """
    import oracle
    cores = len(os.sched_getaffinity(0))
    it, lengths, S = inp, list(w.lengths), w.S
    if tokens is not None and w.layout != "TND" and tokens < w.S:
        it = dict(inp)
        for n in ("q", "k", "v", "g", "beta"):
            it[n] = inp[n][:, :, :tokens] if w.layout == "BNSD" else inp[n][:, :tokens]
        lengths, S = [min(L, tokens) for L in w.lengths], tokens
    cu = np.concatenate([[0], np.cumsum(lengths)]) if w.layout != "TND" else w.cu_seqlens
    units = [(b, h) for b in range(w.B) for h in range(w.Nv)]
    oracle.lib()
    done_tokens, n_units, i = 0, 0, 0
    t0 = time.perf_counter()
    while i < len(units):
        batch = units[i:i + cores]
        i += cores
        oracle.run_units(it, w.layout, w.B, w.Nqk, w.Nv, S, w.D, w.scale, w.lower_bound, cu,
                         units=batch, form=form, threads=cores)
        done_tokens += sum(lengths[b] for b, _ in batch)
        n_units += len(batch)
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done_tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n_units} whole (sequence, value head) units of {w.name}"
                      + ("" if tokens is None else f", first {tokens} tokens each")
                      + (", fp64 recurrence" if form == "recurrent" else ", fp64 chunked form")
                      + f", {dt:.1f} s wall on {cores} threads"}, dt


# ----------------------------------------------------------------------------
# runs
# ----------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = W.workload(args.workload)
    inp = W.generate(w)
    cores = len(os.sched_getaffinity(0))
    tokens = args.ref_tokens
    for _ in range(args.warmup):
        cpu_oracle_sample(w, inp, budget_s=0.0, tokens=min(tokens, 256))
    times, tok = [], 0
    for _ in range(args.steps):
        r, dt = cpu_oracle_sample(w, inp, budget_s=0.0, tokens=tokens)
        times.append(dt)
        tok += r["value"] * dt
    total = sum(times)
    value = tok / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"each step: the first {tokens} tokens of {min(cores, w.units)}"
                                       f" (sequence, value head) units of {w.name}, fp64 "
                                       "recurrence, one unit per host thread"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _config(w: W.Workload, world: int):
    c = w.describe()
    c["parallelism"] = ("single GPU" if world == 1 else
                        f"{world} replicas, one independent copy of the workload per GPU")
    rows = w.S if w.layout == "TND" else w.B * w.S
    in_bytes = 5 * rows * w.Nv * w.D * 2
    c["l2"] = (f"inputs ({in_bytes / 1e9:.2f} GB) larger than L2 (126 MB); no flush"
               if in_bytes > 126e6 else "L2 flushed between steps by a 256 MB write")
    if os.environ.get("KDA_LIB"):  # a variant build of the library (build --define ...)
        c["library"] = os.path.basename(os.environ["KDA_LIB"])
    return c


def run_ours(args, rank, world):
    import torch
    import chunked_kda_prefill_b200 as kda

    local = _env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    w = rank_workload(args.workload, rank, world)
    inp = W.generate(w)
    host = {}
    for n in ("q", "k", "v", "g", "beta"):
        host[n] = torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(
            torch.bfloat16).pin_memory()
    for n in ("A_log", "dt_bias", "initial_state"):
        host[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).pin_memory()
    d = {n: t.to(dev) for n, t in host.items()}
    cu = w.cu_seqlens if (w.layout == "TND" or any(L != w.S for L in w.lengths)) else None
    plan = kda.plan(d["q"], d["v"], d["initial_state"], w.layout, cu_seqlens=cu,
                    segment_chunks=None if args.segment_chunks < 0 else args.segment_chunks)
    ws = plan.workspace()
    out = torch.empty_like(d["v"])
    fs = torch.empty((w.B, w.Nv, w.D, w.D), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    small_l2 = 5 * (w.S if w.layout == "TND" else w.B * w.S) * w.Nv * w.D * 2 <= 126e6
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if small_l2 else None

    def fwd():
        kda.flash_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale, d["initial_state"],
                      d["A_log"], d["dt_bias"], w.lower_bound, w.layout, plan, out=out,
                      final_state=fs, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            if flush is not None:
                flush.zero_()
            fwd()
    kda.device_status(ws, stream)
    torch.cuda.synchronize(dev)
    barrier()

    # ---- device-resident timed region ----
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fl_ms = 0.0
    with ClockSampler(local) as clk:
        torch.cuda.synchronize(dev)
        barrier()
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                if flush is not None:
                    flush.zero_()
                fwd()
            end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    elapsed_ms = start.elapsed_time(end)
    if flush is not None:  # time the flushes alone and take them out of the kernel time
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            f0.record(stream)
            for _ in range(args.steps):
                flush.zero_()
            f1.record(stream)
        torch.cuda.synchronize(dev)
        fl_ms = f0.elapsed_time(f1)
    kda.device_status(ws, stream)
    elapsed_ms = _max_over_ranks(elapsed_ms, dist, dev)
    kernel_ms = (elapsed_ms - fl_ms) / args.steps

    # ---- end to end: pinned host inputs -> device -> forward -> host outputs ----
    # Every step copies its inputs in and its outputs out through the public API.  Steps are
    # pipelined the way a serving loop would run them: two buffer sets and three streams, so the
    # H2D copy of step k+1 and the D2H copy of step k-1 overlap step k's forward.
    e2e = None
    if not args.no_e2e:
        bufs = [{"d": d, "out": out, "fs": fs}]
        bufs.append({"d": {n: torch.empty_like(t) for n, t in d.items()},
                     "out": torch.empty_like(out), "fs": torch.empty_like(fs)})
        for bset in bufs:
            bset["out_h"] = torch.empty(out.shape, dtype=out.dtype).pin_memory()
            bset["fs_h"] = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = bufs[0]["out_h"].numel() * 2 + bufs[0]["fs_h"].numel() * 4
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        steps_e2e = max(1, min(args.steps, args.e2e_steps))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        barrier()
        e0.record(s_in)
        stream.wait_event(e0)
        s_out.wait_event(e0)
        for k in range(steps_e2e):
            i = k % 2
            bset = bufs[i]
            if k >= 2:
                s_in.wait_event(comp_done[i])   # step k-2 has read these inputs
            with torch.cuda.stream(s_in):
                for n, t in host.items():
                    bset["d"][n].copy_(t, non_blocking=True)
            h2d_done[i].record(s_in)
            stream.wait_event(h2d_done[i])
            if k >= 2:
                stream.wait_event(d2h_done[i])  # step k-2's outputs have left these buffers
            dd = bset["d"]
            kda.flash_kda(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], w.scale,
                          dd["initial_state"], dd["A_log"], dd["dt_bias"], w.lower_bound,
                          w.layout, plan, out=bset["out"], final_state=bset["fs"], workspace=ws,
                          stream=stream)
            comp_done[i].record(stream)
            s_out.wait_event(comp_done[i])
            with torch.cuda.stream(s_out):
                bset["out_h"].copy_(bset["out"], non_blocking=True)
                bset["fs_h"].copy_(bset["fs"], non_blocking=True)
            d2h_done[i].record(s_out)
        s_out.wait_stream(s_in)
        s_out.wait_stream(stream)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        barrier()
        kda.device_status(ws, stream)
        e_ms = _max_over_ranks(e0.elapsed_time(e1), dist, dev)
        e2e = {"value": job_throughput(w.token_heads, world, steps_e2e, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": steps_e2e,
               "pipeline": "two buffer sets, three streams: H2D of step k+1 and D2H of step "
                           "k-1 overlap step k"}

    value = job_throughput(w.token_heads, world, args.steps, elapsed_ms)
    peak, peak_kind = measured_peaks()
    abytes = algorithmic_bytes(w, True)
    achieved = abytes / (kernel_ms / 1e3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 inputs, random-init A_log/dt_bias)",
            "config": dict(_config(w, world), schedule=(
                schedule_name(plan, w, ", one CTA each")
                + (" (chunk-parallel scan)" if plan.segment_chunks > 0 else ""))),
            "clocks": clk.report(), "e2e": e2e,
            "gpu_launches": args.steps * kda.kernels_per_forward(plan),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": ncu_traffic(w.name),
                         "kernel": kda.forward_kernel_names(),
                         "algorithmic_bytes": abytes, "kernel_ms": kernel_ms,
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "tensor_tflops": algorithmic_flops(w) / (kernel_ms / 1e3) / 1e12}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], _ = cpu_oracle_sample(w, inp, budget_s=args.cpu_budget)
    if rank == 0 and world == 1 and not args.no_per_config:
        del d, out, fs, ws
        if not args.no_e2e:
            del bufs
        torch.cuda.empty_cache()
        line["per_config"] = per_config(args, dev, kda, cached=(args.workload, inp))
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


PER_CONFIG = (1, 2, 3, 4, 5, 6, 7)


def time_calls(fn, n: int, stream, flush=None) -> list:
    """Device time of each of n calls of fn, each bracketed by its own CUDA events on `stream`;
    `flush` (a buffer larger than L2) is zeroed before every call, outside the brackets."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            if flush is not None:
                flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def per_config(args, dev, kda, cached=None):
    """Every synthetic workload on this GPU: the median and p10/p90 of --per-config-calls calls
    (each timed alone, after 10 warm-up calls; L2 flushed before each call when the inputs fit
    in it), token-heads/s and the HBM roofline fraction at the median, the schedule, and the
    fp64 oracle's token-heads/s in both forms on a bounded sample, with its thread count."""
    import torch
    peak, peak_kind = measured_peaks()
    rows = []
    for idx in PER_CONFIG:
        w = W.workload(idx)
        inp = cached[1] if cached is not None and cached[0] == idx else W.generate(w)
        d = {n: torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(
            torch.bfloat16).to(dev) for n in ("q", "k", "v", "g", "beta")}
        for n in ("A_log", "dt_bias", "initial_state"):
            d[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).to(dev)
        cu = w.cu_seqlens if (w.layout == "TND" or any(L != w.S for L in w.lengths)) else None
        plan = kda.plan(d["q"], d["v"], d["initial_state"], w.layout, cu_seqlens=cu)
        ws = plan.workspace()
        out = torch.empty_like(d["v"])
        fs = torch.empty((w.B, w.Nv, w.D, w.D), dtype=torch.float32, device=dev)
        stream = torch.cuda.Stream(dev)
        in_bytes = 5 * (w.S if w.layout == "TND" else w.B * w.S) * w.Nv * w.D * 2
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes <= 126e6 else None

        def fwd():
            kda.flash_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale, d["initial_state"],
                          d["A_log"], d["dt_bias"], w.lower_bound, w.layout, plan, out=out,
                          final_state=fs, workspace=ws, stream=stream)

        time_calls(fwd, 10, stream, flush)
        ms = np.array(time_calls(fwd, args.per_config_calls, stream, flush))
        kda.device_status(ws, stream)
        med = float(np.median(ms))
        abytes = algorithmic_bytes(w, True)
        row = {"workload": w.name, "calls": int(ms.size), "ms_median": med,
               "ms_p10": float(np.percentile(ms, 10)), "ms_p90": float(np.percentile(ms, 90)),
               "token_heads": w.token_heads, "value": w.token_heads / (med / 1e3), "unit": UNIT,
               "roofline": {"bound": "hbm", "achieved": abytes / (med / 1e3) / 1e9,
                            "peak": peak, "unit": "GB/s",
                            "frac": abytes / (med / 1e3) / 1e9 / peak,
                            "peak_source": f"{peak_kind} hbm_gbs",
                            "algorithmic_bytes": abytes},
               "schedule": schedule_name(plan, w),
               "l2": "flushed before each call" if flush is not None else "inputs larger than L2"}
        del d, out, fs, ws, plan, flush
        torch.cuda.empty_cache()
        if not args.no_cpu_baseline:
            row["oracle"] = {}
            for form in ("recurrent", "chunked"):
                r, _ = cpu_oracle_sample(w, inp, budget_s=args.per_config_cpu_budget,
                                         tokens=min(w.S, 2048) if w.layout != "TND" else None,
                                         form=form)
                row["oracle"][form] = {"value": r["value"], "unit": UNIT, "cores": r["cores"],
                                       "sample": r["sample"]}
        rows.append(row)
        del inp
    return rows


def rank_workload(idx: int, rank: int, world: int) -> W.Workload:
    """The workload replica of one rank: same shapes, its own seed (rank r adds 1000 r)."""
    w = W.workload(idx)
    if world > 1:
        w.seed = w.seed + 1000 * rank
    return w


def job_throughput(token_heads: int, world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job token-heads/s: every rank processes `token_heads` per step; the time is the
    slowest rank's (max over ranks)."""
    return world * token_heads * steps / (elapsed_ms / 1e3)


def _max_over_ranks(x, dist, dev):
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


DECODE_METRIC = "KDA decode step token-heads/s per B200 (one token per sequence and value head)"


def decode_bytes(B: int, Nqk: int, Nv: int, D: int = 128) -> int:
    """Unique HBM bytes of one decode step: fp32 state in and out, bf16 q, k (per qk head), v, g,
    out, beta, and the gate parameters."""
    units = B * Nv
    return (units * D * D * 4 * 2 + B * Nqk * D * 2 * 2 + units * D * 2 * 3 + units * 2
            + Nv * 4 + Nv * D * 4)


def run_decode(args, rank, world):
    """One decode step per (sequence, value head) with the state updated in place."""
    import torch
    import chunked_kda_prefill_b200 as kda

    local = _env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, Nqk, Nv, D = args.decode_batch, 32, 32, 128
    rng = np.random.default_rng(7 + 1000 * rank)

    def bf16(shape):
        return torch.from_numpy(W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
                                .view(np.int16)).view(torch.bfloat16).to(dev)

    q, k = bf16((B, Nqk, D)), bf16((B, Nqk, D))
    v, g, beta = bf16((B, Nv, D)), bf16((B, Nv, D)), bf16((B, Nv))
    A_log = torch.from_numpy(rng.standard_normal(Nv).astype(np.float32)).to(dev)
    dt_bias = torch.from_numpy(rng.standard_normal((Nv, D)).astype(np.float32)).to(dev)
    state = torch.from_numpy((0.1 * rng.standard_normal((B, Nv, D, D))).astype(np.float32)).to(dev)
    out = torch.empty_like(v)
    stream = torch.cuda.Stream(dev)

    def step():
        kda.decode(q, k, v, g, beta, D ** -0.5, state, A_log, dt_bias, -5.0, out=out,
                   state_out=state, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                step()
            end.record(stream)
        torch.cuda.synchronize(dev)
    ms = start.elapsed_time(end) / args.steps
    units = B * Nv
    nbytes = decode_bytes(B, Nqk, Nv, D)
    peak, peak_kind = measured_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    line = {"metric": DECODE_METRIC, "value": world * units / (ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded N(0,1) bf16 inputs, 0.1 N(0,1) fp32 state)",
            "config": {"workload": f"decode_{B}x{Nqk}x{Nv}", "B": B, "Nqk": Nqk, "Nv": Nv,
                       "D": D, "lower_bound": -5.0, "state": "updated in place",
                       "l2": f"state ({units * D * D * 4 / 1e9:.2f} GB) larger than L2"},
            "clocks": clk.report(), "gpu_launches": args.steps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "kernel": "kda_decode_kernel",
                         "algorithmic_bytes": nbytes, "kernel_ms": ms,
                         "peak_source": f"{peak_kind} hbm_gbs"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


CP_METRIC = "KDA prefill tokens/s, one sequence split over ranks (context parallel)"


def run_cp(args, rank, world):
    """Context parallelism: rank r holds the r-th span of cp_span tokens of one sequence
    (cp_heads query/key and value heads, D = 128, BNSD), one all-gather of the span maps.

    With one process, ``--cp-emulate E`` runs the work of E ranks on this GPU one after another
    and reports the slowest rank's time (its summary, fold and forward; the all-gather of
    2 x heads x 64 KiB per rank is not timed), beside one forward over the whole sequence."""
    import torch
    import chunked_kda_prefill_b200 as kda

    local = _env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    ranks = world if world > 1 else max(1, args.cp_emulate)
    H, S_loc, D = args.cp_heads, args.cp_span, 128
    w = W.custom(f"cp_span_1x{H}x{S_loc}", "BNSD", 1, H, H, S_loc, [S_loc], lower_bound=-5.0,
                 init_state="zeros", seed=300 + rank)
    inp = W.generate(w)
    d = {n: torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(
        torch.bfloat16).to(dev) for n in ("q", "k", "v", "g", "beta")}
    for n in ("A_log", "dt_bias", "initial_state"):
        d[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).to(dev)
    plan = kda.plan(d["q"], d["v"], d["initial_state"], "BNSD")
    args_fwd = (d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale)
    tail = (d["A_log"], d["dt_bias"], w.lower_bound, "BNSD", plan)

    def timed(fn, n):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        return a.elapsed_time(b) / n

    with ClockSampler(local) as clk:
        if world > 1:
            ms = timed(lambda: kda.flash_kda_context_parallel(*args_fwd, d["initial_state"],
                                                              *tail), args.steps)
            ms = _max_over_ranks(ms, dist, dev)
            parts, whole = None, None
        else:
            gathered = torch.zeros((ranks, 2, 1, H, D, D), dtype=torch.float32, device=dev)
            t_sum = timed(lambda: kda.forward_summary(
                d["q"], d["k"], d["v"], d["g"], d["beta"], *tail, M=gathered[0, 0],
                R=gathered[0, 1]), args.steps)
            t_fwd = timed(lambda: kda.flash_kda(*args_fwd, d["initial_state"], *tail),
                          args.steps)
            t_chain = [0.0] + [timed(lambda j=j: kda.state_chain(
                d["initial_state"], gathered[:j, 0], gathered[:j, 1]), args.steps)
                for j in range(1, ranks)]
            per_rank = [(t_sum if r < ranks - 1 else 0.0) + t_chain[r] + t_fwd
                        for r in range(ranks)]
            ms = max(per_rank)
            parts = {"summary_ms": t_sum, "forward_ms": t_fwd, "chain_ms": t_chain,
                     "per_rank_ms": per_rank}
            whole = None
            if ranks > 1:  # the whole sequence on this one GPU, for comparison
                wf = W.custom(f"cp_whole_1x{H}x{ranks * S_loc}", "BNSD", 1, H, H,
                              ranks * S_loc, [ranks * S_loc], init_state="zeros", seed=301)
                fi = W.generate(wf)
                fd = {n: torch.from_numpy(np.ascontiguousarray(fi[n]).view(np.int16)).view(
                    torch.bfloat16).to(dev) for n in ("q", "k", "v", "g", "beta")}
                fplan = kda.plan(fd["q"], fd["v"], d["initial_state"], "BNSD")
                whole = {"ms": timed(lambda: kda.flash_kda(
                    fd["q"], fd["k"], fd["v"], fd["g"], fd["beta"], w.scale, d["initial_state"],
                    d["A_log"], d["dt_bias"], w.lower_bound, "BNSD", fplan), args.steps),
                    "schedule": (f"segments of {fplan.segment_chunks} chunks"
                                 if fplan.segment_chunks > 0 else "whole units")}
    token_heads = ranks * S_loc * H
    line = {"metric": CP_METRIC, "value": token_heads / (ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 inputs)",
            "config": {"workload": f"context_parallel_1x{H}x{S_loc}_per_rank", "ranks": ranks,
                       "emulated": world == 1 and ranks > 1, "span_tokens": S_loc, "heads": H,
                       "D": D, "exchange": "one all_gather of [M; R] per rank (2 x 64 KiB "
                       "per head)" + (", not timed (ranks emulated on one GPU)"
                                      if world == 1 else "")},
            "clocks": clk.report(), "parts": parts, "whole_sequence_one_gpu": whole}
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def render_table(path: str) -> str:
    """The per-workload markdown table of a bench JSON line (the last line of `path` that has a
    per_config list)."""
    line = None
    with open(path) as f:
        for raw in f:
            raw = raw.strip()
            if raw.startswith("{") and '"per_config"' in raw:
                line = json.loads(raw)
    if line is None:
        raise SystemExit(f"{path}: no bench line with per_config")
    rows = ["| workload | schedule | ms median (p10-p90), 50 calls | token-heads/s | of HBM peak "
            "| oracle recurrent / chunked, token-heads/s (threads) |",
            "|---|---|---|---|---|---|"]
    for r in line["per_config"]:
        o = r.get("oracle") or {}
        rec, chk = o.get("recurrent"), o.get("chunked")
        ora = (f"{rec['value']:.3g} / {chk['value']:.3g} ({rec['cores']})" if rec and chk else "-")
        rows.append(f"| {r['workload']} | {r['schedule']} | {r['ms_median']:.4f} "
                    f"({r['ms_p10']:.4f}-{r['ms_p90']:.4f}) | {r['value']:.3g} | "
                    f"{100 * r['roofline']['frac']:.1f} % | {ora} |")
    clk = line.get("clocks") or {}
    rows.append("")
    rows.append(f"SM clock {clk.get('sm_mhz')} MHz (max {clk.get('sm_max_mhz')}), throttle reasons "
                f"{clk.get('reasons')}; peak {line['roofline']['peak']} GB/s "
                f"({line['roofline'].get('peak_source')}).")
    return "\n".join(rows)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=5,
                    help="1-5 the five synthetic workloads (5 = the large prefill), 6 head dim "
                         "64, 7 the large prefill at B = 1")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=4096)
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload table (workloads 1-7, rank 0 at N = 1 only)")
    ap.add_argument("--per-config-calls", type=int, default=50)
    ap.add_argument("--per-config-cpu-budget", type=float, default=1.5,
                    help="seconds of oracle time per workload and form")
    ap.add_argument("--mode", default="prefill", choices=["prefill", "decode", "cp"],
                    help="prefill (the default, the headline), the single-token decode step, "
                         "or context parallelism (one sequence split over the ranks)")
    ap.add_argument("--cp-span", type=int, default=8192, help="cp: tokens per rank")
    ap.add_argument("--cp-heads", type=int, default=3, help="cp: heads (Nqk = Nv)")
    ap.add_argument("--cp-emulate", type=int, default=1,
                    help="cp with one process: ranks to emulate one after another")
    ap.add_argument("--decode-batch", type=int, default=256)
    ap.add_argument("--segment-chunks", type=int, default=-1,
                    help="schedule: -1 the planner's choice, 0 whole units, n > 0 segments of n "
                         "chunks (chunk-parallel scan)")
    ap.add_argument("--table", metavar="BENCH_JSON",
                    help="print the per-workload markdown table of a saved bench line and exit")
    args = ap.parse_args()
    if args.table:
        print(render_table(args.table))
        return 0
    args.warmup = max(args.warmup, 3)
    args.per_config_calls = max(args.per_config_calls, 50)
    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.mode == "decode":
        return run_decode(args, rank, world)
    if args.mode == "cp":
        return run_cp(args, rank, world)
    return run_ours(args, rank, world)


if __name__ == "__main__":
    sys.exit(main())

"""Helpers for the GPU tests: seeded inputs -> torch device tensors -> libkda.so, and the
elementwise comparison with the fp64 oracle (atol = rtol = 5e-3, FlashKDA README 精度测试)."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W

ATOL = 5e-3
RTOL = 5e-3


def to_dev(inp: dict, device="cuda") -> dict:
    d = {}
    for n in ("q", "k", "v", "g", "beta"):
        d[n] = torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(
            torch.bfloat16).to(device)
    for n in ("A_log", "dt_bias", "initial_state"):
        d[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).to(device)
    return d


def run_gpu(w: W.Workload, inp: dict, dev: dict | None = None, with_init=True, plan=None):
    """Run the CUDA path; returns (out fp32 numpy in v's layout, final_state fp32 numpy)."""
    dev = dev or to_dev(inp)
    cu = w.cu_seqlens if (w.layout == "TND" or any(L != w.S for L in w.lengths)) else None
    if plan is None:
        plan = kda.plan(dev["q"], dev["v"], dev["initial_state"], w.layout, cu_seqlens=cu)
    out, fs = kda.flash_kda(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], w.scale,
                            dev["initial_state"] if with_init else None, dev["A_log"],
                            dev["dt_bias"], w.lower_bound, w.layout, plan)
    kda.device_status(plan.workspace())
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), fs.cpu().numpy()


def valid_mask(w: W.Workload, shape) -> np.ndarray:
    """Boolean mask over out's storage: True on rows inside a valid length."""
    m = np.zeros(shape[:-1], dtype=bool)
    if w.layout == "TND":
        m[:] = True
    for b, L in enumerate(w.lengths):
        if w.layout == "BNSD":
            m[b, :, :L] = True
        elif w.layout == "BSND":
            m[b, :L] = True
    return m


def unit_rows(w: W.Workload, arr: np.ndarray, b: int, h: int) -> np.ndarray:
    L = w.lengths[b]
    if w.layout == "BNSD":
        return arr[b, h, :L]
    if w.layout == "BSND":
        return arr[b, :L, h]
    cu = w.cu_seqlens
    return arr[cu[b]:cu[b] + L, h]


def compare(gpu: np.ndarray, ref: np.ndarray, what: str):
    """|gpu - ref| <= ATOL + RTOL |ref| elementwise; returns a small report dict."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    rep = {"what": what, "max_abs": float(err.max(initial=0.0)),
           "rmse": float(np.sqrt(np.mean(err ** 2))) if err.size else 0.0,
           "ref_rms": float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0,
           "n_bad": int(bad.sum()), "n": int(err.size)}
    rep["max_err_over_bar"] = float((err / bound).max(initial=0.0))
    log = os.environ.get("KDA_PARITY_LOG")
    if log:  # one JSON line per comparison, e.g. to follow the margins across kernel variants
        with open(log, "a") as f:
            f.write(json.dumps(rep) + "\n")
    assert not bad.any(), f"{what}: {rep} first bad at {np.argwhere(bad)[:3].tolist()}"
    return rep

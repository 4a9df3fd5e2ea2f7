"""Python API over libkda.so, mirroring flash_kda_metadata / flash_kda (FlashKDA README, 快速开始).

    plan = chunked_kda_prefill_b200.plan(q, v, initial_state, "BNSD", cu_seqlens=None)
    out, final_state = chunked_kda_prefill_b200.flash_kda(
        q, k, v, g, beta, 1 / math.sqrt(128), initial_state, A_log, dt_bias, -5.0, "BNSD", plan)

PyTorch supplies device memory and the current stream; the functions below only pass
pointers and sizes to the C ABI (include/kda.h).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib
from ._lib import KdaError, KdaShape, check

LAYOUTS = {"BNSD": 0, "BSND": 1, "TND": 2}


@dataclass
class KdaPlan:
    """Host + device copies of the int32 schedule, and the workspace size it needs."""
    shape: KdaShape
    layout: str
    host: np.ndarray
    dev: torch.Tensor
    workspace_bytes: int
    cu_seqlens: np.ndarray | None
    _workspace: torch.Tensor | None = None

    @property
    def n_units(self) -> int:
        return int(self.host[4])

    @property
    def total_chunks(self) -> int:
        return int(self.host[11])

    @property
    def segment_chunks(self) -> int:
        """Segment length of a chunk-parallel (segmented) schedule; 0 when units run whole."""
        return int(self.host[14])

    def workspace(self) -> torch.Tensor:
        """A workspace owned by the plan, allocated on first use and reused afterwards."""
        if self._workspace is None or self._workspace.device != self.dev.device:
            self._workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8,
                                          device=self.dev.device)
        return self._workspace


def _shape_from(q: torch.Tensor, v: torch.Tensor, layout: str, cu_seqlens) -> KdaShape:
    if layout not in LAYOUTS:
        raise KdaError(2, f"layout {layout!r}")
    if layout == "BNSD":
        B, Nqk, S, D = q.shape
        Nv = v.shape[1]
    elif layout == "BSND":
        B, S, Nqk, D = q.shape
        Nv = v.shape[2]
    else:
        if cu_seqlens is None:
            raise KdaError(7, "TND layout needs cu_seqlens")
        S, Nqk, D = q.shape
        Nv = v.shape[1]
        B = len(cu_seqlens) - 1
    return KdaShape(LAYOUTS[layout], int(B), int(Nqk), int(Nv), int(S), int(D))


def make_plan(shape: KdaShape, layout: str, cu_seqlens=None, num_sms: int | None = None,
              device=None, segment_chunks: int | None = None) -> KdaPlan:
    """Build a plan from an explicit shape (host work only, plus one small device copy).

    ``segment_chunks``: None picks the schedule (kda_plan); 0 runs every unit whole; n > 0 cuts
    units into segments of n chunks (kda_plan_segmented).
    """
    L = _lib.load()
    n = ctypes.c_size_t(0)
    check(L.kda_plan_size(ctypes.byref(shape), ctypes.byref(n)), "kda_plan_size")
    host = np.zeros(n.value, dtype=np.int32)
    cu = None
    cu_ptr = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64)).astype(np.int32)
        cu_ptr = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    if num_sms is None:
        num_sms = (torch.cuda.get_device_properties(device).multi_processor_count
                   if torch.cuda.is_available() else 148)
    hp = host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    if segment_chunks is None:
        check(L.kda_plan(ctypes.byref(shape), cu_ptr, int(num_sms), hp, host.size), "kda_plan")
    else:
        check(L.kda_plan_segmented(ctypes.byref(shape), cu_ptr, int(num_sms), int(segment_chunks),
                                   hp, host.size), "kda_plan_segmented")
    ws = ctypes.c_size_t(0)
    check(L.kda_workspace_size(host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), host.size,
                               ctypes.byref(ws)), "kda_workspace_size")
    if device is not None and torch.cuda.is_available():
        dev = torch.from_numpy(host).to(device)
    else:
        dev = torch.from_numpy(host.copy())
    return KdaPlan(shape, layout, host, dev, int(ws.value), cu)


def plan(q: torch.Tensor, v: torch.Tensor, initial_state: torch.Tensor | None, layout: str,
         cu_seqlens=None, num_sms: int | None = None,
         segment_chunks: int | None = None) -> KdaPlan:
    """flash_kda_metadata counterpart: shapes, layout and valid lengths -> schedule."""
    if isinstance(cu_seqlens, torch.Tensor):
        cu_seqlens = cu_seqlens.detach().to("cpu").numpy()
    shape = _shape_from(q, v, layout, cu_seqlens)
    if initial_state is not None and initial_state.shape[0] != shape.B:
        raise KdaError(3, "initial_state batch does not match the number of sequences")
    return make_plan(shape, layout, cu_seqlens, num_sms, device=q.device,
                     segment_chunks=segment_chunks)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _expect(t, name, dtype, device):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")


def _expect_shape(t, name, shape):
    if tuple(t.shape) != tuple(shape):
        raise KdaError(3, f"{name} has shape {tuple(t.shape)}, the plan needs {tuple(shape)}")


def _io_shapes(sh: KdaShape, layout: str) -> dict:
    """Shapes the plan's problem gives every tensor (include/kda.h, tensor layouts)."""
    B, Nqk, Nv, S, D = sh.B, sh.Nqk, sh.Nv, sh.S, sh.D
    if layout == "BNSD":
        qk, vg, bt = (B, Nqk, S, D), (B, Nv, S, D), (B, Nv, S)
    elif layout == "BSND":
        qk, vg, bt = (B, S, Nqk, D), (B, S, Nv, D), (B, S, Nv)
    else:
        qk, vg, bt = (S, Nqk, D), (S, Nv, D), (S, Nv)
    return {"q": qk, "k": qk, "v": vg, "g": vg, "beta": bt, "out": vg, "A_log": (Nv,),
            "dt_bias": (Nv, D), "state": (B, Nv, D, D)}


def _check_inputs(plan: KdaPlan, layout: str, dev, tensors: dict) -> dict:
    """Dtype, contiguity, device and shape of every tensor against the plan (None = absent).

    The library sees only pointers, so a tensor smaller than the plan's problem must be caught
    here, before a kernel reads past its end.
    """
    if plan.layout != layout:
        raise KdaError(8, "plan was built for another layout")
    if plan.dev.device != dev:
        raise ValueError(f"the plan's device copy is on {plan.dev.device}, the tensors on {dev}; "
                         "build the plan with plan(...) or make_plan(..., device=...)")
    want = _io_shapes(plan.shape, layout)
    for name, t in tensors.items():
        if t is None:
            continue
        key = "state" if name in ("initial_state", "final_state", "M", "R") else name
        dtype = torch.bfloat16 if key in ("q", "k", "v", "g", "beta", "out") else torch.float32
        _expect(t, name, dtype, dev)
        _expect_shape(t, name, want[key])
    return want


def _workspace_bytes(workspace: torch.Tensor, dev) -> int:
    """Size in bytes of a caller's workspace, after checking it is contiguous memory on ``dev``."""
    if workspace.device != dev or not workspace.is_contiguous():
        raise ValueError(f"workspace must be contiguous and on {dev}")
    return workspace.numel() * workspace.element_size()


def flash_kda(q, k, v, g, beta, scale: float, initial_state, A_log, dt_bias, lower_bound: float,
              layout: str, plan: KdaPlan, out: torch.Tensor | None = None,
              final_state: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """The fused forward pass. Returns (out, final_state); out has v's shape and layout."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("flash_kda runs on a CUDA device only")
    _check_inputs(plan, layout, dev, {"q": q, "k": k, "v": v, "g": g, "beta": beta,
                                      "A_log": A_log, "dt_bias": dt_bias,
                                      "initial_state": initial_state, "out": out,
                                      "final_state": final_state})
    sh = plan.shape
    if out is None:
        out = torch.empty_like(v)
    if final_state is None:
        final_state = torch.empty((sh.B, sh.Nv, sh.D, sh.D), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = plan.workspace()
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    L = _lib.load()
    code = L.kda_forward(ctypes.byref(sh), plan.host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                         plan.dev.data_ptr(), plan.host.size, q.data_ptr(), k.data_ptr(),
                         v.data_ptr(), g.data_ptr(), beta.data_ptr(), float(scale),
                         _ptr(initial_state), A_log.data_ptr(), dt_bias.data_ptr(),
                         float(lower_bound), workspace.data_ptr(),
                         _workspace_bytes(workspace, dev),
                         out.data_ptr(), final_state.data_ptr(), s.cuda_stream)
    check(code, "kda_forward")
    return out, final_state


def flash_kda_noalloc(q, k, v, g, beta, scale: float, initial_state, A_log, dt_bias,
                      lower_bound: float, layout: str, plan: KdaPlan, out: torch.Tensor,
                      final_state: torch.Tensor, stream: torch.cuda.Stream | None = None):
    """flash_kda through kda_forward_noalloc: no workspace, the library's fixed scratch instead.

    For callers that cannot allocate device memory; the caller still provides out and
    final_state.  It runs the same kernels as flash_kda.  Raises KdaError(KDA_ERR_CAPACITY) for
    a plan whose workspace would exceed the scratch.  noalloc_status() reads the device status.
    """
    dev = q.device
    if out is None or final_state is None:
        raise ValueError("flash_kda_noalloc needs out and final_state")
    _check_inputs(plan, layout, dev, {"q": q, "k": k, "v": v, "g": g, "beta": beta,
                                      "A_log": A_log, "dt_bias": dt_bias,
                                      "initial_state": initial_state, "out": out,
                                      "final_state": final_state})
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    code = _lib.load().kda_forward_noalloc(
        ctypes.byref(plan.shape), plan.host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        plan.dev.data_ptr(), plan.host.size, q.data_ptr(), k.data_ptr(), v.data_ptr(),
        g.data_ptr(), beta.data_ptr(), float(scale), _ptr(initial_state), A_log.data_ptr(),
        dt_bias.data_ptr(), float(lower_bound), out.data_ptr(), final_state.data_ptr(),
        s.cuda_stream)
    check(code, "kda_forward_noalloc")
    return out, final_state


def decode(q, k, v, g, beta, scale: float, state, A_log, dt_bias, lower_bound: float,
           out: torch.Tensor | None = None, state_out: torch.Tensor | None = None,
           stream: torch.cuda.Stream | None = None):
    """One decode step (one token per sequence) through kda_decode.

    q, k: bf16 [B, Nqk, D]; v, g: bf16 [B, Nv, D]; beta: bf16 [B, Nv]; state: fp32
    [B, Nv, D, D] or None (zeros), D = 128 or 64.  Returns (out [B, Nv, D] bf16, state_out);
    pass ``state_out=state`` to update the state in place.
    """
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("decode runs on a CUDA device only")
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta")):
        _expect(t, name, torch.bfloat16, dev)
    for t, name in ((A_log, "A_log"), (dt_bias, "dt_bias")):
        _expect(t, name, torch.float32, dev)
    if state is not None:
        _expect(state, "state", torch.float32, dev)
    if q.dim() != 3 or v.dim() != 3 or beta.shape != v.shape[:2]:
        raise KdaError(3, "decode expects q/k [B,Nqk,D], v/g [B,Nv,D], beta [B,Nv]")
    B, Nqk, D = q.shape
    Nv = v.shape[1]
    if out is None:
        out = torch.empty_like(v)
    if state_out is None:
        state_out = torch.empty((B, Nv, D, D), dtype=torch.float32, device=dev)
    _expect(out, "out", torch.bfloat16, dev)
    _expect(state_out, "state_out", torch.float32, dev)
    for t, name, want in ((k, "k", q.shape), (v, "v", (B, Nv, D)), (g, "g", (B, Nv, D)),
                          (out, "out", (B, Nv, D)), (A_log, "A_log", (Nv,)),
                          (dt_bias, "dt_bias", (Nv, D)), (state, "state", (B, Nv, D, D)),
                          (state_out, "state_out", (B, Nv, D, D))):
        if t is not None:
            _expect_shape(t, name, want)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    code = _lib.load().kda_decode(B, Nqk, Nv, D, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  g.data_ptr(), beta.data_ptr(), float(scale), _ptr(state),
                                  A_log.data_ptr(), dt_bias.data_ptr(), float(lower_bound),
                                  out.data_ptr(), state_out.data_ptr(), s.cuda_stream)
    check(code, "kda_decode")
    return out, state_out


def forward_summary(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, layout: str,
                    plan: KdaPlan, M: torch.Tensor | None = None, R: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None,
                    stream: torch.cuda.Stream | None = None):
    """Every unit's affine state map over its tokens, S_end = S_start M + R (kda_forward_summary).

    Returns (M, R), fp32 [B, Nv, D, D] each; no outputs are written.  M and R may be given (for
    example two halves of one exchange buffer).
    """
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("forward_summary runs on a CUDA device only")
    _check_inputs(plan, layout, dev, {"q": q, "k": k, "v": v, "g": g, "beta": beta,
                                      "A_log": A_log, "dt_bias": dt_bias, "M": M, "R": R})
    sh = plan.shape
    if M is None:
        M = torch.empty((sh.B, sh.Nv, sh.D, sh.D), dtype=torch.float32, device=dev)
    if R is None:
        R = torch.empty((sh.B, sh.Nv, sh.D, sh.D), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = plan.workspace()
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    code = _lib.load().kda_forward_summary(
        ctypes.byref(sh), plan.host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        plan.dev.data_ptr(), plan.host.size, q.data_ptr(), k.data_ptr(), v.data_ptr(),
        g.data_ptr(), beta.data_ptr(), A_log.data_ptr(), dt_bias.data_ptr(), float(lower_bound),
        workspace.data_ptr(), _workspace_bytes(workspace, dev), M.data_ptr(), R.data_ptr(),
        s.cuda_stream)
    check(code, "kda_forward_summary")
    return M, R


def state_chain(S_in: torch.Tensor | None, M: torch.Tensor, R: torch.Tensor,
                S_out: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """S = S_in; for j: S = S M[j] + R[j]; returns S (kda_state_chain, fp32).

    M and R: [n, B, Nv, D, D] views whose per-step blocks are contiguous and equally spaced (a
    packed stack, or the two halves of an all-gathered [world, 2, B, Nv, D, D] buffer).  S_in:
    [B, Nv, D, D] or None (zeros).  n may be 0.
    """
    if M.dim() != 5 or M.shape != R.shape or M.stride() != R.stride():
        raise ValueError("M and R must be [n, B, Nv, D, D] views with the same layout")
    n, B, Nv, D, _ = M.shape
    mat = B * Nv * D * D
    if n > 0 and not (M[0].is_contiguous() and R[0].is_contiguous()):
        raise ValueError("every step's maps must be contiguous")
    step = M.stride(0) if n > 1 else mat
    dev = M.device
    for t, name in ((M, "M"), (R, "R")):
        if t.dtype != torch.float32 or t.device != dev:
            raise TypeError(f"{name} must be fp32 on {dev}")
    if S_in is not None:
        _expect(S_in, "S_in", torch.float32, dev)
        _expect_shape(S_in, "S_in", (B, Nv, D, D))
    if S_out is None:
        S_out = torch.empty((B, Nv, D, D), dtype=torch.float32, device=dev)
    _expect(S_out, "S_out", torch.float32, dev)
    _expect_shape(S_out, "S_out", (B, Nv, D, D))
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    code = _lib.load().kda_state_chain(B * Nv, D, n, _ptr(S_in), M.data_ptr() if n else None,
                                       R.data_ptr() if n else None, int(step),
                                       S_out.data_ptr(), s.cuda_stream)
    check(code, "kda_state_chain")
    return S_out


def device_status(workspace: torch.Tensor, stream: torch.cuda.Stream | None = None) -> None:
    """Synchronise and raise if the last forward on this workspace recorded a device error."""
    s = stream if stream is not None else torch.cuda.current_stream(workspace.device)
    check(_lib.load().kda_device_status(workspace.data_ptr(), s.cuda_stream), "kda_device_status")


def noalloc_status(device=None, stream: torch.cuda.Stream | None = None) -> None:
    """Synchronise and raise if the last flash_kda_noalloc on this device recorded a device
    error (its status word lives in the library's fixed scratch)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        check(_lib.load().kda_noalloc_status(s.cuda_stream), "kda_noalloc_status")


def kernels_per_forward(plan: KdaPlan | None = None) -> int:
    """Kernels of this library that one kda_forward launches (three under a segmented plan)."""
    return 3 if plan is not None and plan.segment_chunks > 0 else 1


def forward_kernel_names() -> str:
    return "kda_fused_kernel"

"""The fused tcgen05 kernel's per-chunk intermediates against the fp32 two-kernel path.

Both paths are this library's own CUDA code: the two-kernel path keeps every operand in fp32,
the fused path feeds bf16 operands to the tensor cores, so the comparison is relative to each
quantity's scale (bf16 operands: a few parts in 10^3).  A mismatch here points at the phase
that broke (W and U: solve and W/U MMAs; Q~, K^: prologue; Aqk: intra MMA; gamma: cumsum).
Also checks that the fused kernel's outputs agree with the two-kernel path's.
"""
import ctypes

import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
from kda_gpu import to_dev

pytestmark = pytest.mark.gpu

CHUNK_FLOATS = 148480 // 4
FIELDS = {"W": (0, 64 * 128), "U": (8192, 64 * 128), "Qt": (16384, 64 * 128),
          "Kh": (24576, 64 * 128), "Aqk": (32768, 64 * 64), "gC": (36864, 128)}


def _bind(L):
    P = ctypes.POINTER(ctypes.c_int32)
    sz, vp, f = ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
    sh = ctypes.POINTER(kda.KdaShape)
    L.kda_forward_simt.argtypes = [sh, P, vp, sz, vp, vp, vp, vp, vp, f, vp, vp, vp, f, vp, sz,
                                   vp, vp, vp]
    L.kda_forward_debug.argtypes = [sh, P, vp, sz, vp, vp, vp, vp, vp, f, vp, vp, vp, f, vp, sz,
                                    vp, vp, vp, vp, vp]
    L.kda_simt_workspace_size.argtypes = [P, sz, ctypes.POINTER(sz)]
    for n in ("kda_forward_simt", "kda_forward_debug", "kda_simt_workspace_size"):
        getattr(L, n).restype = ctypes.c_int
    return L


def _run_both(w):
    L = _bind(kda.load())
    inp = W.generate(w)
    d = to_dev(inp)
    cu = w.cu_seqlens if (w.layout == "TND" or any(x != w.S for x in w.lengths)) else None
    plan = kda.plan(d["q"], d["v"], d["initial_state"], w.layout, cu_seqlens=cu)
    hp = plan.host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    nbytes = ctypes.c_size_t(0)
    assert L.kda_simt_workspace_size(hp, plan.host.size, ctypes.byref(nbytes)) == 0
    ws = torch.zeros(nbytes.value, dtype=torch.uint8, device="cuda")
    dump = torch.zeros(nbytes.value // 4, dtype=torch.float32, device="cuda")
    outs = {}
    s = torch.cuda.current_stream().cuda_stream
    args = lambda out, fs: (ctypes.byref(plan.shape), hp, plan.dev.data_ptr(), plan.host.size,
                            d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(),
                            d["g"].data_ptr(), d["beta"].data_ptr(), w.scale,
                            d["initial_state"].data_ptr(), d["A_log"].data_ptr(),
                            d["dt_bias"].data_ptr(), w.lower_bound, ws.data_ptr(), ws.numel(),
                            out.data_ptr(), fs.data_ptr())
    for name in ("simt", "fused"):
        out = torch.empty_like(d["v"])
        fs = torch.empty((w.B, w.Nv, 128, 128), dtype=torch.float32, device="cuda")
        if name == "simt":
            assert L.kda_forward_simt(*args(out, fs), s) == 0
            torch.cuda.synchronize()
            simt_ws = ws[256:].view(torch.float32).clone()
        else:
            assert L.kda_forward_debug(*args(out, fs), dump.data_ptr() + 256, None, s) == 0
            torch.cuda.synchronize()
        kda.device_status(ws)
        outs[name] = (out.float().cpu().numpy(), fs.cpu().numpy())
    fused_ws = dump[64:].clone()
    return plan, simt_ws.cpu().numpy(), fused_ws.cpu().numpy(), outs


@pytest.mark.parametrize("case", [("BNSD", 1, 1, 1, 64, [64], -5.0),
                                  ("BNSD", 1, 1, 1, 200, [200], -1.0),
                                  ("TND", 2, 1, 2, 150, [100, 50], -5.0)],
                         ids=lambda c: f"{c[0]}_{c[4]}")
def test_fused_intermediates_match_fp32_path(case, cuda_ok):
    layout, B, Nqk, Nv, S, lens, lb = case
    w = W.custom("dbg", layout, B, Nqk, Nv, S, lens, lower_bound=lb, init_state="normal", seed=7)
    plan, a, b, outs = _run_both(w)
    nchunks = plan.total_chunks
    for c in range(nchunks):
        base = c * CHUNK_FLOATS
        for name, (off, size) in FIELDS.items():
            x = a[base + off: base + off + size]
            y = b[base + off: base + off + size]
            scale = max(float(np.abs(x).max()), 1e-6)
            err = float(np.abs(x - y).max()) / scale
            assert err < 2e-2, f"chunk {c} {name}: max rel err {err:.3e} (scale {scale:.3e})"
    (o1, f1), (o2, f2) = outs["simt"], outs["fused"]
    assert np.abs(o1 - o2).max() < 5e-3 and np.abs(f1 - f2).max() < 5e-3

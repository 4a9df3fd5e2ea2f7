"""kda_forward_noalloc: the forward pass without a caller-provided workspace.

Some callers cannot allocate device memory: a plugin interface that hands over only the tensors,
or a host runtime whose pool forbids extra cudaMalloc calls (which can also synchronise the
device).  The entry point runs the same kernels as kda_forward on the library's fixed per-GPU
scratch instead of a workspace.  These tests call it through the C ABI, read its device status
through kda_noalloc_status, and check every result against the fp64 oracle element by element
(atol = rtol = 5e-3, the tolerance of every parity test) and against kda_forward with its own
workspace, on two calls in a row each (the second call reuses the scratch the first one left).
The file is named to be collected last, and it builds everything it uses itself, so it passes
alone or after the other tests.
"""
import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, to_dev, valid_mask

pytestmark = pytest.mark.gpu

CASES = [
    # name, workload builder, plan's segment length (None: the planner's default)
    ("tiny_1x1x256", lambda: W.workload(1), None),
    ("single_seq_1x3x8192_whole_units", lambda: W.workload(2), 0),
    ("single_seq_1x3x8192_segmented", lambda: W.workload(2), None),
    ("tnd_tails", lambda: W.custom("tnd_tails", "TND", 4, 2, 4, 64 + 1 + 129 + 300,
                                   [64, 1, 129, 300], lower_bound=-3.0, seed=71), None),
    ("headdim64_bsnd_tail", lambda: W.custom("d64", "BSND", 2, 1, 2, 200, [200, 77],
                                             lower_bound=-1.0, scale=64 ** -0.5, seed=73, D=64),
     None),
]


def _noalloc(w, d, plan):
    out = torch.full_like(d["v"], float("nan"))
    fs = torch.full((w.B, w.Nv, w.D, w.D), float("nan"), dtype=torch.float32, device="cuda")
    kda.flash_kda_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale,
                          d["initial_state"], d["A_log"], d["dt_bias"], w.lower_bound,
                          w.layout, plan, out, fs)
    kda.noalloc_status()
    return out.float().cpu().numpy(), fs.cpu().numpy()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(case, cuda_ok):
    name, make, seg = case
    w = make()
    inp = W.generate(w)
    d = to_dev(inp)
    cu = w.cu_seqlens if (w.layout == "TND" or any(L != w.S for L in w.lengths)) else None
    plan = kda.plan(d["q"], d["v"], d["initial_state"], w.layout, cu_seqlens=cu,
                    segment_chunks=seg)
    if name.endswith("_segmented"):
        assert plan.segment_chunks > 0
    o_r, fs_r, _ = oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                    w.lower_bound, w.cu_seqlens)
    ref_out, ref_fs = kda.flash_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale,
                                    d["initial_state"], d["A_log"], d["dt_bias"], w.lower_bound,
                                    w.layout, plan)
    kda.device_status(plan.workspace())
    ref_out = ref_out.float().cpu().numpy()
    ref_fs = ref_fs.cpu().numpy()
    m = valid_mask(w, ref_out.shape)
    for call in range(2):
        o, fs = _noalloc(w, d, plan)
        compare(o[m], o_r[m], f"{name} noalloc out vs oracle, call {call}")
        compare(fs, fs_r, f"{name} noalloc final_state vs oracle, call {call}")
        assert np.all(o[~m] == 0.0), "rows past a valid length must be zero"
        compare(o, ref_out, f"{name} noalloc out vs kda_forward, call {call}")
        compare(fs, ref_fs, f"{name} noalloc final_state vs kda_forward, call {call}")


def test_noalloc_rejects_plans_beyond_its_scratch(cuda_ok):
    # one 65,536-token sequence cut into one-chunk segments: 1,023 state slots of 196,608 bytes
    w = W.custom("cap", "BNSD", 1, 1, 1, 65536, [65536], lower_bound=-5.0, seed=79)
    shape = kda.KdaShape(0, w.B, w.Nqk, w.Nv, w.S, w.D)
    plan = kda.make_plan(shape, w.layout, None, device="cuda", segment_chunks=1)
    assert plan.workspace_bytes > (64 << 20)
    sh = W.shapes(w)
    z = lambda shape, dt=torch.bfloat16: torch.zeros(shape, dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(kda.KdaError) as e:
        kda.flash_kda_noalloc(z(sh["q"]), z(sh["q"]), z(sh["v"]), z(sh["v"]), z(sh["beta"]),
                              w.scale, None, z((w.Nv,), torch.float32),
                              z((w.Nv, w.D), torch.float32), w.lower_bound, w.layout, plan,
                              z(sh["v"]), z((w.B, w.Nv, w.D, w.D), torch.float32))
    assert e.value.name == "KDA_ERR_CAPACITY"

"""kda_forward_noalloc: the forward pass without a caller-provided workspace.

Some callers cannot allocate device memory (for example a plugin interface that hands over
only the tensors, or a host runtime whose pool forbids extra cudaMalloc calls).  The entry point
uses the library's fixed per-GPU scratch instead.  This test calls it through the C ABI twice in
a row and checks each result against the regular kda_forward (with its own workspace) within the
parity tolerance used everywhere else (atol = rtol = 5e-3).  The file is named to be collected
last, and it builds everything it uses itself, so it passes alone or after the other tests.
"""
import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
from kda_gpu import compare, to_dev

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice(cuda_ok):
    w = W.workload(2)  # 1 x 3 x 8192: 384 chunks, within the fixed scratch
    inp = W.generate(w)
    d = to_dev(inp)
    plan = kda.plan(d["q"], d["v"], d["initial_state"], w.layout)
    ref_out, ref_fs = kda.flash_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale,
                                    d["initial_state"], d["A_log"], d["dt_bias"], w.lower_bound,
                                    w.layout, plan)
    kda.device_status(plan.workspace())
    ref_out = ref_out.float().cpu().numpy()
    ref_fs = ref_fs.cpu().numpy()
    for call in range(2):
        out = torch.full_like(d["v"], float("nan"))
        fs = torch.full((w.B, w.Nv, w.D, w.D), float("nan"), dtype=torch.float32, device="cuda")
        kda.flash_kda_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale,
                              d["initial_state"], d["A_log"], d["dt_bias"], w.lower_bound,
                              w.layout, plan, out, fs)
        torch.cuda.synchronize()
        compare(out.float().cpu().numpy(), ref_out, f"noalloc out, call {call}")
        compare(fs.cpu().numpy(), ref_fs, f"noalloc final_state, call {call}")


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_ok):
    w = W.workload(3)  # 1712 chunk-heads: more than the fixed scratch holds
    shape = kda.KdaShape(1, w.B, w.Nqk, w.Nv, w.S, w.D)
    plan = kda.make_plan(shape, w.layout, w.cu_seqlens, device="cuda")
    assert 256 + plan.total_chunks * 148480 > (64 << 20)
    sh = W.shapes(w)
    z = lambda shape, dt=torch.bfloat16: torch.zeros(shape, dtype=dt, device="cuda")  # noqa: E731
    with pytest.raises(kda.KdaError) as e:
        kda.flash_kda_noalloc(z(sh["q"]), z(sh["q"]), z(sh["v"]), z(sh["v"]), z(sh["beta"]),
                              w.scale, None, z((w.Nv,), torch.float32),
                              z((w.Nv, w.D), torch.float32), w.lower_bound, w.layout, plan,
                              z(sh["v"]), z((w.B, w.Nv, w.D, w.D), torch.float32))
    assert e.value.name == "KDA_ERR_CAPACITY"

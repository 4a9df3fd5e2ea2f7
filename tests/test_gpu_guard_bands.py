"""Writes stay inside their buffers (a stand-in for a bounds checker, which this setup lacks).

out, final_state and the workspace are views into larger allocations whose guard bands, 8 KiB on
each side, hold a known byte pattern.  After the forward every guard byte must be unchanged, and
the results must equal those of a plain call with the same plan bit for bit (and the oracle within
atol = rtol = 5e-3).  Cases: a ragged packed batch (1-, 64- and 129-token sequences), a BSND GQA
varlen batch under the segmented schedule (the workspace then holds the segment states), and head
dim 64.
"""
import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, run_gpu, to_dev, valid_mask

pytestmark = pytest.mark.gpu

GUARD_BYTES = 8192   # a multiple of 256, so every view keeps the allocation's alignment
PATTERN = 0xA5


def guarded(numel: int, dtype, device):
    """(allocation, view of numel elements inside it, guard length in elements)."""
    esz = torch.empty(0, dtype=dtype).element_size()
    g = GUARD_BYTES // esz
    big = torch.empty(numel + 2 * g, dtype=dtype, device=device)
    big.view(torch.uint8).fill_(PATTERN)
    return big, big[g:g + numel], g


def guards_intact(big: torch.Tensor, g: int, numel: int) -> bool:
    raw = big.view(torch.uint8)
    esz = big.element_size()
    return bool((raw[:g * esz] == PATTERN).all()) and bool((raw[(g + numel) * esz:] == PATTERN).all())


CASES = [
    # name, layout, B, Nqk, Nv, S, lengths, lower_bound, D, segment_chunks
    ("tnd_ragged", "TND", 3, 1, 2, 64 + 1 + 129, [64, 1, 129], -5.0, 128, None),
    ("bsnd_gqa_segmented", "BSND", 2, 2, 4, 300, [300, 170], -1.0, 128, 2),
    ("bnsd_d64", "BNSD", 2, 1, 2, 200, [200, 77], -3.0, 64, None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_writes_stay_inside_their_buffers(case, cuda_ok):
    name, layout, B, Nqk, Nv, S, lengths, lb, D, seg = case
    w = W.custom(name, layout, B, Nqk, Nv, S, lengths, lower_bound=lb, scale=D ** -0.5,
                 init_state="normal", seed=61, D=D)
    inp = W.generate(w)
    d = to_dev(inp)
    cu = w.cu_seqlens if (layout == "TND" or any(L != S for L in lengths)) else None
    plan = kda.plan(d["q"], d["v"], d["initial_state"], layout, cu_seqlens=cu, segment_chunks=seg)
    if seg is not None:
        assert plan.segment_chunks == seg and plan.workspace_bytes > 256
    o_ref, fs_ref = run_gpu(w, inp, dev=d, plan=plan)

    n_out, n_fs = d["v"].numel(), B * Nv * D * D
    big_o, out, go = guarded(n_out, torch.bfloat16, d["v"].device)
    big_f, fs, gf = guarded(n_fs, torch.float32, d["v"].device)
    big_w, ws, gw = guarded(plan.workspace_bytes, torch.uint8, d["v"].device)
    kda.flash_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], w.scale, d["initial_state"],
                  d["A_log"], d["dt_bias"], lb, layout, plan, out=out.view(d["v"].shape),
                  final_state=fs.view(B, Nv, D, D), workspace=ws)
    kda.device_status(ws)
    torch.cuda.synchronize()
    assert guards_intact(big_o, go, n_out), "write outside out"
    assert guards_intact(big_f, gf, n_fs), "write outside final_state"
    assert guards_intact(big_w, gw, plan.workspace_bytes), "write outside the workspace"

    o = out.view(d["v"].shape).float().cpu().numpy()
    f = fs.view(B, Nv, D, D).cpu().numpy()
    assert np.array_equal(o.view(np.uint32), o_ref.view(np.uint32))
    assert np.array_equal(f.view(np.uint32), fs_ref.view(np.uint32))
    r_out, r_fs, _ = oracle.flash_kda(inp, layout, B, Nqk, Nv, S, D, w.scale, lb, cu)
    m = valid_mask(w, o.shape)
    compare(o[m], r_out[m], f"{name} out")
    compare(f, r_fs, f"{name} final_state")
    assert np.all(o[~m] == 0.0)

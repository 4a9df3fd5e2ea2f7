"""The chunk-parallel (segmented) schedule against the fp64 oracle.

Under a segmented plan a unit's chunks run as independent segments: per segment its affine map
S -> S M + R (from S = I with v = 0, and from S = 0), then the segment start states chained in
fp32, then every segment again from its true start state.  Results must match the oracle within
atol = rtol = 5e-3 for every segment length, including one-chunk segments, tails, varlen, GQA,
TND, and no decay (lower_bound = 0), where the identity run carries the whole history.
"""
import numpy as np
import pytest

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, run_gpu, to_dev, valid_mask

pytestmark = pytest.mark.gpu


def _plan(w, dev, seg):
    cu = w.cu_seqlens if (w.layout == "TND" or any(L != w.S for L in w.lengths)) else None
    return kda.plan(dev["q"], dev["v"], dev["initial_state"], w.layout, cu_seqlens=cu,
                    segment_chunks=seg)


CASES = [
    # name, layout, B, Nqk, Nv, S, lengths, lower_bound, init, segment_chunks
    ("one_unit_seg1", "BNSD", 1, 1, 1, 1000, [1000], -5.0, "normal", 1),
    ("one_unit_seg3", "BNSD", 1, 1, 1, 1000, [1000], -5.0, "normal", 3),
    ("one_unit_seg7", "BNSD", 1, 1, 1, 1000, [1000], -2.0, "zeros", 7),
    ("no_decay_seg4", "BNSD", 1, 1, 1, 2048, [2048], 0.0, "normal", 4),
    ("slow_decay_seg5", "BSND", 1, 1, 2, 3000, [3000], -0.1, "normal", 5),
    ("gqa_varlen_seg2", "BSND", 2, 2, 4, 700, [700, 300], -3.0, "normal", 2),
    ("tnd_seg3", "TND", 3, 1, 2, 130 + 500 + 64, [130, 500, 64], -5.0, "normal", 3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_segmented_parity(case, cuda_ok):
    name, layout, B, Nqk, Nv, S, lens, lb, init, seg = case
    w = W.custom(name, layout, B, Nqk, Nv, S, lens, lower_bound=lb, init_state=init, seed=53)
    inp = W.generate(w)
    dev = to_dev(inp)
    plan = _plan(w, dev, seg)
    assert plan.segment_chunks == seg
    o_g, fs_g = run_gpu(w, inp, dev=dev, plan=plan)
    o_r, fs_r, _ = oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                    w.lower_bound, w.cu_seqlens)
    m = valid_mask(w, o_g.shape)
    compare(o_g[m], o_r[m], f"{name} out")
    compare(fs_g, fs_r, f"{name} final_state")
    assert np.all(o_g[~m] == 0.0), "rows past a valid length must be zero"


def test_segmented_agrees_with_whole_units_and_is_deterministic(cuda_ok):
    w = W.workload(2)  # 3 units x 128 chunks: the default plan segments it
    inp = W.generate(w)
    dev = to_dev(inp)
    auto = _plan(w, dev, None)
    assert auto.segment_chunks > 0
    whole = _plan(w, dev, 0)
    o1, f1 = run_gpu(w, inp, dev=dev, plan=auto)
    o2, f2 = run_gpu(w, inp, dev=dev, plan=whole)
    o3, f3 = run_gpu(w, inp, dev=dev, plan=auto)
    compare(o1, o2, "segmented vs whole-unit out")
    compare(f1, f2, "segmented vs whole-unit final_state")
    assert np.array_equal(o1, o3) and np.array_equal(f1.view(np.uint32), f3.view(np.uint32))

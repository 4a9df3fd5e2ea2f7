"""CUDA path vs the fp64 oracle, element by element (atol = rtol = 5e-3), plus bookkeeping that
must be bit-exact (layouts, varlen packing, GQA, padding, chaining, determinism)."""
import os

import numpy as np
import pytest

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, run_gpu, to_dev, unit_rows, valid_mask

pytestmark = pytest.mark.gpu


def oracle_run(w, inp, units=None, form="chunked"):
    return oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale, w.lower_bound,
                            w.cu_seqlens, form=form, units=units)


def check_full(w, inp, form="chunked"):
    o_g, fs_g = run_gpu(w, inp)
    o_r, fs_r, _ = oracle_run(w, inp, form=form)
    m = valid_mask(w, o_g.shape)
    r1 = compare(o_g[m], o_r[m], f"{w.name} out")
    r2 = compare(fs_g, fs_r, f"{w.name} final_state")
    assert np.all(o_g[~m] == 0.0), "rows past a valid length must be zero"
    return r1, r2


@pytest.mark.parametrize("idx", [1, 2, 3])
def test_workload_full_parity(idx, cuda_ok):
    w = W.workload(idx)
    check_full(w, W.generate(w))


@pytest.mark.parametrize("idx", [4, 5, 7])
def test_workload_every_unit_parity(idx, cuda_ok):
    """Full-size run (the benchmarked launch) against the oracle on every (sequence, head) unit,
    element by element: out on every valid row and every final state.  The oracle runs its
    token-by-token form (pinned equal to the chunked form) on all host threads.  Workload 7 takes
    the segmented schedule by default, so this covers that schedule at full size."""
    w = W.workload(idx)
    inp = W.generate(w)
    o_g, fs_g = run_gpu(w, inp)
    res = oracle.run_units(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale, w.lower_bound,
                           w.cu_seqlens, form="recurrent", threads=os.cpu_count())
    assert len(res) == w.B * w.Nv
    for (b, h), (o_r, fs_r) in res.items():
        compare(unit_rows(w, o_g, b, h), o_r, f"{w.name} out ({b},{h})")
        compare(fs_g[b, h], fs_r, f"{w.name} final_state ({b},{h})")
    m = valid_mask(w, o_g.shape)
    assert np.all(o_g[~m] == 0.0)
    assert np.all(np.isfinite(o_g)) and np.all(np.isfinite(fs_g))


@pytest.mark.parametrize("idx", [4, 5, 7])
def test_workload_sampled_parity(idx, cuda_ok):
    """Quick variant of the above: the chunked oracle on a sample of whole units (first, last,
    longest and shortest sequence; first and last head)."""
    w = W.workload(idx)
    inp = W.generate(w)
    o_g, fs_g = run_gpu(w, inp)
    lens = np.array(w.lengths)
    bs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, w.B - 1})
    units = [(b, h) for b in bs for h in (0, w.Nv - 1)]
    res = oracle.run_units(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale, w.lower_bound,
                           w.cu_seqlens, units=units)
    for (b, h), (o_r, fs_r) in res.items():
        compare(unit_rows(w, o_g, b, h), o_r, f"{w.name} out ({b},{h})")
        compare(fs_g[b, h], fs_r, f"{w.name} final_state ({b},{h})")


SMALL = [
    # name, layout, B, Nqk, Nv, S, lengths, lower_bound, init
    ("len1", "BNSD", 1, 1, 1, 1, [1], -5.0, "normal"),
    ("len63", "BNSD", 1, 1, 2, 63, [63], -5.0, "normal"),
    ("len64", "BSND", 1, 2, 2, 64, [64], -3.0, "zeros"),
    ("len65", "BNSD", 1, 1, 1, 65, [65], -5.0, "normal"),
    ("len130_lb0", "BNSD", 1, 1, 1, 130, [130], 0.0, "normal"),
    ("len200_lb01", "BSND", 1, 1, 3, 200, [200], -0.1, "normal"),
    ("gqa_varlen", "BSND", 3, 2, 6, 150, [150, 1, 77], -2.0, "normal"),
    ("tnd_mix", "TND", 4, 1, 2, 64 + 1 + 129 + 300, [64, 1, 129, 300], -5.0, "normal"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c[0])
def test_small_cases_parity(case, cuda_ok):
    name, layout, B, Nqk, Nv, S, lens, lb, init = case
    w = W.custom(name, layout, B, Nqk, Nv, S, lens, lower_bound=lb, init_state=init, seed=17)
    inp = W.generate(w)
    check_full(w, inp)


@pytest.mark.parametrize("lb,S", [(0.0, 256), (0.0, 2048), (-0.1, 8192)])
def test_long_memory_stress(lb, S, cuda_ok):
    """No decay (lower_bound = 0) and slow decay over many chunks: rounding would pile up."""
    w = W.custom(f"stress{lb}_{S}", "BNSD", 1, 1, 1, S, [S], lower_bound=lb,
                 init_state="normal", seed=23)
    check_full(w, W.generate(w))


@pytest.mark.parametrize("D,lb,seg", [(128, -0.1, None), (128, 0.0, 0), (64, -0.5, None)])
def test_max_length_single_sequence(D, lb, seg, cuda_ok):
    """One 65,536-token sequence (the longest the FlashKDA README's constraints name), two heads:
    the planner's default (segmented) schedule and whole units, slow or no decay, D = 128 and
    64.  Every output row and the final state against the oracle."""
    w = W.custom(f"maxlen_{D}_{lb}_{seg}", "BSND", 1, 1, 2, 65536, [65536], lower_bound=lb,
                 scale=D ** -0.5, init_state="normal", seed=41, D=D)
    inp = W.generate(w)
    dev = to_dev(inp)
    plan = kda.plan(dev["q"], dev["v"], dev["initial_state"], "BSND", segment_chunks=seg)
    if seg is None:
        assert plan.segment_chunks > 0  # 2 units of 1024 chunks: the chunk-parallel schedule
    o_g, fs_g = run_gpu(w, inp, dev=dev, plan=plan)
    o_r, fs_r, _ = oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                    w.lower_bound, None)
    compare(o_g, o_r, f"{w.name} out")
    compare(fs_g, fs_r, f"{w.name} final_state")


def _same(a, b):
    return np.array_equal(a.view(np.uint32) if a.dtype == np.float32 else a,
                          b.view(np.uint32) if b.dtype == np.float32 else b)


def test_layouts_bit_exact(cuda_ok):
    w_bnsd = W.custom("x", "BNSD", 2, 2, 4, 200, [200, 130], lower_bound=-4.0, seed=31)
    inp = W.generate(w_bnsd)
    o1, f1 = run_gpu(w_bnsd, inp)
    inp_bsnd = dict(inp)
    for n in ("q", "k", "v", "g"):
        inp_bsnd[n] = np.ascontiguousarray(inp[n].transpose(0, 2, 1, 3))
    inp_bsnd["beta"] = np.ascontiguousarray(inp["beta"].transpose(0, 2, 1))
    w_bsnd = W.custom("x", "BSND", 2, 2, 4, 200, [200, 130], lower_bound=-4.0, seed=31)
    o2, f2 = run_gpu(w_bsnd, inp_bsnd)
    assert _same(o2.transpose(0, 2, 1, 3), o1) and _same(f2, f1)
    inp_tnd = dict(inp)
    for n in ("q", "k", "v", "g", "beta"):
        inp_tnd[n] = np.concatenate([inp_bsnd[n][b, :L] for b, L in enumerate([200, 130])])
    w_tnd = W.custom("x", "TND", 2, 2, 4, 330, [200, 130], lower_bound=-4.0, seed=31)
    o3, f3 = run_gpu(w_tnd, inp_tnd)
    assert _same(o3[:200], o2[0, :200]) and _same(o3[200:], o2[1, :130]) and _same(f3, f1)


def test_varlen_equals_separate_calls_bit_exact(cuda_ok):
    lens = [100, 64, 3]
    w = W.custom("v", "TND", 3, 1, 2, sum(lens), lens, lower_bound=-5.0, seed=41)
    inp = W.generate(w)
    o, f = run_gpu(w, inp)
    cu = w.cu_seqlens
    for b, L in enumerate(lens):
        one = {n: inp[n][cu[b]:cu[b + 1]] for n in ("q", "k", "v", "g", "beta")}
        one.update(A_log=inp["A_log"], dt_bias=inp["dt_bias"],
                   initial_state=inp["initial_state"][b:b + 1])
        w1 = W.custom("v1", "TND", 1, 1, 2, L, [L], lower_bound=-5.0, seed=41)
        o1, f1 = run_gpu(w1, one)
        assert _same(o1, o[cu[b]:cu[b + 1]]) and _same(f1[0], f[b])


def test_gqa_equals_repeated_heads_bit_exact(cuda_ok):
    w = W.custom("g", "BNSD", 1, 2, 6, 100, [100], lower_bound=-5.0, seed=43)
    inp = W.generate(w)
    o, f = run_gpu(w, inp)
    rep = dict(inp)
    rep["q"] = np.repeat(inp["q"], 3, axis=1)
    rep["k"] = np.repeat(inp["k"], 3, axis=1)
    w2 = W.custom("g2", "BNSD", 1, 6, 6, 100, [100], lower_bound=-5.0, seed=43)
    o2, f2 = run_gpu(w2, rep)
    assert _same(o, o2) and _same(f, f2)


def test_padding_never_read_bit_exact(cuda_ok):
    w = W.custom("p", "BNSD", 2, 1, 2, 160, [160, 70], lower_bound=-5.0, seed=47)
    o1, f1 = run_gpu(w, W.generate(w))
    o2, f2 = run_gpu(w, W.generate(w, pad_value=float("nan")))
    assert _same(o1, o2) and _same(f1, f2)
    assert np.all(o2[1, :, 70:] == 0.0)


def test_chaining_through_final_state_bit_exact(cuda_ok):
    """Two calls split at a chunk boundary == one call (the state is passed in fp32)."""
    S, split = 320, 128
    w = W.custom("c", "BNSD", 1, 1, 2, S, [S], lower_bound=-1.0, seed=53)
    inp = W.generate(w)
    o, f = run_gpu(w, inp)
    a = dict(inp)
    b = dict(inp)
    for n in ("q", "k", "v", "g", "beta"):
        a[n] = np.ascontiguousarray(inp[n][:, :, :split])
        b[n] = np.ascontiguousarray(inp[n][:, :, split:])
    wa = W.custom("ca", "BNSD", 1, 1, 2, split, [split], lower_bound=-1.0, seed=53)
    oa, fa = run_gpu(wa, a)
    b["initial_state"] = fa
    wb = W.custom("cb", "BNSD", 1, 1, 2, S - split, [S - split], lower_bound=-1.0, seed=53)
    ob, fb = run_gpu(wb, b)
    assert _same(np.concatenate([oa, ob], axis=2), o) and _same(fb, f)


def test_zero_initial_state_equals_null_and_determinism(cuda_ok):
    w = W.custom("z", "BSND", 1, 1, 2, 130, [130], lower_bound=-5.0, init_state="zeros", seed=59)
    inp = W.generate(w)
    o1, f1 = run_gpu(w, inp)
    o2, f2 = run_gpu(w, inp, with_init=False)
    o3, f3 = run_gpu(w, inp)
    assert _same(o1, o2) and _same(f1, f2) and _same(o1, o3) and _same(f1, f3)


def test_plan_mismatch_reported_by_device(cuda_ok):
    """A device plan that differs from the host plan is caught by the kernels, not used."""
    w = W.workload(1)
    inp = W.generate(w)
    dev = to_dev(inp)
    p = kda.plan(dev["q"], dev["v"], dev["initial_state"], "BNSD")
    p.dev[15] += 1  # corrupt the device copy's checksum word only
    kda.flash_kda(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], w.scale,
                  dev["initial_state"], dev["A_log"], dev["dt_bias"], w.lower_bound, "BNSD", p)
    with pytest.raises(kda.KdaError) as e:
        kda.device_status(p.workspace())
    assert e.value.name == "KDA_ERR_PLAN"

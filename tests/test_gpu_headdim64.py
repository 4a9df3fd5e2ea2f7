"""Head dim D = 64 (Dk = Dv = 64) against the fp64 oracle at D = 64.

The FlashKDA README (约束说明) fixes D = 128; FLA PR 656 ("[kda] add recursive block intra",
summary and timing table) benchmarks K = 64 heads beside K = 128.  The library runs a D = 64
problem through its D = 128 kernels with the upper 64 channels of q, k, v, g read as zeros, so
these tests check the things that differ: tensor maps that end at D, dt_bias and states indexed
with row length D, output and final-state stores bounded by D, the zero padding rows, the
segmented schedule's 128 x 128 state slots around D x D states, and the decode step at D = 64.
The oracle runs at D = 64 throughout (it knows nothing of the padding).  Tolerance: atol = rtol
= 5e-3, as for D = 128.
"""
import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, run_gpu, to_dev, valid_mask

pytestmark = pytest.mark.gpu

D = 64
SCALE64 = D ** -0.5


def _plan(w, dev, seg=None):
    cu = w.cu_seqlens if (w.layout == "TND" or any(L != w.S for L in w.lengths)) else None
    return kda.plan(dev["q"], dev["v"], dev["initial_state"], w.layout, cu_seqlens=cu,
                    segment_chunks=seg)


CASES = [
    # name, layout, B, Nqk, Nv, S, lengths, lower_bound, init, segment_chunks
    ("d64_bnsd_tail", "BNSD", 1, 2, 2, 300, [300], -5.0, "normal", None),
    ("d64_bsnd_gqa_varlen", "BSND", 2, 2, 4, 500, [500, 203], -3.0, "normal", None),
    ("d64_tnd", "TND", 3, 1, 2, 130 + 64 + 257, [130, 64, 257], -5.0, "zeros", None),
    ("d64_no_decay", "BNSD", 1, 1, 1, 640, [640], 0.0, "normal", None),
    ("d64_one_token", "BSND", 1, 1, 1, 1, [1], -5.0, "normal", None),
    ("d64_segmented", "BNSD", 1, 1, 2, 1000, [1000], -2.0, "normal", 3),
    ("d64_segmented_varlen", "BSND", 2, 1, 2, 700, [700, 300], -0.5, "normal", 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_headdim64_parity(case, cuda_ok):
    name, layout, B, Nqk, Nv, S, lens, lb, init, seg = case
    w = W.custom(name, layout, B, Nqk, Nv, S, lens, lower_bound=lb, scale=SCALE64,
                 init_state=init, seed=71, D=D)
    inp = W.generate(w)
    dev = to_dev(inp)
    plan = _plan(w, dev, seg)
    assert plan.shape.D == D
    if seg is not None:
        assert plan.segment_chunks == seg
    o_g, fs_g = run_gpu(w, inp, dev=dev, plan=plan)
    assert o_g.shape[-1] == D and fs_g.shape[-2:] == (D, D)
    o_r, fs_r, _ = oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                    w.lower_bound, w.cu_seqlens)
    m = valid_mask(w, o_g.shape)
    compare(o_g[m], o_r[m], f"{name} out")
    compare(fs_g, fs_r, f"{name} final_state")
    assert np.all(o_g[~m] == 0.0), "rows past a valid length must be zero"


def test_headdim64_pages_shape_sampled_units(cuda_ok):
    """The pages' K = 64 shape B=1, T=8192, H=32 (FLA PR 656 timing table), BNSD, run whole on
    the GPU; the oracle checks two sampled heads in full (every token and the final state)."""
    w = W.custom("d64_b1_t8192_h32", "BNSD", 1, 32, 32, 8192, [8192], lower_bound=-5.0,
                 scale=SCALE64, init_state="normal", seed=72, D=D)
    inp = W.generate(w)
    o_g, fs_g = run_gpu(w, inp)
    units = [(0, 5), (0, 30)]
    o_r, fs_r, done = oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                       w.lower_bound, units=units)
    assert sorted(done) == sorted(units)
    for b, h in units:
        compare(o_g[b, h], o_r[b, h], f"out unit {(b, h)}")
        compare(fs_g[b, h], fs_r[b, h], f"final_state unit {(b, h)}")
    assert np.all(np.isfinite(o_g)) and np.all(np.isfinite(fs_g))


def _bits(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def _dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("lb", [-5.0, 0.0])
def test_decode_headdim64_matches_oracle(lb, cuda_ok):
    rng = np.random.default_rng(73)
    B, Nqk, Nv = 2, 2, 4
    x = {"q": _bits(rng, (B, Nqk, D)), "k": _bits(rng, (B, Nqk, D)), "v": _bits(rng, (B, Nv, D)),
         "g": _bits(rng, (B, Nv, D)), "beta": _bits(rng, (B, Nv))}
    A_log = rng.standard_normal(Nv).astype(np.float32)
    dt_bias = rng.standard_normal((Nv, D)).astype(np.float32)
    S0 = (0.5 * rng.standard_normal((B, Nv, D, D))).astype(np.float32)
    out, S1 = kda.decode(*(_dev_bits(x[n]) for n in ("q", "k", "v", "g", "beta")), SCALE64,
                         torch.from_numpy(S0).cuda(), torch.from_numpy(A_log).cuda(),
                         torch.from_numpy(dt_bias).cuda(), lb)
    torch.cuda.synchronize()
    G = Nv // Nqk
    w = oracle.widen_bf16
    for b in range(B):
        for h in range(Nv):
            o, S = oracle.unit(w(x["q"][b, h // G])[None], w(x["k"][b, h // G])[None],
                               w(x["v"][b, h])[None], w(x["g"][b, h])[None],
                               w(x["beta"][b, h:h + 1]), dt_bias[h].astype(np.float64),
                               float(A_log[h]), lb, SCALE64, S0[b, h].astype(np.float64),
                               form="recurrent")
            compare(out[b, h].float().cpu().numpy(), o[0], f"decode out {(b, h)}")
            compare(S1[b, h].cpu().numpy(), S, f"decode state {(b, h)}")


def test_prefill_then_decode_headdim64(cuda_ok):
    """kda_forward over L tokens then T decode steps == the oracle over L + T tokens, D = 64."""
    L, T, lb = 150, 4, -1.0
    w = W.custom("d64_chain", "BSND", 2, 1, 2, L + T, [L + T, L + T], lower_bound=lb,
                 scale=SCALE64, init_state="normal", seed=74, D=D)
    inp = W.generate(w)
    d = to_dev(inp)
    pre = {n: d[n][:, :L].contiguous() for n in ("q", "k", "v", "g", "beta")}
    plan = kda.plan(pre["q"], pre["v"], d["initial_state"], "BSND")
    _, state = kda.flash_kda(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"], w.scale,
                             d["initial_state"], d["A_log"], d["dt_bias"], lb, "BSND", plan)
    outs = []
    for t in range(L, L + T):
        step = [d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")]
        o, state = kda.decode(*step, w.scale, state, d["A_log"], d["dt_bias"], lb,
                              state_out=state)
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    ref_out, ref_fs, _ = oracle.flash_kda(inp, "BSND", w.B, w.Nqk, w.Nv, w.S, w.D, w.scale, lb,
                                          form="recurrent")
    for i, t in enumerate(range(L, L + T)):
        compare(outs[i], ref_out[:, t], f"decode out at token {t}")
    compare(state.cpu().numpy(), ref_fs, "state after prefill + decode")

"""Context parallelism on the GPU: kda_state_chain, kda_forward_summary and the whole schedule.

- ``kda_state_chain`` against its definition (S <- S M_j + R_j folded in fp64 here), for 0, 1
  and 5 steps, packed and interleaved ([M; R] pairs) map layouts, in place, D = 128 and 64.
- ``kda_forward_summary``: the maps (M, R) of a span must carry any start state S0 to the
  span's end state: S0 M + R equals the oracle's final state from S0 (atol = rtol = 5e-3).
- ``flash_kda_context_parallel`` with its ranks run one after another in one process (the
  exchange is the stacked summaries, what the all-gather delivers): the spans' outputs and the
  last span's state equal the oracle over the whole sequence, BNSD and BSND with GQA, D = 128
  and 64.  Ranks never wait on one another, so one GPU runs them safely.
"""
import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("n", [0, 1, 5])
@pytest.mark.parametrize("interleaved", [False, True])
def test_state_chain_matches_definition(D, n, interleaved, cuda_ok):
    rng = np.random.default_rng(200 + D + n)
    B, Nv = 2, 3
    S0 = rng.standard_normal((B, Nv, D, D)).astype(np.float32)
    # maps of the kind a span produces: a contraction plus a rank-limited correction
    Ms = (0.9 * np.eye(D) + 0.02 * rng.standard_normal((n, B, Nv, D, D))).astype(np.float32)
    Rs = (0.1 * rng.standard_normal((n, B, Nv, D, D))).astype(np.float32)
    if interleaved:
        buf = torch.from_numpy(np.stack([Ms, Rs], axis=1).copy()).cuda()  # [n, 2, B, Nv, D, D]
        M, R = buf[:, 0], buf[:, 1]
    else:
        M, R = torch.from_numpy(Ms).cuda(), torch.from_numpy(Rs).cuda()
    S_in = torch.from_numpy(S0).cuda()
    got = kda.state_chain(S_in, M, R)
    ref = S0.astype(np.float64)
    for j in range(n):
        ref = ref @ Ms[j].astype(np.float64) + Rs[j]
    torch.cuda.synchronize()
    np.testing.assert_allclose(got.cpu().numpy(), ref, rtol=1e-4, atol=1e-4)
    # in place, and from zeros
    S_io = S_in.clone()
    kda.state_chain(S_io, M, R, S_out=S_io)
    z = kda.state_chain(None, M, R)
    refz = np.zeros_like(ref)
    for j in range(n):
        refz = refz @ Ms[j].astype(np.float64) + Rs[j]
    torch.cuda.synchronize()
    assert torch.equal(S_io, got)
    np.testing.assert_allclose(z.cpu().numpy(), refz, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("D,layout,lb", [(128, "BNSD", -5.0), (128, "BSND", 0.0), (64, "BNSD", -2.0)])
def test_summary_carries_any_start_state(D, layout, lb, cuda_ok):
    w = W.custom(f"sum_{D}_{layout}", layout, 2, 1, 2, 300, [300, 300], lower_bound=lb,
                 scale=D ** -0.5, init_state="normal", seed=210, D=D)
    inp = W.generate(w)
    d = to_dev(inp)
    plan = kda.plan(d["q"], d["v"], d["initial_state"], layout)
    M, R = kda.forward_summary(d["q"], d["k"], d["v"], d["g"], d["beta"], d["A_log"],
                               d["dt_bias"], lb, layout, plan)
    kda.device_status(plan.workspace())
    torch.cuda.synchronize()
    S0 = inp["initial_state"].astype(np.float64)
    pred = np.einsum("bhij,bhjk->bhik", S0, M.cpu().numpy().astype(np.float64)) + \
        R.cpu().numpy()
    _, ref_fs, _ = oracle.flash_kda(inp, layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale, lb)
    compare(pred, ref_fs, "S0 M + R vs the oracle's final state")
    # R alone is the end state from zero
    inp0 = dict(inp, initial_state=np.zeros_like(inp["initial_state"]))
    _, ref0, _ = oracle.flash_kda(inp0, layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale, lb)
    compare(R.cpu().numpy(), ref0, "R vs the oracle's final state from zero")


@pytest.mark.parametrize("seg", [0, 1, 2, 3])
def test_summary_segmented_composition(seg, cuda_ok):
    """Segment maps composed into unit maps (segments of 1-3 chunks, units of 6 and 3 chunks
    with tails; 0 = whole units) carry S0 to the oracle's final state."""
    w = W.custom(f"sum_seg{seg}", "BSND", 2, 1, 2, 350, [350, 170], lower_bound=-0.5,
                 init_state="normal", seed=230 + seg)
    inp = W.generate(w)
    d = to_dev(inp)
    cu = w.cu_seqlens
    plan = kda.plan(d["q"], d["v"], d["initial_state"], "BSND", cu_seqlens=cu,
                    segment_chunks=seg)
    assert plan.segment_chunks == seg
    M, R = kda.forward_summary(d["q"], d["k"], d["v"], d["g"], d["beta"], d["A_log"],
                               d["dt_bias"], w.lower_bound, "BSND", plan)
    kda.device_status(plan.workspace())
    torch.cuda.synchronize()
    S0 = inp["initial_state"].astype(np.float64)
    pred = np.einsum("bhij,bhjk->bhik", S0, M.cpu().numpy().astype(np.float64)) + \
        R.cpu().numpy()
    _, ref_fs, _ = oracle.flash_kda(inp, "BSND", w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                    w.lower_bound, cu)
    compare(pred, ref_fs, f"segments of {seg}: S0 M + R vs the oracle's final state")


def _span(dev, layout, r, s_loc):
    sl = slice(r * s_loc, (r + 1) * s_loc)
    out = {}
    for n in ("q", "k", "v", "g", "beta"):
        t = dev[n]
        out[n] = (t[:, :, sl] if layout == "BNSD" else t[:, sl]).contiguous()
    return out


@pytest.mark.parametrize("world,layout,Nqk,Nv,D,s_loc", [
    (4, "BNSD", 1, 2, 128, 320),
    (3, "BSND", 2, 4, 128, 200),
    (2, "BNSD", 1, 3, 64, 512),
])
def test_context_parallel_ranks_in_sequence(world, layout, Nqk, Nv, D, s_loc, cuda_ok):
    S = world * s_loc
    w = W.custom(f"cp_{world}_{layout}_{D}", layout, 1, Nqk, Nv, S, [S], lower_bound=-1.0,
                 scale=D ** -0.5, init_state="normal", seed=220 + world, D=D)
    inp = W.generate(w)
    d = to_dev(inp)
    spans = [_span(d, layout, r, s_loc) for r in range(world)]
    plans = [kda.plan(sp["q"], sp["v"], d["initial_state"], layout) for sp in spans]
    # what the all-gather delivers: [world, 2, B, Nv, D, D], the last rank's pair zero
    gathered = torch.zeros((world, 2, w.B, w.Nv, D, D), dtype=torch.float32, device="cuda")
    for r in range(world - 1):
        sp = spans[r]
        kda.forward_summary(sp["q"], sp["k"], sp["v"], sp["g"], sp["beta"], d["A_log"],
                            d["dt_bias"], w.lower_bound, layout, plans[r], M=gathered[r, 0],
                            R=gathered[r, 1])
    outs, state = [], None
    for r in range(world):
        sp = spans[r]
        o, state = kda.flash_kda_context_parallel(
            sp["q"], sp["k"], sp["v"], sp["g"], sp["beta"], w.scale, d["initial_state"],
            d["A_log"], d["dt_bias"], w.lower_bound, layout, plans[r], rank=r, world=world,
            exchange=lambda local: gathered)
        outs.append(o.float().cpu().numpy())
    kda.device_status(plans[-1].workspace())
    torch.cuda.synchronize()
    o_g = np.concatenate(outs, axis=2 if layout == "BNSD" else 1)
    ref_out, ref_fs, _ = oracle.flash_kda(inp, layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                          w.lower_bound)
    compare(o_g, ref_out, "context-parallel out")
    compare(state.cpu().numpy(), ref_fs, "context-parallel final state (last rank)")

"""The single-token decode step (kda_decode) against the fp64 oracle's recurrence.

A decode step is one token of the recurrence per (sequence, value head), with the same in-op
activations as the prefill.  The oracle runs its token-by-token recurrence (the definition) on
the same bf16 inputs; out and state must agree within atol = rtol = 5e-3.  The step that
follows a prefill is checked by chaining: kda_forward over L tokens, then T decode steps, must
equal the oracle over L + T tokens.
"""
import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda
import kda_workloads as W
import oracle
from kda_gpu import compare, to_dev

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, std=1.0):
    return W.f32_to_bf16_bits((std * rng.standard_normal(shape)).astype(np.float32))


def _step_inputs(rng, B, Nqk, Nv):
    return {"q": _bf16(rng, (B, Nqk, 128)), "k": _bf16(rng, (B, Nqk, 128)),
            "v": _bf16(rng, (B, Nv, 128)), "g": _bf16(rng, (B, Nv, 128)),
            "beta": _bf16(rng, (B, Nv))}


def _dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _oracle_step(x, A_log, dt_bias, S0, lb, scale, B, Nqk, Nv):
    """One recurrence step per (b, h) in fp64 (the oracle's token-by-token form)."""
    G = Nv // Nqk
    out = np.zeros((B, Nv, 128))
    S1 = np.zeros((B, Nv, 128, 128))
    for b in range(B):
        for h in range(Nv):
            w = oracle.widen_bf16
            o, S = oracle.unit(w(x["q"][b, h // G])[None], w(x["k"][b, h // G])[None],
                               w(x["v"][b, h])[None], w(x["g"][b, h])[None],
                               w(x["beta"][b, h:h + 1]), dt_bias[h].astype(np.float64),
                               float(A_log[h]), lb, scale, S0[b, h].astype(np.float64),
                               form="recurrent")
            out[b, h], S1[b, h] = o[0], S
    return out, S1


@pytest.mark.parametrize("B,Nqk,Nv,lb", [(3, 2, 4, -5.0), (2, 1, 3, 0.0), (1, 4, 4, -0.1)])
def test_decode_step_matches_oracle(B, Nqk, Nv, lb, cuda_ok):
    rng = np.random.default_rng(100 + B + Nv)
    x = _step_inputs(rng, B, Nqk, Nv)
    A_log = rng.standard_normal(Nv).astype(np.float32)
    dt_bias = rng.standard_normal((Nv, 128)).astype(np.float32)
    S0 = (0.5 * rng.standard_normal((B, Nv, 128, 128))).astype(np.float32)
    scale = 128 ** -0.5
    out, S1 = kda.decode(*(_dev_bits(x[n]) for n in ("q", "k", "v", "g", "beta")), scale,
                         torch.from_numpy(S0).cuda(), torch.from_numpy(A_log).cuda(),
                         torch.from_numpy(dt_bias).cuda(), lb)
    torch.cuda.synchronize()
    ref_out, ref_S = _oracle_step(x, A_log, dt_bias, S0, lb, scale, B, Nqk, Nv)
    compare(out.float().cpu().numpy(), ref_out, "decode out")
    compare(S1.cpu().numpy(), ref_S, "decode state")


def test_decode_in_place_and_zero_state(cuda_ok):
    rng = np.random.default_rng(7)
    B, Nqk, Nv = 2, 2, 4
    x = {n: _dev_bits(a) for n, a in _step_inputs(rng, B, Nqk, Nv).items()}
    A_log = torch.from_numpy(rng.standard_normal(Nv).astype(np.float32)).cuda()
    dt = torch.from_numpy(rng.standard_normal((Nv, 128)).astype(np.float32)).cuda()
    S0 = torch.from_numpy(rng.standard_normal((B, Nv, 128, 128)).astype(np.float32)).cuda()
    args = [x[n] for n in ("q", "k", "v", "g", "beta")]
    o1, S1 = kda.decode(*args, 0.1, S0, A_log, dt, -3.0)
    S_inplace = S0.clone()
    o2, S2 = kda.decode(*args, 0.1, S_inplace, A_log, dt, -3.0, state_out=S_inplace)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S_inplace.data_ptr()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)  # in place == out of place, bit for bit
    z = torch.zeros_like(S0)
    o3, S3 = kda.decode(*args, 0.1, None, A_log, dt, -3.0)
    o4, S4 = kda.decode(*args, 0.1, z, A_log, dt, -3.0)
    torch.cuda.synchronize()
    assert torch.equal(o3, o4) and torch.equal(S3, S4)  # no state == zero state


@pytest.mark.parametrize("lb", [-5.0, -0.1])
def test_prefill_then_decode_equals_longer_prefill(lb, cuda_ok):
    """kda_forward over L tokens, then T decode steps from its final_state == the oracle over
    L + T tokens (the decode outputs are the last T rows, the state is the final state)."""
    L, T = 200, 5
    w = W.custom("chain", "BSND", 2, 2, 4, L + T, [L + T, L + T], lower_bound=lb,
                 init_state="normal", seed=31)
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

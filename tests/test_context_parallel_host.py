"""Context parallelism, host side: the rank bookkeeping over real gloo process groups on CPU.

``flash_kda_context_parallel`` orders library calls around one all-gather (its module
docstring).  Here the three library calls are replaced by fp64 stand-ins built on the oracle
(the summary from the oracle's recurrence from S = I with v = 0 and from S = 0; the fold as the
plain matrix recurrence; the forward as the oracle from the given start state), so what is
checked is the schedule itself: which ranks summarise, that the last rank contributes nothing,
the order of the gathered maps, which of them each rank folds, and that the spans' outputs and
the last rank's state equal the oracle over the whole sequence.  World sizes 2, 3 and 4
(the last with GQA groups of 2).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import chunked_kda_prefill_b200 as kda  # noqa: E402
import kda_workloads as W  # noqa: E402
import oracle  # noqa: E402

S_LOC = 100  # tokens per rank (a partial last chunk inside every span)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(world, layout, Nqk=1, Nv=2):
    return W.custom(f"cp_{layout}_{world}", layout, 2, Nqk, Nv, world * S_LOC,
                    [world * S_LOC] * 2, lower_bound=-1.0, init_state="normal", seed=90 + world)


def _span(inp, layout, r):
    """Rank r's tokens of every sequence (bf16 bit arrays), as contiguous arrays."""
    sl = slice(r * S_LOC, (r + 1) * S_LOC)
    out = {}
    for n in ("q", "k", "v", "g"):
        a = inp[n]
        out[n] = np.ascontiguousarray(a[:, :, sl] if layout == "BNSD" else a[:, sl])
    b = inp["beta"]
    out["beta"] = np.ascontiguousarray(b[:, :, sl] if layout == "BNSD" else b[:, sl])
    return out


class OracleOps:
    """fp64 stand-ins for the library calls (CPU tensors carry bf16 bits as int16)."""

    layout = "BNSD"
    Nqk = 1

    @classmethod
    def _units(cls, q, k, v, g, beta, A_log, dt_bias, lb, scale, starts, zero_v=False):
        bits = lambda t: t.numpy().view(np.uint16)  # noqa: E731
        qb, kb, vb, gb, bb = (bits(t) for t in (q, k, v, g, beta))
        B = qb.shape[0]
        Nv = vb.shape[1] if cls.layout == "BNSD" else vb.shape[2]
        G = Nv // cls.Nqk
        w = oracle.widen_bf16
        outs, states = {}, {}
        for b in range(B):
            for h in range(Nv):
                pick = (lambda a, hh: a[b, hh]) if cls.layout == "BNSD" else \
                    (lambda a, hh: a[b, :, hh])
                vv = w(pick(vb, h))
                o, S = oracle.unit(w(pick(qb, h // G)), w(pick(kb, h // G)),
                                   np.zeros_like(vv) if zero_v else vv, w(pick(gb, h)),
                                   w(pick(bb, h)), dt_bias[h].numpy().astype(np.float64),
                                   float(A_log[h]), lb, scale, starts(b, h), form="recurrent")
                outs[(b, h)], states[(b, h)] = o, S
        return outs, states, B, Nv

    @classmethod
    def summary(cls, q, k, v, g, beta, A_log, dt_bias, lb, layout, plan, M, R):
        D = M.shape[-1]
        _, Ms, B, Nv = cls._units(q, k, v, g, beta, A_log, dt_bias, lb, 1.0,
                                  lambda b, h: np.eye(D), zero_v=True)
        _, Rs, _, _ = cls._units(q, k, v, g, beta, A_log, dt_bias, lb, 1.0,
                                 lambda b, h: np.zeros((D, D)))
        for b in range(B):
            for h in range(Nv):
                M[b, h] = torch.from_numpy(Ms[(b, h)])
                R[b, h] = torch.from_numpy(Rs[(b, h)])
        cls.calls.append("summary")
        return M, R

    @classmethod
    def chain(cls, S_in, M, R):
        S = (torch.zeros_like(M[0]) if S_in is None else S_in).double()
        for j in range(M.shape[0]):
            S = S @ M[j].double() + R[j].double()
        cls.calls.append(f"chain{M.shape[0]}")
        return S.float()

    @classmethod
    def forward(cls, q, k, v, g, beta, scale, S0, A_log, dt_bias, lb, layout, plan):
        D = q.shape[-1]
        st = (lambda b, h: np.zeros((D, D))) if S0 is None else \
            (lambda b, h: S0[b, h].double().numpy())
        outs, states, B, Nv = cls._units(q, k, v, g, beta, A_log, dt_bias, lb, scale, st)
        L = q.shape[2] if layout == "BNSD" else q.shape[1]
        out = np.zeros((B, Nv, L, D) if layout == "BNSD" else (B, L, Nv, D))
        fs = np.zeros((B, Nv, D, D))
        for (b, h), o in outs.items():
            if layout == "BNSD":
                out[b, h] = o
            else:
                out[b, :, h] = o
            fs[b, h] = states[(b, h)]
        cls.calls.append("forward")
        return torch.from_numpy(out), torch.from_numpy(fs)


def _worker(rank, world, port, layout, path, Nqk, Nv):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        w = _workload(world, layout, Nqk, Nv)
        inp = W.generate(w)
        sp = _span(inp, layout, rank)
        t = {n: torch.from_numpy(a.view(np.int16)) for n, a in sp.items()}
        shape = kda.KdaShape(kda.LAYOUTS[layout], w.B, w.Nqk, w.Nv, S_LOC, w.D)
        plan = kda.make_plan(shape, layout)
        OracleOps.layout, OracleOps.Nqk, OracleOps.calls = layout, w.Nqk, []
        out, fs = kda.flash_kda_context_parallel(
            t["q"], t["k"], t["v"], t["g"], t["beta"], w.scale,
            torch.from_numpy(inp["initial_state"]), torch.from_numpy(inp["A_log"]),
            torch.from_numpy(inp["dt_bias"]), w.lower_bound, layout, plan, ops=OracleOps)
        np.savez(f"{path}.{rank}.npz", out=out.numpy(), fs=fs.numpy(),
                 calls=np.array(OracleOps.calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,Nqk,Nv", [(2, "BNSD", 1, 2), (3, "BSND", 1, 2),
                                                 (4, "BSND", 2, 4)])
def test_context_parallel_schedule_gloo(world, layout, Nqk, Nv, tmp_path):
    path = str(tmp_path / "cp")
    mp.spawn(_worker, args=(world, _free_port(), layout, path, Nqk, Nv), nprocs=world, join=True)
    w = _workload(world, layout, Nqk, Nv)
    inp = W.generate(w)
    ref_out, ref_fs, _ = oracle.flash_kda(inp, layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                          w.lower_bound, form="recurrent")
    for r in range(world):
        d = np.load(f"{path}.{r}.npz")
        calls = list(d["calls"])
        expect = (["summary"] if r < world - 1 else []) + ([f"chain{r}"] if r > 0 else []) + \
            ["forward"]
        assert calls == expect, (r, calls)
        sl = slice(r * S_LOC, (r + 1) * S_LOC)
        ref = ref_out[:, :, sl] if layout == "BNSD" else ref_out[:, sl]
        # (the exchanged maps are fp32, so agreement is to fp32 rounding, not fp64)
        np.testing.assert_allclose(d["out"], ref, rtol=1e-5, atol=1e-5)
        if r == world - 1:
            np.testing.assert_allclose(d["fs"], ref_fs, rtol=1e-5, atol=1e-5)


def test_single_rank_is_one_forward():
    OracleOps.calls = []
    w = W.custom("cp_single", "BNSD", 1, 1, 1, 70, [70], init_state="normal", seed=97)
    inp = W.generate(w)
    t = {n: torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16))
         for n in ("q", "k", "v", "g", "beta")}
    shape = kda.KdaShape(0, 1, 1, 1, 70, 128)
    plan = kda.make_plan(shape, "BNSD")
    OracleOps.layout, OracleOps.Nqk = "BNSD", 1
    kda.flash_kda_context_parallel(t["q"], t["k"], t["v"], t["g"], t["beta"], w.scale, None,
                                   torch.from_numpy(inp["A_log"]),
                                   torch.from_numpy(inp["dt_bias"]), w.lower_bound, "BNSD", plan,
                                   ops=OracleOps)
    assert OracleOps.calls == ["forward"]


def test_rejects_packed_layout_and_bad_rank():
    with pytest.raises(ValueError):
        kda.flash_kda_context_parallel(None, None, None, None, None, 1.0, None, None, None, -1.0,
                                       "TND", None)
    shape = kda.KdaShape(0, 1, 1, 1, 64, 128)
    plan = kda.make_plan(shape, "BNSD")
    with pytest.raises(ValueError):
        kda.flash_kda_context_parallel(None, None, None, None, None, 1.0, None, None, None, -1.0,
                                       "BNSD", plan, rank=2, world=2, ops=OracleOps)

"""The interface the FlashKDA README fixes (参数说明, 返回值说明, 约束说明, 快速开始), stored as
data in ``tests/golden/flash_kda_io_contract.txt``, against the binding, the input generator, the
library's host checks and the oracle's layout walker.

The oracle check is a pin in its own right: one nonzero state entry S0[a, b] (a != b), a query
that is the unit vector e_b at one token, keys orthogonal to e_b, no values and no decay
(lower_bound = 0).  The delta rule then leaves the state alone, and the output at that token is
scale * S0 e_b = scale * e_a.  It must appear at the place the contract's shape table gives for
that (sequence, head, token) in each layout, in channel a and not b: a walker that transposed the
state (Dk, Dv instead of the contract's Dv, Dk) or read a layout's axes in another order fails.
"""
import math
import os

import numpy as np
import pytest

import chunked_kda_prefill_b200 as kda
from chunked_kda_prefill_b200 import api
from chunked_kda_prefill_b200._lib import KdaShape
import kda_workloads as W
import oracle
from test_abi import _fwd, _plan, _shape, gpu_visible

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "flash_kda_io_contract.txt")


def _contract():
    tensors, facts = {}, {}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        parts = line.split()
        if len(parts) == 4 and parts[3] in ("bf16", "f32"):
            name, layout, shape, dtype = parts
            for lay in (("BNSD", "BSND", "TND") if layout == "*" else (layout,)):
                tensors[(name, lay)] = (shape, dtype)
        else:
            facts[parts[0]] = parts[1:]
    return tensors, facts


TENSORS, FACTS = _contract()
SYMS = dict(B=2, Nqk=3, Nv=6, S=5, T=7, D=128)


def _eval(shape: str, layout: str):
    if shape.startswith("like:"):
        return _eval(TENSORS[(shape[5:], layout)][0], layout)
    return tuple(SYMS[s] for s in shape.split(","))


def test_contract_file_is_complete():
    names = {"q", "k", "v", "g", "beta", "out", "initial_state", "final_state", "A_log",
             "dt_bias"}
    for lay in ("BNSD", "BSND", "TND"):
        assert {n for (n, l) in TENSORS if l == lay} == names
    assert FACTS["state_dims"] == ["Dv,Dk"]
    assert [float(x) for x in FACTS["lower_bound"]] == [-5.0, 0.0]


@pytest.mark.parametrize("layout", ["BNSD", "BSND", "TND"])
def test_binding_shapes_follow_the_contract(layout):
    S = SYMS["T"] if layout == "TND" else SYMS["S"]
    got = api._io_shapes(KdaShape(kda.LAYOUTS[layout], SYMS["B"], SYMS["Nqk"], SYMS["Nv"], S,
                                  SYMS["D"]), layout)
    alias = {"initial_state": "state", "final_state": "state"}
    for (name, lay), (shape, _) in TENSORS.items():
        if lay == layout:
            assert got[alias.get(name, name)] == _eval(shape, layout), (name, layout)


@pytest.mark.parametrize("layout", ["BNSD", "BSND", "TND"])
def test_generator_shapes_follow_the_contract(layout):
    S = SYMS["T"] if layout == "TND" else SYMS["S"]
    lens = [3, 4] if layout == "TND" else [S, S]
    w = W.custom("contract", layout, SYMS["B"], SYMS["Nqk"], SYMS["Nv"], S, lens,
                 init_state="normal", seed=1)
    inp = W.generate(w)
    for name in ("q", "k", "v", "g", "beta", "initial_state", "A_log", "dt_bias"):
        shape, dtype = TENSORS[(name, layout)]
        assert inp[name].shape == _eval(shape, layout), name
        assert inp[name].dtype == (np.uint16 if dtype == "bf16" else np.float32), name


def test_lower_bound_range_is_the_contracts():
    lo, hi = (float(x) for x in FACTS["lower_bound"])
    sh = _shape(layout=0, B=1, Nqk=1, Nv=1, S=256)
    st, p = _plan(_lib(), sh)
    assert st == 0
    # inside the closed range only the missing GPU stops the call (status 11 or 13); with a
    # GPU visible the call would launch on placeholder pointers, so it is not made
    if not gpu_visible():
        for lb in (lo, hi, 0.5 * (lo + hi)):
            assert _fwd(_lib(), sh, p, lb=lb) in (11, 13), lb
    for lb in (lo - 1e-3, hi + 1e-3):
        assert _fwd(_lib(), sh, p, lb=lb) == 6, lb


def _lib():
    return kda.load()


def test_quick_start_example_is_the_second_workload():
    ex = dict(kv.split("=", 1) for kv in FACTS["example"])
    w = W.workload(2)
    assert (w.B, w.Nqk, w.Nv, w.S, w.D) == tuple(int(ex[k]) for k in ("B", "Nqk", "Nv", "S", "D"))
    assert w.layout == ex["layout"] and w.init_state == ex["initial_state"]
    assert w.lower_bound == float(ex["lower_bound"])
    assert ex["scale"] == "D^-0.5" and w.scale == pytest.approx(int(ex["D"]) ** -0.5)


def _place(shape: str, layout: str, b: int, head: int, t: int, cu):
    """Index of (sequence b, head, token t) in a tensor of the given contract shape."""
    idx = []
    for s in shape.split(","):
        if s == "B":
            idx.append(b)
        elif s in ("Nqk", "Nv"):
            idx.append(head)
        elif s == "S":
            idx.append(t)
        elif s == "T":
            idx.append(int(cu[b]) + t)
        else:
            idx.append(slice(None))
    return tuple(idx)


@pytest.mark.parametrize("layout", ["BNSD", "BSND", "TND"])
def test_oracle_walker_and_state_orientation(layout):
    B, Nqk, Nv, S, D = 2, 2, 4, 5, 128
    cu = np.array([0, 4, 9]) if layout == "TND" else None
    rows = int(cu[-1]) if layout == "TND" else S
    # value head 2 reads query/key head 1: contiguous GQA groups of 2 (the pages fix only
    # Nv % Nqk == 0; head h % Nqk would be 0 here)
    b, h, t = 1, 2, 3
    a_ch, b_ch, c_ch, w_ch = 7, 90, 31, 50   # state row a, column b, key direction c, value w
    ONE, TWO = np.uint16(0x3F80), np.uint16(0x4000)   # bf16 1.0 and 2.0
    sym = dict(B=B, Nqk=Nqk, Nv=Nv, S=rows, T=rows, D=D)
    dims = lambda name: tuple(sym[s] for s in TENSORS[(name, layout)][0].split(","))  # noqa
    at = lambda name, head: _place(TENSORS[(name, layout)][0], layout, b, head, t, cu)  # noqa
    inp = {n: np.zeros(dims(n), dtype=np.uint16) for n in ("q", "k", "v", "g", "beta")}
    inp["k"][..., c_ch] = ONE           # every key is e_c, orthogonal to e_b
    inp["q"][at("q", 1)][b_ch] = ONE    # the query at (b, q/k head 1, t) is e_b
    inp["v"][at("v", h)][w_ch] = ONE    # one value, at (b, h, t)
    inp["beta"][at("beta", h)] = TWO    # its write strength sigma(2); sigma(0) = 1/2 elsewhere
    inp["A_log"] = np.zeros(Nv, np.float32)
    inp["dt_bias"] = np.zeros((Nv, D), np.float32)
    S0 = np.zeros((B, Nv, D, D), np.float32)
    S0[b, h, a_ch, b_ch] = 1.0          # contract: [.., Dv, Dk], so row a is a value channel
    inp["initial_state"] = S0
    scale = D ** -0.5
    out, fs, _ = oracle.flash_kda(inp, layout, B, Nqk, Nv, rows, D, scale, 0.0, cu,
                                  form="recurrent")
    assert out.shape == dims("v")
    # output: scale * S_t e_b = scale * e_a at (b, h, t) only (the write lives in column c);
    # the normalisation's epsilon shrinks unit rows by a factor 1 - O(1e-6)
    where = tuple(a_ch if isinstance(i, slice) else i for i in at("v", h))
    assert math.isclose(out[where], scale, rel_tol=1e-5)
    mask = np.ones(out.shape, bool)
    mask[where] = False
    assert np.all(out[mask] == 0.0)
    # final state: S0 plus column c = sigma(2) e_w after token t, then halved by the one token
    # after it (erase with beta = 1/2, no value)
    expect = S0.astype(np.float64)
    expect[b, h, w_ch, c_ch] = 0.5 / (1.0 + math.exp(-2.0))
    np.testing.assert_allclose(fs, expect, rtol=1e-5, atol=0)
    assert np.all(fs[expect == 0.0] == 0.0)

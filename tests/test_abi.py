"""C ABI on the host (no GPU): exports, planner, workspace sizing and argument checks.

The checks follow the FlashKDA README 约束说明: D = 128, B >= 1, S > 0, 1 <= Nqk <= Nv,
Nv % Nqk == 0, lower_bound in [-5, 0], TND cu_seqlens a strictly increasing prefix sum from 0
to T, BNSD/BSND valid lengths in [1, S].
"""
import ctypes
import os
import re

import numpy as np
import torch
import pytest

import chunked_kda_prefill_b200 as kda
from chunked_kda_prefill_b200._lib import KdaShape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P_I32 = ctypes.POINTER(ctypes.c_int32)


@pytest.fixture(scope="module")
def L():
    return kda.load()


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "kda.h")).read()
    return sorted(set(re.findall(r"KDA_API[^;(]*?\b(kda_\w+)\s*\(", txt)))


def test_header_declares_the_bound_symbols():
    assert header_symbols() == sorted(kda.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in header_symbols():
        assert hasattr(L, name), name


def _shape(layout=0, B=1, Nqk=1, Nv=1, S=256, D=128):
    return KdaShape(layout, B, Nqk, Nv, S, D)


def _plan(L, shape, cu=None, sms=148):
    n = ctypes.c_size_t(0)
    st = L.kda_plan_size(ctypes.byref(shape), ctypes.byref(n))
    if st:
        return st, None
    buf = np.zeros(n.value, dtype=np.int32)
    cu_p = None
    if cu is not None:
        cu = np.asarray(cu, dtype=np.int32)
        cu_p = cu.ctypes.data_as(P_I32)
    st = L.kda_plan(ctypes.byref(shape), cu_p, sms, buf.ctypes.data_as(P_I32), buf.size)
    return st, buf


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), 5), (dict(D=256), 5), (dict(D=0), 5), (dict(B=0), 3), (dict(S=0), 3), (dict(Nqk=0), 4), (dict(Nqk=3, Nv=2), 4),
    (dict(Nqk=3, Nv=4), 4), (dict(layout=3), 2), (dict(layout=-1), 2)])
def test_shape_checks(L, kw, code):
    st, _ = _plan(L, _shape(**kw))
    assert st == code


@pytest.mark.parametrize("layout,B,S,cu,code", [
    (2, 2, 100, None, 7),                 # TND needs cu_seqlens
    (2, 2, 100, [1, 50, 100], 7),         # must start at 0
    (2, 2, 100, [0, 50, 99], 7),          # must end at T
    (2, 2, 100, [0, 50, 50, 100], 7),     # (B=2 reads 3 entries) not strictly increasing
    (2, 2, 100, [0, 100, 100], 7),        # empty sequence
    (0, 2, 100, [0, 0, 50], 7),           # BNSD length 0
    (0, 2, 100, [0, 101, 150], 7),        # BNSD length > S
    (1, 2, 100, [0, 60, 160], 0),         # BSND lengths 60, 100: fine
    (1, 2, 100, [3, 60, 160], 7),         # BSND: prefix sums start at 0
    (1, 2, 100, [0, 60, 59], 7),          # BSND: not increasing (length -1)
    (1, 2, 100, [0, 60, 60], 7),          # BSND: an empty sequence
    (1, 2, 100, [0, 60, 161], 7),         # BSND: second length 101 > S
    (1, 3, 100, [0, 100, 200, 300], 0),   # BSND: every length S, cu[B] == B*S
    (1, 3, 100, [0, 100, 250, 300], 7),   # BSND: 150 > S although cu[B] == B*S
    (2, 2, 100, [0, 37, 100], 0),
])
def test_seqlen_checks(L, layout, B, S, cu, code):
    st, _ = _plan(L, _shape(layout=layout, B=B, S=S, Nqk=2, Nv=4), cu)
    assert st == code


def test_plan_records_longest_first(L):
    cu = [0, 10, 200, 265]
    st, p = _plan(L, _shape(layout=2, B=3, Nqk=1, Nv=2, S=265), cu)
    assert st == 0
    assert p[0] == 0x4B444131 and p[4] == 6 and p[11] == (3 + 2 + 1) * 2 and p[12] == 3
    recs = p[16:].reshape(6, 8)
    # (b, h, hq, tok_start, len, chunks, chunk_offset)
    assert [tuple(r[:7]) for r in recs] == [
        (1, 0, 0, 10, 190, 3, 0), (1, 1, 0, 10, 190, 3, 3), (2, 0, 0, 200, 65, 2, 6),
        (2, 1, 0, 200, 65, 2, 8), (0, 0, 0, 0, 10, 1, 10), (0, 1, 0, 0, 10, 1, 11)]
    ws = ctypes.c_size_t(0)
    assert L.kda_workspace_size(p.ctypes.data_as(P_I32), p.size, ctypes.byref(ws)) == 0
    assert ws.value >= 256


def test_plan_gqa_head_map(L):
    st, p = _plan(L, _shape(layout=0, B=1, Nqk=4, Nv=16, S=64))
    recs = p[16:].reshape(16, 8)
    assert [int(r[2]) for r in recs] == [h // 4 for h in range(16)]


def test_plan_capacity_and_corruption(L):
    sh = _shape(layout=0, B=2, Nqk=2, Nv=2, S=300)
    n = ctypes.c_size_t(0)
    assert L.kda_plan_size(ctypes.byref(sh), ctypes.byref(n)) == 0
    small = np.zeros(n.value - 1, dtype=np.int32)
    assert L.kda_plan(ctypes.byref(sh), None, 148, small.ctypes.data_as(P_I32), small.size) == 8
    st, p = _plan(L, sh)
    ws = ctypes.c_size_t(0)
    bad = p.copy()
    bad[16 + 4] += 1  # edit a record: the checksum no longer matches
    assert L.kda_workspace_size(bad.ctypes.data_as(P_I32), bad.size, ctypes.byref(ws)) == 8
    assert L.kda_workspace_size(p.ctypes.data_as(P_I32), p.size - 1, ctypes.byref(ws)) == 8


def gpu_visible() -> bool:
    """True when a CUDA device is visible.  A call with placeholder pointers that passes every
    host check would then launch kernels on those addresses, so such calls are only made on a
    host without a GPU (where they must stop at the device check)."""
    try:
        import torch
        return bool(torch.cuda.is_available())
    except Exception:
        return True


def _fwd(L, shape, plan, **over):
    """kda_forward with fake (never dereferenced) device pointers; every check is on the host."""
    a = dict(q=0x10000000, k=0x20000000, v=0x30000000, g=0x40000000, beta=0x50000000,
             scale=0.088, S0=0x60000000, A_log=0x70000000, dt=0x71000000, lb=-5.0,
             ws=0x80000000, ws_bytes=1 << 40, out=0x90000000, fs=0xA0000000, plan_dev=0xB0000000)
    a.update(over)
    return L.kda_forward(ctypes.byref(shape), plan.ctypes.data_as(P_I32), a["plan_dev"],
                         plan.size, a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"],
                         a["S0"], a["A_log"], a["dt"], a["lb"], a["ws"], a["ws_bytes"], a["out"],
                         a["fs"], None)


def test_forward_argument_checks(L):
    sh = _shape(layout=0, B=1, Nqk=1, Nv=1, S=256)
    st, p = _plan(L, sh)
    assert st == 0
    assert _fwd(L, sh, p, q=None) == 1
    assert _fwd(L, sh, p, out=None) == 1
    assert _fwd(L, sh, p, lb=0.5) == 6
    assert _fwd(L, sh, p, lb=-5.01) == 6
    assert _fwd(L, sh, p, lb=float("nan")) == 6
    assert _fwd(L, sh, p, scale=float("inf")) == 6
    assert _fwd(L, sh, p, ws_bytes=100) == 10
    assert _fwd(L, sh, p, ws=0x80000010) == 10          # not 256-byte aligned
    assert _fwd(L, sh, p, fs=0x60000000) == 9           # final_state aliases initial_state
    assert _fwd(L, sh, p, out=0x30000000 + 64) == 9     # out overlaps v
    assert _fwd(L, sh, p, q=0x10000008) == 14           # q not 16-byte aligned
    assert _fwd(L, sh, p, beta=0x50000001) == 14        # beta not 2-byte aligned
    other = _shape(layout=0, B=1, Nqk=1, Nv=1, S=512)
    assert _fwd(L, other, p) == 8                       # plan built for another shape
    # all host checks pass: what remains needs a GPU (no device here -> CUDA/device error)
    if not gpu_visible():
        assert _fwd(L, sh, p) in (11, 13)


def test_status_strings(L):
    for code in range(16):
        s = L.kda_status_string(code).decode()
        assert s.startswith("KDA_")


def _dec(L, B=2, Nqk=1, Nv=2, D=128, **kw):
    a = dict(q=0x10000000, k=0x11000000, v=0x12000000, g=0x13000000, beta=0x14000000, scale=0.09,
             s0=0x20000000, A_log=0x15000000, dt=0x16000000, lb=-5.0, out=0x17000000,
             s1=0x30000000)
    a.update(kw)
    return L.kda_decode(B, Nqk, Nv, D, a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"],
                        a["s0"], a["A_log"], a["dt"], a["lb"], a["out"], a["s1"], None)


def test_head_dim_64_plans(L):
    # D = 64 runs through the D = 128 kernels (upper channels read as zeros); the plan records D
    for layout, cu in ((0, None), (1, [0, 100, 256]), (2, [0, 7, 256])):
        B = 1 if cu is None else len(cu) - 1
        st, buf = _plan(L, _shape(layout=layout, B=B, Nqk=2, Nv=4, S=256, D=64), cu)
        assert st == 0, (layout, st)
        ws = ctypes.c_size_t(0)
        assert L.kda_workspace_size(buf.ctypes.data_as(P_I32), buf.size, ctypes.byref(ws)) == 0
        assert ws.value >= 256


def test_state_chain_argument_checks(L):
    c = lambda units=2, D=128, n=1, S_in=0x10000000, M=0x20000000, R=0x30000000, stride=0, \
        S_out=0x40000000: L.kda_state_chain(units, D, n, S_in, M, R, stride, S_out, None)  # noqa: E731
    assert c(D=96) == 5
    assert c(units=0) == 3
    assert c(n=-1) == 3
    assert c(stride=100) == 3                   # below units * D * D
    assert c(stride=2 * 128 * 128 * 2 + 1) == 3  # not a multiple of 4
    assert c(S_out=None) == 1
    assert c(M=None) == 1
    assert c(n=0, M=None, R=None, S_out=None) == 1
    assert c(M=0x20000004) == 14                # M not 16-byte aligned
    assert c(S_in=0x40000010) == 9              # S_in overlaps S_out without being it
    assert c(R=0x40000000 - 4 * 128 * 128) == 9  # R (2 states, 128 KiB) runs into S_out


def test_decode_argument_checks(L):
    assert _dec(L, D=96) == 5
    assert _dec(L, D=256) == 5
    assert _dec(L, B=0) == 3
    assert _dec(L, Nv=3, Nqk=2) == 4
    assert _dec(L, q=None) == 1
    assert _dec(L, s1=None) == 1
    assert _dec(L, lb=0.25) == 6
    assert _dec(L, scale=float("nan")) == 6
    assert _dec(L, v=0x12000008) == 14                  # v not 16-byte aligned
    assert _dec(L, beta=0x14000001) == 14               # beta not 2-byte aligned
    assert _dec(L, s1=0x20000000 + 4096) == 9           # state_out partly overlaps state_in
    assert _dec(L, out=0x12000000 + 256) == 9           # out overlaps v
    assert _dec(L, out=0x30000000 + 4096) == 9          # out overlaps state_out
    # in place (state_out == state_in) and a zero initial state are allowed: the remaining
    # checks need a GPU (none here -> CUDA/device error)
    if not gpu_visible():
        assert _dec(L, s1=0x20000000) in (11, 13)
        assert _dec(L, s0=None) in (11, 13)


def _plan_seg(L, shape, seg, cu=None, sms=148):
    n = ctypes.c_size_t(0)
    assert L.kda_plan_size(ctypes.byref(shape), ctypes.byref(n)) == 0
    buf = np.zeros(n.value, dtype=np.int32)
    cu_p = None
    if cu is not None:
        cu = np.asarray(cu, dtype=np.int32)
        cu_p = cu.ctypes.data_as(P_I32)
    st = L.kda_plan_segmented(ctypes.byref(shape), cu_p, sms, seg, buf.ctypes.data_as(P_I32),
                              buf.size)
    return st, buf


def _ws(L, p):
    ws = ctypes.c_size_t(0)
    assert L.kda_workspace_size(p.ctypes.data_as(P_I32), p.size, ctypes.byref(ws)) == 0
    return ws.value


def test_default_schedule_segments_only_few_long_units(L):
    # 3 units of 128 chunks on 148 SMs: segmented; the cost model's pick, which measured fastest
    # (6-chunk segments: 0.296 ms against 0.323 with 3, 0.327 with 8, 1.549 whole)
    st, p = _plan(L, _shape(layout=0, B=1, Nqk=3, Nv=3, S=8192))
    assert st == 0 and p[14] == 6
    # 32 units of 63 and 44 chunks: 11-chunk segments (0.504 ms against 0.583 with 6, 0.519
    # with 12, 0.742 whole)
    st, p = _plan(L, _shape(layout=1, B=2, Nqk=4, Nv=16, S=4000), cu=[0, 4000, 6777])
    assert st == 0 and p[14] == 11
    # 128 units of 256 chunks: whole units
    st, p = _plan(L, _shape(layout=0, B=4, Nqk=32, Nv=32, S=16384))
    assert st == 0 and p[14] == 0 and _ws(L, p) == 256
    # the large prefill at B = 1, 32 units of 256 chunks: 52-chunk segments (1.924 ms measured,
    # against 2.957 ms for one wave of whole units)
    st, p = _plan(L, _shape(layout=0, B=1, Nqk=32, Nv=32, S=16384))
    assert st == 0 and p[14] == 52
    # one unit of 4 chunks: too short to split
    st, p = _plan(L, _shape(layout=0, B=1, Nqk=1, Nv=1, S=256))
    assert st == 0 and p[14] == 0
    # few SMs: 3 units already fill them
    st, p = _plan(L, _shape(layout=0, B=1, Nqk=3, Nv=3, S=8192), sms=4)
    assert st == 0 and p[14] == 0


def test_segmented_plan_state_slots(L):
    # varlen BSND: lengths 4000 and 2777 -> 63 and 44 chunks per unit, 16 heads each
    sh = _shape(layout=1, B=2, Nqk=4, Nv=16, S=4000)
    st, p = _plan_seg(L, sh, 8, cu=[0, 4000, 6777])
    assert st == 0 and p[14] == 8
    recs = p[16:].reshape(32, 8)
    nseg = [(int(r[5]) + 7) // 8 for r in recs]
    assert sorted(set(nseg)) == [6, 8]
    # PR_SEG_BASE: prefix sum of (segments - 1) over the earlier units, in plan order
    expect, acc = [], 0
    for s in nseg:
        expect.append(acc)
        acc += s - 1
    assert [int(r[7]) for r in recs] == expect
    assert _ws(L, p) == 256 + acc * 3 * 128 * 128 * 4
    # segment_chunks = 0 is the whole-unit schedule; negative is rejected
    st, p0 = _plan_seg(L, sh, 0, cu=[0, 4000, 6777])
    assert st == 0 and p0[14] == 0 and _ws(L, p0) == 256
    assert _plan_seg(L, sh, -1, cu=[0, 4000, 6777])[0] == 3
    # a corrupted segment length fails validation
    bad = p.copy()
    bad[14] = -2
    ws = ctypes.c_size_t(0)
    assert L.kda_workspace_size(bad.ctypes.data_as(P_I32), bad.size, ctypes.byref(ws)) == 8


@pytest.mark.parametrize("layout", ["BNSD", "BSND", "TND"])
def test_binding_checks_tensors_against_the_plan(layout):
    """The library sees only pointers, so the binding rejects tensors that do not match the
    plan's shape (a short tensor would otherwise be read past its end)."""
    from chunked_kda_prefill_b200 import api
    B, Nqk, Nv, S, D = 2, 1, 2, 100, 128
    cu = [0, 60, 100] if layout == "TND" else None
    shape = KdaShape(kda.LAYOUTS[layout], B, Nqk, Nv, S, D)
    plan = kda.make_plan(shape, layout, cu)
    want = api._io_shapes(shape, layout)
    bf = lambda n: torch.zeros(want[n], dtype=torch.bfloat16)  # noqa: E731
    f32 = lambda n: torch.zeros(want[n], dtype=torch.float32)  # noqa: E731
    good = {n: bf(n) for n in ("q", "k", "v", "g", "beta", "out")}
    good.update(A_log=f32("A_log"), dt_bias=f32("dt_bias"), initial_state=f32("state"),
                final_state=f32("state"))
    cpu = torch.device("cpu")
    api._check_inputs(plan, layout, cpu, good)
    api._check_inputs(plan, layout, cpu, dict(good, initial_state=None, out=None))
    for name in good:
        t = good[name]
        short = t.reshape(-1)[:-1]
        with pytest.raises(kda.KdaError) as e:
            api._check_inputs(plan, layout, cpu, dict(good, **{name: short}))
        assert e.value.code == 3, name
    with pytest.raises(TypeError):
        api._check_inputs(plan, layout, cpu, dict(good, q=good["q"].float()))
    with pytest.raises(ValueError):
        api._check_inputs(plan, layout, cpu, dict(good, v=good["v"].transpose(0, 1)))
    other = "BSND" if layout != "BSND" else "BNSD"
    with pytest.raises(kda.KdaError) as e:
        api._check_inputs(plan, other, cpu, good)
    assert e.value.code == 8
    # a plan whose device copy is not where the tensors are (here: a host plan, meta tensors)
    with pytest.raises(ValueError):
        api._check_inputs(plan, layout, torch.device("meta"), {})
    # workspace: its size in bytes, and only contiguous memory on the tensors' device
    assert api._workspace_bytes(torch.empty(10, dtype=torch.float32), cpu) == 40
    with pytest.raises(ValueError):
        api._workspace_bytes(torch.empty(4, 4)[:, 0], cpu)
    with pytest.raises(ValueError):
        api._workspace_bytes(torch.empty(16, device="meta"), cpu)

"""Properties of the host planner over random problems (hypothesis; no GPU).

For any valid shape, layout, set of valid lengths, SM count and schedule, the plan must:
- hold one record per (sequence, value head), each exactly once;
- map value head h to query/key head h / (Nv / Nqk) (contiguous GQA groups);
- give each record its sequence's token start (TND: cu[b]; BNSD/BSND: 0) and valid length, and
  ceil(length / 64) chunks;
- order records by chunk count, most first, ties by (sequence, head), with chunk offsets the
  running sum of chunks and the header's totals equal to the sum and the maximum;
- under a segmented schedule, give each record the running sum of (segments - 1) of the records
  before it as its state-slot base, and size the workspace for exactly that many slot triples;
- pick a segmented schedule by default only when at least two SMs are free per unit and the
  longest unit has at least 4 chunks.
"""
import ctypes

import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import HealthCheck, given, settings, strategies as st  # noqa: E402

import chunked_kda_prefill_b200 as kda  # noqa: E402
from chunked_kda_prefill_b200._lib import KdaShape  # noqa: E402

P_I32 = ctypes.POINTER(ctypes.c_int32)
HEADER, RECORD = 16, 8
SLOT_BYTES = 3 * 128 * 128 * 4   # one segment's M, R and start state, fp32 at the largest D


@st.composite
def problems(draw):
    layout = draw(st.sampled_from([0, 1, 2]))
    B = draw(st.integers(1, 5))
    Nqk = draw(st.integers(1, 3))
    Nv = Nqk * draw(st.integers(1, 3))
    D = draw(st.sampled_from([64, 128]))
    if layout == 2:
        lens = draw(st.lists(st.integers(1, 700), min_size=B, max_size=B))
        S = sum(lens)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    else:
        S = draw(st.integers(1, 700))
        if draw(st.booleans()):
            lens = draw(st.lists(st.integers(1, S), min_size=B, max_size=B))
            cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        else:
            lens, cu = [S] * B, None
    sms = draw(st.sampled_from([1, 4, 16, 148]))
    seg = draw(st.sampled_from([None, 0, 1, 2, 3, 7]))
    return layout, B, Nqk, Nv, S, D, lens, cu, sms, seg


def _make(L, shape, cu, sms, seg):
    n = ctypes.c_size_t(0)
    assert L.kda_plan_size(ctypes.byref(shape), ctypes.byref(n)) == 0
    buf = np.zeros(n.value, dtype=np.int32)
    cu_p = None if cu is None else cu.ctypes.data_as(P_I32)
    if seg is None:
        st_ = L.kda_plan(ctypes.byref(shape), cu_p, sms, buf.ctypes.data_as(P_I32), buf.size)
    else:
        st_ = L.kda_plan_segmented(ctypes.byref(shape), cu_p, sms, seg,
                                   buf.ctypes.data_as(P_I32), buf.size)
    return st_, buf


@settings(max_examples=300, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(problems())
def test_plan_properties(prob):
    layout, B, Nqk, Nv, S, D, lens, cu, sms, seg = prob
    L = kda.load()
    shape = KdaShape(layout, B, Nqk, Nv, S, D)
    status, p = _make(L, shape, cu, sms, seg)
    assert status == 0
    n_units = B * Nv
    assert p[4] == n_units and p.size == HEADER + n_units * RECORD
    recs = p[HEADER:].reshape(n_units, RECORD).astype(np.int64)

    G = Nv // Nqk
    chunks = lambda L_: -(-L_ // 64)  # noqa: E731
    seen = set()
    for b, h, hq, tok0, ln, nch, off, base in recs:
        assert (b, h) not in seen
        seen.add((b, h))
        assert hq == h // G
        assert tok0 == (cu[b] if layout == 2 else 0)
        assert ln == lens[b] and nch == chunks(ln)
    assert len(seen) == n_units

    order = sorted(((-chunks(lens[b]), b, h) for b in range(B) for h in range(Nv)))
    assert [(int(r[0]), int(r[1])) for r in recs] == [(b, h) for _, b, h in order]
    offs = np.concatenate([[0], np.cumsum(recs[:, 5])[:-1]])
    assert np.array_equal(recs[:, 6], offs)
    assert p[11] == recs[:, 5].sum() and p[12] == recs[:, 5].max()

    n_seg = int(p[14])
    if seg is not None:
        assert n_seg == seg
    ws = ctypes.c_size_t(0)
    assert L.kda_workspace_size(p.ctypes.data_as(P_I32), p.size, ctypes.byref(ws)) == 0
    if n_seg > 0:
        extra = [-(-int(c) // n_seg) - 1 for c in recs[:, 5]]
        bases = np.concatenate([[0], np.cumsum(extra)[:-1]])
        assert np.array_equal(recs[:, 7], bases)
        assert ws.value == 256 + sum(extra) * SLOT_BYTES
    else:
        assert ws.value == 256
    if seg is None and n_seg > 0:
        assert 2 * n_units <= sms and p[12] >= 4

"""Checks that pin the fp64 oracle to facts other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
closed form, a textbook special case, brute force on tiny inputs, or a structural
invariant of the method.  ``tests/test_oracle.py`` runs them on the correct
oracle; ``tests/test_oracle_mutations.py`` plants mistakes in the oracle and
checks that at least one pin fails for each.

The method (Kimi Delta Attention, per the FlashKDA README and vLLM PR 43195):
    S_t = S_{t-1} Diag(exp(g_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = scale * S_t q_t,
with q/k L2-normalised, beta = sigmoid(logit), g activated from the raw gate.
"""
from __future__ import annotations

import math

import numpy as np

import oracle

SCALE = 1.0 / math.sqrt(128.0)


def _rand_unit_inputs(rng, L, Dk, Dv, lb=-5.0, unit_keys=True):
    q = rng.standard_normal((L, Dk))
    k = rng.standard_normal((L, Dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, Dv))
    # decays in (lb, 0): a spread of fast and slow channels
    g = lb / (1.0 + np.exp(-rng.standard_normal((L, Dk)) * 2.0))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    S0 = rng.standard_normal((Dv, Dk)) * 0.3
    return q, k, v, g, beta, S0


def _rel(a, b):
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


# ---------------------------------------------------------------------------
# I1: chunked form == recurrence (any chunk size, tails included)
# ---------------------------------------------------------------------------

def pin_chunked_equals_recurrent(seed=0, Ds=((16, 16), (8, 12)), Ls=(1, 5, 17, 40),
                                 Cs=(1, 2, 3, 16, 64), lb=-5.0, tol=1e-9):
    rng = np.random.default_rng(seed)
    for Dk, Dv in Ds:
        for L in Ls:
            q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L, Dk, Dv, lb)
            o_r, S_r = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
            for C in Cs:
                o_c, S_c = oracle.chunked(q, k, v, g, beta, SCALE, S0, C=C)
                assert _rel(o_c, o_r) < tol, (Dk, Dv, L, C, _rel(o_c, o_r))
                assert _rel(S_c, S_r) < tol, (Dk, Dv, L, C, _rel(S_c, S_r))


def pin_chunked_equals_recurrent_d128(seed=1, L=150, lb=-5.0, tol=1e-9):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L, 128, 128, lb)
    o_r, S_r = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
    o_c, S_c = oracle.chunked(q, k, v, g, beta, SCALE, S0, C=64)
    assert _rel(o_c, o_r) < tol, _rel(o_c, o_r)
    assert _rel(S_c, S_r) < tol, _rel(S_c, S_r)


def pin_chunked_equals_recurrent_d64(seed=10, L=150, lb=-5.0, tol=1e-9):
    """I1 at the second head dim the library builds (D = 64)."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L, 64, 64, lb)
    o_r, S_r = oracle.recurrent(q, k, v, g, beta, 1.0 / 8.0, S0)
    o_c, S_c = oracle.chunked(q, k, v, g, beta, 1.0 / 8.0, S0, C=64)
    assert _rel(o_c, o_r) < tol, _rel(o_c, o_r)
    assert _rel(S_c, S_r) < tol, _rel(S_c, S_r)


# ---------------------------------------------------------------------------
# I1b: a span's state map is affine in its start state.  With M the end state from S0 = I and
# v = 0, and R the end state from S0 = 0, every S0 ends at S0 M + R; maps of consecutive spans
# compose, and the second span run from the folded state gives the whole sequence's outputs.
# (The identity follows from S_t = S_{t-1} Diag(e^g_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T
# being affine in S_{t-1}; the chunk-parallel and context-parallel schedules rest on it.)
# ---------------------------------------------------------------------------

def pin_affine_span_map(seed=11, L1=37, L2=29, Dk=12, Dv=9, lb=-0.05, tol=1e-10):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L1 + L2, Dk, Dv, lb)
    o_full, S_full = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
    spans = (slice(0, L1), slice(L1, L1 + L2))
    maps = []
    for sp in spans:
        # M (Dk x Dk) is the end state of a Dk-row state that starts at I and takes no values
        n = sp.stop - sp.start
        _, M = oracle.recurrent(q[sp], k[sp], np.zeros((n, Dk)), g[sp], beta[sp], SCALE,
                                np.eye(Dk))
        _, R = oracle.recurrent(q[sp], k[sp], v[sp], g[sp], beta[sp], SCALE,
                                np.zeros((Dv, Dk)))
        maps.append((M, R))
    S_mid = S0 @ maps[0][0] + maps[0][1]
    _, S_mid_ref = oracle.recurrent(q[spans[0]], k[spans[0]], v[spans[0]], g[spans[0]],
                                    beta[spans[0]], SCALE, S0)
    assert _rel(S_mid, S_mid_ref) < tol, _rel(S_mid, S_mid_ref)
    S_end = S_mid @ maps[1][0] + maps[1][1]
    assert _rel(S_end, S_full) < tol, _rel(S_end, S_full)
    o2, S2 = oracle.recurrent(q[spans[1]], k[spans[1]], v[spans[1]], g[spans[1]],
                              beta[spans[1]], SCALE, S_mid)
    assert _rel(o2, o_full[spans[1]]) < tol and _rel(S2, S_full) < tol
    # slow decays (lb near 0) keep the start state in play, so the check is not vacuous
    assert _rel(S_full, maps[0][1] @ maps[1][0] + maps[1][1]) > 1e-3


# ---------------------------------------------------------------------------
# I2: beta = 0 -> pure decay, closed form
#   S_T = S0 Diag(exp(sum_t g_t)),  o_t = scale * S0 (exp(G_t) * q_t)
# ---------------------------------------------------------------------------

def pin_beta_zero_pure_decay(seed=2, L=70, Dk=16, Dv=8, tol=1e-12):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L, Dk, Dv, lb=-0.3)
    beta = np.zeros(L)
    G = np.cumsum(g, axis=0)
    o_exp = SCALE * (np.exp(G) * q) @ S0.T
    S_exp = S0 * np.exp(G[-1])[None, :]
    for form in ("recurrent", "chunked"):
        if form == "recurrent":
            o, S = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
        else:
            o, S = oracle.chunked(q, k, v, g, beta, SCALE, S0, C=16)
        assert _rel(o, o_exp) < tol, (form, _rel(o, o_exp))
        assert _rel(S, S_exp) < tol, (form, _rel(S, S_exp))


# ---------------------------------------------------------------------------
# I3: g = 0 -> ungated delta rule, textbook dense products
#   S <- S (I - beta k k^T) + beta v k^T
# ---------------------------------------------------------------------------

def pin_g_zero_textbook_delta_rule(seed=3, L=50, Dk=12, Dv=10, tol=1e-11):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L, Dk, Dv)
    g = np.zeros_like(g)
    S = S0.copy()
    o_exp = np.zeros((L, Dv))
    for t in range(L):
        S = S @ (np.eye(Dk) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        o_exp[t] = SCALE * S @ q[t]
    for C in (64, 5):
        o, Sf = oracle.chunked(q, k, v, g, beta, SCALE, S0, C=C)
        assert _rel(o, o_exp) < tol, _rel(o, o_exp)
        assert _rel(Sf, S) < tol, _rel(Sf, S)
    o, Sf = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
    assert _rel(o, o_exp) < tol and _rel(Sf, S) < tol


# ---------------------------------------------------------------------------
# I4a: basis keys, beta = 1, g = 0: each step overwrites one state column with v_t
# ---------------------------------------------------------------------------

def pin_basis_keys_overwrite(seed=4, L=40, D=8, tol=1e-12):
    rng = np.random.default_rng(seed)
    S0 = rng.standard_normal((D, D))
    v = rng.standard_normal((L, D))
    cols = rng.integers(0, D, size=L)          # written column at step t
    qcols = rng.integers(0, D, size=L)         # queried column at step t
    k = np.eye(D)[cols]
    q = np.eye(D)[qcols]
    g = np.zeros((L, D))
    beta = np.ones(L)
    cur = S0.copy()
    o_exp = np.zeros((L, D))
    for t in range(L):
        cur[:, cols[t]] = v[t]
        o_exp[t] = SCALE * cur[:, qcols[t]]
    for form in ("recurrent", "chunked"):
        if form == "recurrent":
            o, S = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
        else:
            o, S = oracle.chunked(q, k, v, g, beta, SCALE, S0, C=16)
        assert _rel(o, o_exp) < tol, form
        assert _rel(S, cur) < tol, form


# ---------------------------------------------------------------------------
# I4b: repeated unit key, g = 0, q = k: a per-channel exponential moving average
#   m_t = (1 - beta_t) m_{t-1} + beta_t v_t,  m_0 = S0 k,  o_t = scale m_t
# ---------------------------------------------------------------------------

def pin_repeated_key_ema(seed=5, L=60, Dk=16, Dv=6, tol=1e-12):
    rng = np.random.default_rng(seed)
    kk = rng.standard_normal(Dk)
    kk /= np.linalg.norm(kk)
    k = np.tile(kk, (L, 1))
    q = k.copy()
    v = rng.standard_normal((L, Dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    S0 = rng.standard_normal((Dv, Dk))
    m = S0 @ kk
    o_exp = np.zeros((L, Dv))
    for t in range(L):
        m = (1 - beta[t]) * m + beta[t] * v[t]
        o_exp[t] = SCALE * m
    for form in ("recurrent", "chunked"):
        if form == "recurrent":
            o, _ = oracle.recurrent(q, k, v, np.zeros((L, Dk)), beta, SCALE, S0)
        else:
            o, _ = oracle.chunked(q, k, v, np.zeros((L, Dk)), beta, SCALE, S0, C=7)
        assert _rel(o, o_exp) < tol, form


# ---------------------------------------------------------------------------
# I5: brute force on tiny inputs (the literal matrix form of the recurrence)
# ---------------------------------------------------------------------------

def pin_brute_force_tiny(seed=6, tol=1e-12):
    rng = np.random.default_rng(seed)
    for D in (2, 4):
        for L in (1, 3, 8):
            q, k, v, g, beta, S0 = _rand_unit_inputs(rng, L, D, D, lb=-2.0)
            S = S0.copy()
            o_exp = np.zeros((L, D))
            for t in range(L):
                S = (S @ np.diag(np.exp(g[t])) @ (np.eye(D) - beta[t] * np.outer(k[t], k[t]))
                     + beta[t] * np.outer(v[t], k[t]))
                o_exp[t] = SCALE * S @ q[t]
            for C in (3, 64):
                o, Sf = oracle.chunked(q, k, v, g, beta, SCALE, S0, C=C)
                assert _rel(o, o_exp) < tol and _rel(Sf, S) < tol, (D, L, C)
            o, Sf = oracle.recurrent(q, k, v, g, beta, SCALE, S0)
            assert _rel(o, o_exp) < tol and _rel(Sf, S) < tol, (D, L)


def pin_unit_lower_inverse(seed=7, tol=1e-10):
    rng = np.random.default_rng(seed)
    for n in (1, 2, 5, 16, 64):
        T = np.tril(rng.standard_normal((n, n)) * 0.3, -1)
        X = oracle.unit_lower_inverse(T)
        ref = np.linalg.inv(np.eye(n) + T)
        assert _rel(X, ref) < tol, n


# ---------------------------------------------------------------------------
# Activations (FlashKDA parameter table)
# ---------------------------------------------------------------------------

def pin_activations(seed=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((5, 16))
    dt = rng.standard_normal(16)
    # lower_bound = 0 switches the gate off exactly
    assert np.all(oracle.gate(x, dt, 0.7, 0.0) == 0.0)
    # sigmoid(0) = 1/2: with A_log = 0 and g_raw + dt_bias = 0 the gate is lower_bound / 2
    g = oracle.gate(np.full((1, 4), 0.25), np.full(4, -0.25), 0.0, -3.0)
    assert np.all(g == -1.5), g
    # the bound is a bound: g in (lower_bound, 0)
    for lb in (-5.0, -2.0, -0.1):
        g = oracle.gate(x * 3, dt, 0.5, lb)
        assert np.all(g < 0) and np.all(g > lb)
    # g depends on g_raw + dt_bias only, and exp(A_log) scales that sum
    g1 = oracle.gate(x, dt, 0.0, -5.0)
    g2 = oracle.gate(x + dt[None, :], np.zeros(16), 0.0, -5.0)
    assert np.allclose(g1, g2, rtol=0, atol=1e-14)
    g3 = oracle.gate(x, dt, math.log(2.0), -5.0)
    g4 = oracle.gate(2 * (x + dt[None, :]), np.zeros(16), 0.0, -5.0)
    assert np.allclose(g3, g4, rtol=0, atol=1e-14)
    # textbook logistic values
    b = oracle.beta_sigmoid(np.array([0.0, math.log(3.0), -math.log(3.0), 40.0]))
    assert b[0] == 0.5 and abs(b[1] - 0.75) < 1e-15 and abs(b[2] - 0.25) < 1e-15
    assert abs(b[3] - 1.0) < 1e-15
    # L2 normalise: unit rows, scale invariance, zero row -> 0 (not NaN), 3-4-5 triangle
    y = oracle.l2norm(x * 7.0)
    assert np.allclose(np.linalg.norm(y, axis=1), 1.0, atol=1e-9)
    assert np.allclose(oracle.l2norm(x), oracle.l2norm(x * 64.0), atol=1e-9)
    z = oracle.l2norm(np.zeros((1, 8)))
    assert np.all(z == 0.0)
    t = oracle.l2norm(np.array([[3.0, 4.0]]))
    assert np.allclose(t, [[0.6, 0.8]], atol=1e-7)


# ---------------------------------------------------------------------------
# Whole-op structure (raw bf16 inputs through the layouts)
# ---------------------------------------------------------------------------

def _bits(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    u = x.view(np.uint32)
    return ((u + ((u >> 16) & 1) + 0x7FFF) >> 16).astype(np.uint16)


def _raw_inputs(rng, B, Nqk, Nv, S, D):
    return {"q": _bits(rng, (B, Nqk, S, D)), "k": _bits(rng, (B, Nqk, S, D)),
            "v": _bits(rng, (B, Nv, S, D)), "g": _bits(rng, (B, Nv, S, D)),
            "beta": _bits(rng, (B, Nv, S)),
            "A_log": rng.standard_normal(Nv).astype(np.float32),
            "dt_bias": rng.standard_normal((Nv, D)).astype(np.float32),
            "initial_state": (rng.standard_normal((B, Nv, D, D)) * 0.1).astype(np.float32)}


def pin_structure(seed=9, D=16, tol=1e-12):
    rng = np.random.default_rng(seed)
    B, Nqk, Nv, S = 2, 1, 2, 37
    lens = [37, 20]
    cu = np.array([0, 37, 57])
    inp = _raw_inputs(rng, B, Nqk, Nv, S, D)
    lb = -1.0
    o_bnsd, fs_bnsd, _ = oracle.flash_kda(inp, "BNSD", B, Nqk, Nv, S, D, SCALE, lb, cu)
    # BSND: the same data, transposed storage
    inp_bsnd = dict(inp)
    for n in ("q", "k", "v", "g"):
        inp_bsnd[n] = np.ascontiguousarray(inp[n].transpose(0, 2, 1, 3))
    inp_bsnd["beta"] = np.ascontiguousarray(inp["beta"].transpose(0, 2, 1))
    o_bsnd, fs_bsnd, _ = oracle.flash_kda(inp_bsnd, "BSND", B, Nqk, Nv, S, D, SCALE, lb, cu)
    assert np.array_equal(o_bsnd.transpose(0, 2, 1, 3), o_bnsd)
    assert np.array_equal(fs_bsnd, fs_bnsd)
    # TND: packed valid rows only
    inp_tnd = dict(inp)
    for n in ("q", "k", "v", "g"):
        inp_tnd[n] = np.concatenate([inp_bsnd[n][b, :lens[b]] for b in range(B)])
    inp_tnd["beta"] = np.concatenate([inp_bsnd["beta"][b, :lens[b]] for b in range(B)])
    o_tnd, fs_tnd, _ = oracle.flash_kda(inp_tnd, "TND", B, Nqk, Nv, int(cu[-1]), D, SCALE, lb, cu)
    for b in range(B):
        assert np.array_equal(o_tnd[cu[b]:cu[b + 1]], o_bsnd[b, :lens[b]])
    assert np.array_equal(fs_tnd, fs_bnsd)
    # rows outside a valid length are zero
    assert np.all(o_bnsd[1, :, 20:] == 0.0)
    # varlen == separate calls (sequence 1 alone, as its own batch of one)
    one = {n: (inp[n][1:2] if n not in ("A_log", "dt_bias") else inp[n]) for n in inp}
    o1, fs1, _ = oracle.flash_kda(one, "BNSD", 1, Nqk, Nv, S, D, SCALE, lb, np.array([0, 20]))
    assert np.array_equal(o1[0], o_bnsd[1]) and np.array_equal(fs1[0], fs_bnsd[1])
    # GQA == explicitly repeated q/k heads
    rep = dict(inp)
    rep["q"] = np.repeat(inp["q"], 2, axis=1)
    rep["k"] = np.repeat(inp["k"], 2, axis=1)
    o_rep, fs_rep, _ = oracle.flash_kda(rep, "BNSD", B, 2, Nv, S, D, SCALE, lb, cu)
    assert np.array_equal(o_rep, o_bnsd) and np.array_equal(fs_rep, fs_bnsd)
    # chaining two calls through final_state == one call (split inside a chunk)
    for form, split in (("recurrent", 13), ("chunked", 16)):
        full, fsf, _ = oracle.flash_kda(inp, "BNSD", B, Nqk, Nv, S, D, SCALE, lb, None, form=form,
                                        C=16)
        a = {n: (inp[n][:, :, :split] if n in ("q", "k", "v", "g", "beta") else inp[n])
             for n in inp}
        o_a, fs_a, _ = oracle.flash_kda(a, "BNSD", B, Nqk, Nv, split, D, SCALE, lb, None,
                                        form=form, C=16)
        bb = {n: (inp[n][:, :, split:] if n in ("q", "k", "v", "g", "beta") else inp[n])
              for n in inp}
        bb["initial_state"] = fs_a.astype(np.float64)
        o_b, fs_b, _ = oracle.flash_kda(bb, "BNSD", B, Nqk, Nv, S - split, D, SCALE, lb, None,
                                        form=form, C=16)
        assert _rel(np.concatenate([o_a, o_b], axis=2), full) < tol, form
        assert _rel(fs_b, fsf) < tol, form
    # raw q, k scaled by a power of two: output unchanged up to the eps term
    sc = dict(inp)
    for n in ("q", "k"):
        sc[n] = (inp[n].astype(np.uint32) + (3 << 7)).astype(np.uint16)   # x * 2^3 (exponent +3)
    o_sc, fs_sc, _ = oracle.flash_kda(sc, "BNSD", B, Nqk, Nv, S, D, SCALE, lb, cu)
    assert _rel(o_sc, o_bnsd) < 1e-6 and _rel(fs_sc, fs_bnsd) < 1e-6


ALL_PINS = [pin_chunked_equals_recurrent, pin_chunked_equals_recurrent_d128,
            pin_chunked_equals_recurrent_d64, pin_affine_span_map,
            pin_beta_zero_pure_decay, pin_g_zero_textbook_delta_rule, pin_basis_keys_overwrite,
            pin_repeated_key_ema, pin_brute_force_tiny, pin_unit_lower_inverse, pin_activations,
            pin_structure]

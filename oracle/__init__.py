"""fp64 CPU oracle for chunked KDA prefill -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  It shares no code with the CUDA library
(``chunked_kda_prefill_b200``) and neither imports the other; both take their
inputs from ``kda_workloads``.

The arithmetic lives in ``kda_oracle.c`` (plain fp64 C, one function per step,
each citing the passage it follows).  This module only compiles and loads it,
widens bf16 bit patterns to fp64, and walks the three tensor layouts of the
FlashKDA problem statement (BNSD / BSND / packed TND with cu_seqlens) unit by
unit, where a unit is one (sequence, value head).

Readings the pages leave open:
  * gate g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h])): parity
    unpinned, since the pages name the inputs but print no formula;
  * L2 normalise with eps = 1e-6 inside the square root;
  * GQA: value head h reads q/k head h // (Nv // Nqk);
  * BNSD/BSND with cu_seqlens: sequence b occupies storage rows [0, len_b) of slot b;
  * rows past a valid length are defined as zero in ``out``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE fp64, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    L = ctypes.CDLL(path)
    i, d = ctypes.c_int, ctypes.c_double
    L.kda_oracle_gate.argtypes = [i, i, _dp, _dp, d, d, _dp]
    L.kda_oracle_beta.argtypes = [i, _dp, _dp]
    L.kda_oracle_l2norm.argtypes = [i, i, _dp, d, _dp]
    L.kda_oracle_recurrent.argtypes = [i, i, i, _dp, _dp, _dp, _dp, _dp, d, _dp, _dp, _dp]
    L.kda_oracle_chunked.argtypes = [i, i, i, i, _dp, _dp, _dp, _dp, _dp, d, _dp, _dp, _dp]
    L.kda_oracle_unit_lower_inverse.argtypes = [i, _dp, _dp]
    L.kda_oracle_unit.argtypes = [i, i, i, i, i, _dp, _dp, _dp, _dp, _dp, _dp, d, d, d,
                                  _dp, _dp, _dp]
    for f in ("kda_oracle_gate", "kda_oracle_beta", "kda_oracle_l2norm",
              "kda_oracle_recurrent", "kda_oracle_chunked",
              "kda_oracle_unit_lower_inverse", "kda_oracle_unit"):
        getattr(L, f).restype = None
    return L


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB_PATH)
    return _lib


def compile_source(text: str, path: str) -> str:
    """Compile C source `text` (a variant of kda_oracle.c) to the shared library `path`, with
    the flags of build().  Used by the planted-mistake tests, which patch a copy of the source."""
    os.makedirs(os.path.dirname(path), exist_ok=True)
    src = path + ".c"
    with open(src, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-o", path, src, "-lm"])
    return path


def source() -> str:
    """The text of kda_oracle.c."""
    with open(_SRC) as f:
        return f.read()


class use_library:
    """Context manager: route every oracle call through another compiled copy of the oracle
    (a planted-mistake variant from compile_source) and restore the real one on exit."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        lib()
        with _lock:
            self._saved = _lib
            _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self._saved
        return False


def _c(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


# ----------------------------------------------------------------------------
# Step-level entry points (fp64 arrays in, fp64 arrays out)
# ----------------------------------------------------------------------------

def gate(g_raw, dt_bias, A_log: float, lower_bound: float) -> np.ndarray:
    g_raw = _c(g_raw)
    n, D = g_raw.shape
    out = np.empty_like(g_raw)
    lib().kda_oracle_gate(n, D, _p(g_raw), _p(_c(dt_bias)), float(A_log), float(lower_bound),
                          _p(out))
    return out


def beta_sigmoid(logits) -> np.ndarray:
    x = _c(logits)
    out = np.empty_like(x)
    lib().kda_oracle_beta(x.size, _p(x), _p(out))
    return out


def l2norm(x, eps: float = 1e-6) -> np.ndarray:
    x = _c(x)
    n, D = x.shape
    out = np.empty_like(x)
    lib().kda_oracle_l2norm(n, D, _p(x), float(eps), _p(out))
    return out


def recurrent(q, k, v, g, beta, scale: float, S0):
    """Token-by-token recurrence on already-activated inputs. Returns (out [L,Dv], S [Dv,Dk])."""
    q, k, v, g, beta, S0 = map(_c, (q, k, v, g, beta, S0))
    L, Dk = k.shape
    Dv = v.shape[1]
    out = np.zeros((L, Dv))
    S = np.empty((Dv, Dk))
    lib().kda_oracle_recurrent(L, Dk, Dv, _p(q), _p(k), _p(v), _p(g), _p(beta), float(scale),
                               _p(S0), _p(out), _p(S))
    return out, S


def chunked(q, k, v, g, beta, scale: float, S0, C: int = 64):
    """Chunked (WY) form with chunk size C on already-activated inputs."""
    q, k, v, g, beta, S0 = map(_c, (q, k, v, g, beta, S0))
    L, Dk = k.shape
    Dv = v.shape[1]
    out = np.zeros((L, Dv))
    S = np.empty((Dv, Dk))
    lib().kda_oracle_chunked(L, Dk, Dv, int(C), _p(q), _p(k), _p(v), _p(g), _p(beta),
                             float(scale), _p(S0), _p(out), _p(S))
    return out, S


def unit_lower_inverse(T) -> np.ndarray:
    T = _c(T)
    n = T.shape[0]
    X = np.empty_like(T)
    lib().kda_oracle_unit_lower_inverse(n, _p(T), _p(X))
    return X


def unit(q_raw, k_raw, v, g_raw, beta_logit, dt_bias, A_log, lower_bound, scale, S0,
         form: str = "chunked", C: int = 64):
    """One unit from raw inputs: normalise, activate, then recur. fp64 in/out."""
    q_raw, k_raw, v, g_raw, beta_logit, dt_bias, S0 = map(
        _c, (q_raw, k_raw, v, g_raw, beta_logit, dt_bias, S0))
    L, Dk = k_raw.shape
    Dv = v.shape[1]
    out = np.zeros((L, Dv))
    S = np.empty((Dv, Dk))
    lib().kda_oracle_unit(0 if form == "recurrent" else 1, int(C), L, Dk, Dv, _p(q_raw),
                          _p(k_raw), _p(v), _p(g_raw), _p(beta_logit), _p(dt_bias),
                          float(A_log), float(lower_bound), float(scale), _p(S0), _p(out),
                          _p(S))
    return out, S


# ----------------------------------------------------------------------------
# Whole-op entry point over the FlashKDA layouts
# ----------------------------------------------------------------------------

def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern (uint16) -> fp64, exactly."""
    b = np.ascontiguousarray(bits).view(np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rows(a: np.ndarray, layout: str, b: int, head: int, start: int, length: int,
          cu: np.ndarray) -> np.ndarray:
    """Rows [start, start+length) of sequence b, head ``head`` (last axis kept)."""
    if layout == "BNSD":
        return a[b, head, start:start + length]
    if layout == "BSND":
        return a[b, start:start + length, head]
    if layout == "TND":
        t0 = int(cu[b]) + start
        return a[t0:t0 + length, head]
    raise ValueError(layout)


def units_of(layout: str, B: int, Nv: int, S: int, cu_seqlens) -> list:
    """All (b, h, length) units."""
    cu = _lengths(layout, B, S, cu_seqlens)
    return [(b, h, int(cu[b + 1] - cu[b])) for b in range(B) for h in range(Nv)]


def _lengths(layout, B, S, cu_seqlens):
    if cu_seqlens is None:
        if layout == "TND":
            raise ValueError("TND needs cu_seqlens")
        return np.arange(B + 1, dtype=np.int64) * S
    return np.asarray(cu_seqlens, dtype=np.int64)


def run_units(inp: dict, layout: str, B: int, Nqk: int, Nv: int, S: int, D: int, scale: float,
              lower_bound: float, cu_seqlens=None, units=None, form: str = "chunked", C: int = 64,
              threads: int | None = None) -> dict:
    """The op on raw inputs for a list of (b, h) units; returns {(b, h): (out [L, D], S [D, D])}.

    ``inp`` holds bf16 bit arrays (q, k, v, g, beta) and fp32 A_log, dt_bias, initial_state.
    """
    cu = _lengths(layout, B, S, cu_seqlens)
    G = Nv // Nqk
    q = inp["q"]; k = inp["k"]; v = inp["v"]; g = inp["g"]; beta = inp["beta"]
    A_log = np.asarray(inp["A_log"], dtype=np.float64)
    dt_bias = np.asarray(inp["dt_bias"], dtype=np.float64)
    S0 = inp["initial_state"]
    if units is None:
        units = [(b, h) for b in range(B) for h in range(Nv)]
    tnd_cu = cu if layout == "TND" else None

    def run(bh):
        b, h = bh
        L = int(cu[b + 1] - cu[b])
        hq = h // G
        qr = widen_bf16(_rows(q, layout, b, hq, 0, L, tnd_cu))
        kr = widen_bf16(_rows(k, layout, b, hq, 0, L, tnd_cu))
        vr = widen_bf16(_rows(v, layout, b, h, 0, L, tnd_cu))
        gr = widen_bf16(_rows(g, layout, b, h, 0, L, tnd_cu))
        if layout == "BNSD":
            br = widen_bf16(beta[b, h, 0:L])
        elif layout == "BSND":
            br = widen_bf16(beta[b, 0:L, h])
        else:
            br = widen_bf16(beta[int(cu[b]):int(cu[b]) + L, h])
        return bh, unit(qr, kr, vr, gr, br, dt_bias[h], A_log[h], lower_bound, scale,
                        np.asarray(S0[b, h], dtype=np.float64), form=form, C=C)

    nthreads = threads or max(1, min(len(units), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        return dict(ex.map(run, units))


def flash_kda(inp: dict, layout: str, B: int, Nqk: int, Nv: int, S: int, D: int, scale: float,
              lower_bound: float, cu_seqlens=None, form: str = "chunked", C: int = 64,
              units=None, threads: int | None = None):
    """The whole op on raw inputs (bf16 bit arrays + fp32 params), in fp64.

    Returns ``(out, final_state, done)``: ``out`` has v's shape (zeros outside the
    valid rows and for units not computed), ``final_state`` is [B, Nv, D, D] and
    ``done`` lists the (b, h) units computed.
    """
    cu = _lengths(layout, B, S, cu_seqlens)
    res = run_units(inp, layout, B, Nqk, Nv, S, D, scale, lower_bound, cu_seqlens, units, form,
                    C, threads)
    out = np.zeros(inp["v"].shape, dtype=np.float64)
    fs = np.zeros((B, Nv, D, D), dtype=np.float64)
    for (b, h), (o, Sf) in res.items():
        L = int(cu[b + 1] - cu[b])
        if layout == "BNSD":
            out[b, h, 0:L] = o
        elif layout == "BSND":
            out[b, 0:L, h] = o
        else:
            out[int(cu[b]):int(cu[b]) + L, h] = o
        fs[b, h] = Sf
    return out, fs, list(res.keys())

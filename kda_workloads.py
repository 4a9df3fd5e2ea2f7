"""Seeded synthetic inputs for chunked KDA prefill.

This module is the one piece shared by the oracle-side tests and the CUDA path:
it draws random tensors and rounds them to bf16, and it holds none of the
method's arithmetic (no gate, no normalisation, no recurrence).

Workloads follow the FlashKDA problem statement (CANNBot-DSL ``flash_kda``
README, "参数说明" parameter table): q/k/v/g/beta are bf16 ~ N(0, 1) in one of the
BNSD / BSND / TND layouts, A_log [Nv] and dt_bias [Nv, D] are fp32 ~ N(0, 1),
initial_state is fp32 [B, Nv, D, D] (zeros or N(0, 0.1^2)), D = 128.

Draws: tensor number j of q, k, v, g, beta, A_log, dt_bias, initial_state (j = 0..7) is
filled in row-major blocks of 2^22 elements, block i from
``numpy.random.default_rng([seed, j, i]).standard_normal(dtype=float32)``, in parallel on the
host threads.  bf16 values are produced by round-to-nearest-even from the fp32 draws.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

LAYOUTS = ("BNSD", "BSND", "TND")


# ----------------------------------------------------------------------------
# bf16 helpers (storage format only)
# ----------------------------------------------------------------------------

_BLOCK = 1 << 22  # elements per block of the parallel draws and conversions


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even); return the uint16 bit pattern.  NaN becomes
    the quiet NaN 0x7FC0.  Works block by block on all host threads."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)

    def block(i):
        f = flat[i:i + _BLOCK]
        u = f.view(np.uint32)
        r = u >> np.uint32(16)
        r &= np.uint32(1)
        r += np.uint32(0x7FFF)
        r += u
        r >>= np.uint32(16)
        o = out[i:i + _BLOCK]
        o[...] = r
        nan = np.isnan(f)
        if nan.any():
            o[nan] = np.uint16(0x7FC0)

    starts = range(0, flat.size, _BLOCK)
    if flat.size <= _BLOCK:
        for i in starts:
            block(i)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(block, starts))
    return out.reshape(x.shape)


def normal_f32(seed: int, stream: int, shape) -> np.ndarray:
    """fp32 draws ~ N(0, 1) of the given shape: block i of 2^22 elements (row-major order) comes
    from numpy.random.default_rng([seed, stream, i]), so the blocks are drawn in parallel and
    every element depends only on (seed, stream, its index)."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.float32)

    def block(j):
        i = j * _BLOCK
        rng = np.random.default_rng([seed, stream, j])
        out[i:i + _BLOCK] = rng.standard_normal(size=min(_BLOCK, n - i), dtype=np.float32)

    nb = (n + _BLOCK - 1) // _BLOCK
    if nb <= 1:
        for j in range(nb):
            block(j)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(block, range(nb)))
    return out.reshape(shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen a bf16 bit pattern (uint16) to fp32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    layout: str
    B: int              # number of sequences (batch slots for BNSD/BSND)
    Nqk: int
    Nv: int
    S: int              # storage length per batch slot; T (packed tokens) for TND
    D: int
    lengths: list       # valid length of each sequence
    lower_bound: float
    scale: float
    init_state: str     # "zeros" or "normal"
    seed: int
    init_std: float = 0.1
    extra: dict = field(default_factory=dict)

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lengths)]).astype(np.int32)

    @property
    def token_heads(self) -> int:
        """Valid tokens x value heads (the throughput unit)."""
        return int(sum(self.lengths)) * self.Nv

    @property
    def units(self) -> int:
        return self.B * self.Nv

    def describe(self) -> dict:
        return {"workload": self.name, "layout": self.layout, "B": self.B, "Nqk": self.Nqk,
                "Nv": self.Nv, "S": self.S, "D": self.D, "lower_bound": self.lower_bound,
                "scale": self.scale, "initial_state": self.init_state, "seed": self.seed,
                "valid_token_heads": self.token_heads}


def packed_lengths(n_seq: int, total: int, max_len: int, seed: int) -> list:
    """Packed varlen lengths: n_seq uniform draws in [1, max_len] rescaled to sum to total.

    Draw n_seq integers U[1, max_len], scale by total/sum, floor, clamp to
    [1, max_len]; then hand the remainder out +1 each, in index order, to
    sequences still below max_len (repeating passes until it is spent).
    """
    rng = np.random.default_rng(seed)
    raw = rng.integers(1, max_len + 1, size=n_seq)
    lens = np.floor(raw * (total / raw.sum())).astype(np.int64)
    lens = np.clip(lens, 1, max_len)
    rem = total - int(lens.sum())
    while rem > 0:
        progressed = False
        for i in range(n_seq):
            if rem == 0:
                break
            if lens[i] < max_len:
                lens[i] += 1
                rem -= 1
                progressed = True
        if not progressed:
            raise ValueError("cannot distribute remainder")
    while rem < 0:  # clamping at 1 can overshoot; take back from the longest
        i = int(np.argmax(lens))
        lens[i] -= 1
        rem += 1
    return [int(x) for x in lens]


SCALE128 = 1.0 / math.sqrt(128.0)


def workload(idx: int) -> Workload:
    """The five synthetic workloads (1-based index); 6: head dim 64; 7: the large prefill at B = 1."""
    if idx == 1:
        return Workload("tiny_bnsd_1x1x256", "BNSD", 1, 1, 1, 256, 128, [256], -5.0, SCALE128,
                        "zeros", seed=1)
    if idx == 2:
        return Workload("single_seq_bnsd_1x3x8192", "BNSD", 1, 3, 3, 8192, 128, [8192], -5.0,
                        SCALE128, "zeros", seed=2)
    if idx == 3:
        return Workload("gqa_tail_bsnd_2x4x16_s4000", "BSND", 2, 4, 16, 4000, 128, [4000, 2777],
                        -2.0, SCALE128, "normal", seed=3)
    if idx == 4:
        lens = packed_lengths(12, 65536, 16384, seed=0)
        return Workload("packed_tnd_t65536_12seq_h32", "TND", 12, 32, 32, 65536, 128, lens, -5.0,
                        SCALE128, "normal", seed=4)
    if idx == 5:
        return Workload("large_bnsd_4x32x16384", "BNSD", 4, 32, 32, 16384, 128, [16384] * 4, -5.0,
                        SCALE128, "zeros", seed=5)
    if idx == 6:
        # head dim 64: the largest K = 64 shape of FLA PR 656's timing table (B=8, T=4096, H=32)
        return Workload("headdim64_bnsd_8x32x4096", "BNSD", 8, 32, 32, 4096, 64, [4096] * 8,
                        -5.0, 1.0 / math.sqrt(64.0), "zeros", seed=6)
    if idx == 7:
        # one batch row of the large prefill: 32 units for 148 SMs, so the default schedule cuts
        # each unit into segments (chunk-parallel scan)
        return Workload("single_batch_bnsd_1x32x16384", "BNSD", 1, 32, 32, 16384, 128, [16384],
                        -5.0, SCALE128, "zeros", seed=7)
    raise ValueError(idx)


def custom(name, layout, B, Nqk, Nv, S, lengths, lower_bound=-5.0, scale=SCALE128,
           init_state="normal", seed=0, D=128) -> Workload:
    return Workload(name, layout, B, Nqk, Nv, S, D, list(lengths), lower_bound, scale, init_state,
                    seed)


# ----------------------------------------------------------------------------
# Shapes and generation
# ----------------------------------------------------------------------------

def shapes(w: Workload) -> dict:
    if w.layout == "BNSD":
        return {"q": (w.B, w.Nqk, w.S, w.D), "v": (w.B, w.Nv, w.S, w.D), "beta": (w.B, w.Nv, w.S)}
    if w.layout == "BSND":
        return {"q": (w.B, w.S, w.Nqk, w.D), "v": (w.B, w.S, w.Nv, w.D), "beta": (w.B, w.S, w.Nv)}
    if w.layout == "TND":
        return {"q": (w.S, w.Nqk, w.D), "v": (w.S, w.Nv, w.D), "beta": (w.S, w.Nv)}
    raise ValueError(w.layout)


def generate(w: Workload, pad_value: float | None = None) -> dict:
    """Draw the inputs of ``w``.

    Returns bf16 tensors as uint16 bit arrays (``q``, ``k``, ``v``, ``g``,
    ``beta``), fp32 ``A_log``, ``dt_bias``, ``initial_state`` and int32
    ``cu_seqlens``.  If ``pad_value`` is given, every storage row outside a
    valid length (BNSD/BSND rows >= len_b) is overwritten with it, e.g. NaN to
    prove padding is never read.
    """
    sh = shapes(w)
    out = {}
    for stream, (name, key) in enumerate((("q", "q"), ("k", "q"), ("v", "v"), ("g", "v"),
                                          ("beta", "beta"))):
        out[name] = f32_to_bf16_bits(normal_f32(w.seed, stream, sh[key]))
    out["A_log"] = normal_f32(w.seed, 5, (w.Nv,))
    out["dt_bias"] = normal_f32(w.seed, 6, (w.Nv, w.D))
    if w.init_state == "zeros":
        out["initial_state"] = np.zeros((w.B, w.Nv, w.D, w.D), dtype=np.float32)
    else:
        out["initial_state"] = normal_f32(w.seed, 7, (w.B, w.Nv, w.D, w.D)) * np.float32(w.init_std)
    out["cu_seqlens"] = w.cu_seqlens
    if pad_value is not None and w.layout != "TND":
        pv = f32_to_bf16_bits(np.array([pad_value], dtype=np.float32))[0]
        for b, L in enumerate(w.lengths):
            for name in ("q", "k", "v", "g", "beta"):
                a = out[name]
                if w.layout == "BNSD":
                    a[b, :, L:] = pv
                else:
                    a[b, L:] = pv
    return out

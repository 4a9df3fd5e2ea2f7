"""The degenerate corners of the method's inputs, CUDA path vs the fp64 oracle (atol = rtol =
5e-3 on valid rows, exact zeros past the valid lengths).

- zero query/key rows: the normalisation maps them to zero (its epsilon keeps 0/0 away), and a
  whole chunk of zero keys leaves the state to decay alone;
- saturated gates: raw gates of +-30 put g at the lower bound (-5, the fastest decay the pages
  allow, where the chunk's cumulative decay underflows fp32 without the per-block reference
  points) or at 0 (no decay);
- saturated write strengths: beta logits of +-30 give beta = 1 (a full overwrite along k) or 0
  (no write).
"""
import numpy as np
import pytest

import kda_workloads as W
import oracle
from kda_gpu import compare, run_gpu, valid_mask

pytestmark = pytest.mark.gpu

CASES = ["zero_rows", "saturated_gates", "saturated_beta", "all_three"]


def _degenerate_inputs(case):
    w = W.custom(f"deg_{case}", "BSND", 2, 1, 2, 200, [200, 131], lower_bound=-5.0,
                 init_state="normal", seed=71)
    inp = W.generate(w)
    rng = np.random.default_rng(72)
    bf = W.f32_to_bf16_bits
    if case in ("zero_rows", "all_three"):
        for n in ("q", "k"):
            rows = rng.random(inp[n].shape[:3]) < 0.2          # [B, S, Nqk]
            inp[n][rows] = 0
        inp["k"][0, 64:128] = 0                                # a whole chunk of zero keys
    if case in ("saturated_gates", "all_three"):
        sign = np.where(rng.random(inp["g"].shape) < 0.5, -30.0, 30.0).astype(np.float32)
        inp["g"] = bf(sign)
        inp["A_log"] = np.zeros_like(inp["A_log"])             # e^A_log = 1
        inp["dt_bias"] = np.zeros_like(inp["dt_bias"])
    if case in ("saturated_beta", "all_three"):
        sign = np.where(rng.random(inp["beta"].shape) < 0.5, -30.0, 30.0).astype(np.float32)
        inp["beta"] = bf(sign)
    return w, inp


@pytest.mark.parametrize("case", CASES)
def test_degenerate_inputs(case, cuda_ok):
    w, inp = _degenerate_inputs(case)
    o_g, fs_g = run_gpu(w, inp)
    o_r, fs_r, _ = oracle.flash_kda(inp, w.layout, w.B, w.Nqk, w.Nv, w.S, w.D, w.scale,
                                    w.lower_bound, w.cu_seqlens)
    m = valid_mask(w, o_g.shape)
    compare(o_g[m], o_r[m], f"{case} out")
    compare(fs_g, fs_r, f"{case} final_state")
    assert np.all(o_g[~m] == 0.0)

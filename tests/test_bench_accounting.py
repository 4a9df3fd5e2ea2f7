"""The roofline numerator of bench.py, pinned to counts done by hand for two workloads.

Large prefill, B=4, Nqk=Nv=32, S=16384, D=128 (65,536 rows, all valid):
  q, k 2*65536*32*128*2 = 1,073,741,824;  v, g 2*65536*32*128*2 = 1,073,741,824;
  beta 65536*32*2 = 4,194,304;  out 65536*32*128*2 = 536,870,912;
  initial + final state 2*4*32*128*128*4 = 16,777,216;  A_log + dt_bias 32*4 + 32*128*4 = 16,512;
  total 2,705,342,592 bytes.
GQA tail, BSND, B=2, S=4000, Nqk=4, Nv=16, lengths 4000 and 2777 (6,777 valid rows of 8,000):
  q, k 2*6777*4*128*2 = 13,879,296;  v, g 2*6777*16*128*2 = 55,517,184;  beta 6777*16*2 = 216,864;
  out (every storage row: padding rows are written as zeros) 8000*16*128*2 = 32,768,000;
  states 2*2*16*128*128*4 = 4,194,304;  A_log + dt_bias 16*4 + 16*128*4 = 8,256;
  total 106,583,904 bytes.
Flops of the large prefill: 32,768 chunk-heads * (5*2*64*64*128 + 3*2*64*128*128) =
32,768 * 11,534,336 = 377,957,122,048.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import kda_workloads as W  # noqa: E402


def test_large_prefill_bytes_and_flops():
    w = W.workload(5)
    assert bench.algorithmic_bytes(w, True) == 2_705_342_592
    assert bench.algorithmic_bytes(w, False) == 2_705_342_592 - 4 * 32 * 128 * 128 * 4
    assert bench.algorithmic_flops(w) == 377_957_122_048


def test_ragged_workload_counts_valid_input_rows_only():
    assert bench.algorithmic_bytes(W.workload(3), True) == 106_583_904

"""The sm_100a plumbing under the fused kernel, one piece at a time, against torch.

Each case runs one M=128 tcgen05 MMA (bf16 in, fp32 out) with operands in the 128B-swizzled
shared-memory layouts (K-major or MN-major) or with A in TMEM, and one TMA load whose
swizzled shared-memory image must match the layout the kernels write by hand.
"""
import ctypes

import numpy as np
import pytest
import torch

import chunked_kda_prefill_b200 as kda

pytestmark = pytest.mark.gpu


def _lib():
    L = kda.load()
    f = L.kda_selftest
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


CASES = [  # variant, N, K   (0 SS K/K, 1 SS MN/K, 2 SS K/MN, 3 TS K, 5 TS MN)
    (0, 64, 128), (0, 16, 128), (0, 48, 128), (0, 128, 64), (1, 64, 64), (1, 64, 128),
    (2, 128, 64), (2, 64, 128), (3, 64, 128), (3, 128, 64), (5, 128, 64), (5, 64, 128)]


@pytest.mark.parametrize("variant,N,K", CASES)
def test_mma_plumbing(variant, N, K, cuda_ok):
    f = _lib()
    g = torch.Generator().manual_seed(100 + variant * 7 + N + K)
    A = torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    a_in = A.t().contiguous() if variant == 1 else A
    b_in = B.t().contiguous() if variant in (2, 5) else B
    a_d, b_d = a_in.cuda(), b_in.cuda()
    D = torch.full((128, N), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    rc = f(variant, a_d.data_ptr(), b_d.data_ptr(), D.data_ptr(), N, K, None, None, 0, 0,
           err.data_ptr(), s.cuda_stream)
    assert rc == 0
    ref = A.double() @ B.double().t()
    got = D.cpu().double()
    assert torch.allclose(got, ref, rtol=1e-5, atol=1e-4), (got - ref).abs().max()


def _sw128(rows, r, c):
    atom, chunk = c >> 6, (c >> 3) & 7
    return atom * rows * 128 + r * 128 + ((chunk ^ (r & 7)) << 4) + ((c & 7) << 1)


def test_tma_swizzle_matches_hand_layout(cuda_ok):
    f = _lib()
    src = torch.arange(256 * 128, dtype=torch.int32).remainder(65521).to(torch.int16)
    src_d = src.view(256, 128).cuda()
    raw = torch.zeros(8192, dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    row0 = 64
    rc = f(4, None, None, None, 0, 0, raw.data_ptr(), src_d.data_ptr(), 256, row0, err.data_ptr(),
           torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    raw_h = raw.cpu().numpy()
    s = src.view(256, 128).numpy()
    for r in range(64):
        for c in range(128):
            assert raw_h[_sw128(64, r, c) // 2] == s[row0 + r, c], (r, c)


def _tf32(x):
    """Round-toward-zero to tf32 (keep 10 mantissa bits) so the MMA sees exactly these values."""
    u = x.contiguous().view(torch.int32) & ~0x1FFF
    return u.view(torch.float32)


@pytest.mark.parametrize("variant,N,K", [(6, 64, 64), (6, 128, 32), (7, 64, 64), (7, 128, 32)])
def test_tf32_mma_plumbing(variant, N, K, cuda_ok):
    f = _lib()
    g = torch.Generator().manual_seed(300 + variant * 11 + N + K)
    A = _tf32(torch.randn(128, K, generator=g))
    B = _tf32(torch.randn(N, K, generator=g))
    a_d, b_d = A.cuda(), B.cuda()
    D = torch.full((128, N), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = f(variant, a_d.data_ptr(), b_d.data_ptr(), D.data_ptr(), N, K, None, None, 0, 0,
           err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    ref = A.double() @ B.double().t()
    got = D.cpu().double()
    assert torch.allclose(got, ref, rtol=1e-5, atol=1e-4), (got - ref).abs().max()

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


def test_bounded_wait_gives_up_and_the_context_survives(cuda_ok):
    """Failure detection without a fault: a bounded mbarrier wait on a barrier that nothing
    arrives on must run out, report it through the status word, and leave the context usable."""
    f = _lib()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert f(8, None, None, None, 0, 0, None, None, 0, 0, err.data_ptr(), s) == 3
    assert int(err.item()) == 3
    # the same context still runs a normal MMA case correctly
    g = torch.Generator().manual_seed(5)
    A = torch.randn(128, 64, generator=g).to(torch.bfloat16)
    B = torch.randn(64, 64, generator=g).to(torch.bfloat16)
    D = torch.full((128, 64), float("nan"), dtype=torch.float32, device="cuda")
    assert f(0, A.cuda().data_ptr(), B.cuda().data_ptr(), D.data_ptr(), 64, 64, None, None, 0, 0,
             err.data_ptr(), s) == 0
    ref = A.double() @ B.double().t()
    assert torch.allclose(D.cpu().double(), ref, rtol=1e-5, atol=1e-4)


def test_device_timeout_word_maps_to_status_code(cuda_ok):
    """A kernel that gave up a bounded wait leaves DS_TIMEOUT (2) in the workspace status word;
    kda_device_status reports it as KDA_ERR_TIMEOUT, and a plan mismatch (1) as KDA_ERR_PLAN."""
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    kda.device_status(ws)  # 0: fine
    for word, name in ((2, "KDA_ERR_TIMEOUT"), (1, "KDA_ERR_PLAN")):
        ws[0] = word
        with pytest.raises(kda.KdaError) as e:
            kda.device_status(ws)
        assert e.value.name == name


def test_ex2_accuracy(cuda_ok):
    """ex2.approx.ftz.f32 (every decay factor 2^x of the fused kernel) against exp2 in fp64 over
    the arguments the kernel forms: gate arguments and log2-space cumulative-sum differences."""
    L = kda.load()
    f = L.kda_selftest_ex2
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-126.0, 127.0, 1 << 20, dtype=torch.float32),
                   (torch.rand(1 << 20, generator=g) * 253.0 - 126.0).to(torch.float32),
                   torch.tensor([-130.0, -150.0, -500.0], dtype=torch.float32)])
    xd = x.cuda()
    yd = torch.empty_like(xd)
    assert f(xd.data_ptr(), yd.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream) == 0
    xs = x.double().numpy()
    y = yd.cpu().double().numpy()
    ref = np.exp2(xs)
    normal = xs >= -125.0
    rel = np.abs(y[normal] - ref[normal]) / ref[normal]
    assert rel.max() < 2.0 ** -21, rel.max()
    # results below the smallest normal float are flushed to zero (ftz)
    assert np.all(y[xs <= -127.0] <= 2.0 ** -126)
    print(f"ex2.approx.ftz.f32: max relative error {rel.max():.3e} = 2^{np.log2(rel.max()):.2f}")


def test_m64_accumulator_layout(cuda_ok):
    """Where the rows and columns of an M=64 tcgen05 accumulator land in TMEM (cta_group::1,
    kind::f16).  A = I (64 x 64), so D[m][n] = B[n][m]: one run with B[n][k] = k + 1 marks every
    cell with its row, one with B[n][k] = n + 1 with its column.  Every (row, column) must land
    in exactly one (lane, TMEM column) of the 128 lanes x 128 columns read back."""
    f = _lib()
    N, K = 64, 64
    A = torch.eye(64, K).to(torch.bfloat16).cuda()
    kk = torch.arange(K, dtype=torch.float32)
    nn = torch.arange(N, dtype=torch.float32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    raw = []
    for B in ((kk[None, :] + 1).expand(N, K), (nn[:, None] + 1).expand(N, K)):
        D = torch.full((128, 2 * N), -1.0, dtype=torch.float32, device="cuda")
        Bd = B.contiguous().to(torch.bfloat16).cuda()
        assert f(9, A.data_ptr(), Bd.data_ptr(), D.data_ptr(), N, K, None, None, 0, 0,
                 err.data_ptr(), s.cuda_stream) == 0
        raw.append(D.cpu().numpy())
    rows, cols = raw
    cells = {}
    for lane in range(128):
        for col in range(2 * N):
            if rows[lane, col] > 0:
                m, n = int(rows[lane, col]) - 1, int(cols[lane, col]) - 1
                assert (m, n) not in cells, f"row {m} column {n} found twice"
                cells[(m, n)] = (lane, col)
    assert len(cells) == 64 * N, f"{len(cells)} of {64 * N} cells found"
    # measured on B200: row m in lane (m % 16) + 32 (m / 16), i.e. the first 16 lanes of each
    # warp's lane quarter; column n in TMEM column n
    for (m, n), (lane, col) in cells.items():
        assert lane == (m % 16) + 32 * (m // 16) and col == n, (m, n, lane, col)

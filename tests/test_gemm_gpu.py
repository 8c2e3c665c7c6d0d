"""The persistent tcgen05 GEMM on its own (pl_debug_gemm), against an fp64 matmul.

Covers K-major and MN-major operands on both sides, bf16 and fp16, tile-exact
and ragged shapes (M, N, K not multiples of the 128 x 256 x 64 tiling).
Tolerance: |D - ref| <= 1e-5 * sum_k |A(m,k) B(n,k)| + 1e-6 (fp32 accumulation
of exactly representable 16-bit products).
"""
import pytest
import torch

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gemm_tile")]


def _lib():
    import rl_post_policy_b200 as m
    return m, m.pl_debug_gemm


def run(M, N, K, a_mn, b_mn, dtype, seed=0):
    m, f = _lib()
    g = torch.Generator().manual_seed(seed)
    A32 = torch.randn(M, K, generator=g)
    B32 = torch.randn(N, K, generator=g)
    A = A32.to(dtype)
    B = B32.to(dtype)
    def pitched(t, rows, cols):
        ld = (cols + 7) // 8 * 8
        out = torch.zeros(rows, ld, dtype=t.dtype)
        out[:, :cols] = t
        return out.cuda(), ld

    Ad, lda = pitched(A.t(), K, M) if a_mn else pitched(A, M, K)
    Bd, ldb = pitched(B.t(), K, N) if b_mn else pitched(B, N, K)
    D = torch.full((M, N), float("nan"), device="cuda")
    rc = f(Ad, a_mn, lda, Bd, b_mn, ldb, D, M, N, K, m.dtype_mode(dtype))
    m.check(rc, "pl_debug_gemm")
    torch.cuda.synchronize()
    m.check(m.pl_device_status(None), "device status")
    ref = A.double() @ B.double().t()
    bound = A.double().abs() @ B.double().abs().t()
    err = (D.cpu().double() - ref).abs()
    assert torch.all(err <= 1e-5 * bound + 1e-6), float((err - 1e-5 * bound).max())


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
def test_tile_exact(a_mn, b_mn, dtype):
    run(256, 512, 192, a_mn, b_mn, dtype)


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("shape", [(100, 300, 200), (1, 8, 8), (130, 264, 72), (384, 1000, 1032)])
def test_ragged(a_mn, b_mn, shape):
    M, N, K = shape
    run(M, N, K, a_mn, b_mn, torch.bfloat16, seed=M + N + K)


def test_many_tiles_persistent():
    # more tiles than SMs: every CTA walks several tiles and both accumulators
    run(1024, 8192, 256, 0, 0, torch.bfloat16, seed=3)
    run(2048, 1024, 1024, 1, 1, torch.bfloat16, seed=4)


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 1)])
@pytest.mark.parametrize("shape", [(256, 512, 192), (333, 300, 136), (1, 4, 8), (700, 2052, 520)])
def test_tma_output_paths(a_mn, b_mn, shape):
    """The staged TMA store (path 1) and TMA add (path 2): D = A.B, then D += A.B
    over a random start, on a pitched D whose pad rows and columns must stay
    untouched (the TMA unit drops what lies past [M, N])."""
    m = __import__("rl_post_policy_b200")
    M, N, K = shape
    g = torch.Generator().manual_seed(M * 7 + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)

    def pitched(t, rows, cols):
        ld = (cols + 7) // 8 * 8
        out = torch.zeros(rows, ld, dtype=t.dtype)
        out[:, :cols] = t
        return out.cuda(), ld

    Ad, lda = pitched(A.t(), K, M) if a_mn else pitched(A, M, K)
    Bd, ldb = pitched(B.t(), K, N) if b_mn else pitched(B, N, K)
    ldd = N + 8
    sentinel = 12345.0
    R = torch.randn(M, N, generator=g)
    ref = A.double() @ B.double().t()
    bound = A.double().abs() @ B.double().abs().t()
    mode = m.dtype_mode(torch.bfloat16)

    def fresh(start):
        D = torch.full((M + 5, ldd), sentinel)
        D[:M, :N] = start
        return D.cuda()

    def check(D, want, extra):
        torch.cuda.synchronize()
        m.check(m.pl_device_status(None), "device status")
        D = D.cpu().double()
        err = (D[:M, :N] - want).abs()
        assert torch.all(err <= 1e-5 * (bound + extra) + 1e-6), float(err.max())
        assert torch.all(D[:M, N:] == sentinel) and torch.all(D[M:] == sentinel)

    D = fresh(float("nan"))
    m.check(m.pl_debug_gemm_out(Ad, a_mn, lda, Bd, b_mn, ldb, D, ldd, 1, M, N, K, mode), "store")
    check(D, ref, 0.0)
    m.check(m.pl_debug_gemm_out(Ad, a_mn, lda, Bd, b_mn, ldb, D, ldd, 2, M, N, K, mode), "add")
    check(D, 2 * ref, bound)
    D = fresh(R)
    m.check(m.pl_debug_gemm_out(Ad, a_mn, lda, Bd, b_mn, ldb, D, ldd, 2, M, N, K, mode), "add")
    check(D, R.double() + ref, R.double().abs())


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 1)])
@pytest.mark.parametrize("N", [40960, 40900], ids=["N_tile_exact", "N_ragged"])
def test_last_wave_in_half_tiles(a_mn, b_mn, N):
    # 80 tiles of 256 x 512 on the 74 pairs of a B200: the last 6 run as 12 tiles
    # 256 wide (with the tile512 fixture), including the partial last column tile
    m = __import__("rl_post_policy_b200")
    assert m.pl_debug_tail_halves(80, 74) == 6
    try:
        for no_tail in (0, 1):
            assert m.pl_debug_set_gemm_tail(no_tail) == 0
            run(256, N, 192, a_mn, b_mn, torch.bfloat16, seed=N + a_mn)
    finally:
        m.pl_debug_set_gemm_tail(0)

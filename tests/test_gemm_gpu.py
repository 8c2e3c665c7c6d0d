"""The persistent tcgen05 GEMM on its own (pl_debug_gemm), against an fp64 matmul.

Covers K-major and MN-major operands on both sides, bf16 and fp16, tile-exact
and ragged shapes (M, N, K not multiples of the 128 x 256 x 64 tiling).
Tolerance: |D - ref| <= 1e-5 * sum_k |A(m,k) B(n,k)| + 1e-6 (fp32 accumulation
of exactly representable 16-bit products).
"""
import numpy as np
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

"""Q4_K GEMV and its input-gradient backward on the GPU against the oracle, element by
element, held to the same bound as every other contraction: |y - y_ref| <= 1e-5 * T with
T = sum |terms| (terms exact in the oracle's f64). The kernels keep every f32 chain short
at any size: the forward sums a super-block's 32 products, then 16 super-blocks, then the
rest, and the backward caps a row range at 2048 rows and adds the ranges in groups of 16."""
import numpy as np
import pytest
import torch

import block_quantized_w4a8_b200 as w4a8
import oracle
from block_quantized_w4a8_b200 import inputs

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _check(got, ref, T, what):
    err = np.abs(got.astype(np.float64) - ref)
    tol = TOL * T
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside; worst {np.max(err / np.maximum(T, 1e-300))}"


# (M, N, K): one token, two, an odd count (a one-token tail launch), ragged N (row groups
# of 4 and CTAs of 32 rows), a single super-block, full decode size, long K (more than 16
# super-blocks per warp: all three levels of the sum)
SHAPES = [(1, 300, 256), (2, 77, 512), (3, 129, 1024), (5, 1000, 2048), (1, 4096, 4096), (1, 64, 65536)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemv_q4_k_vs_oracle(M, N, K):
    W = inputs.make_q4_k(N, K, seed=N + K)
    x = inputs.randn((M, K), seed=M + 1)
    yref, T = oracle.gemv_q4_k(x.numpy(), W.numpy(), N, nthreads=8)
    y = w4a8.gemv_q4_k(x.cuda(), W.cuda())
    torch.cuda.synchronize()
    _check(y.cpu().numpy(), yref, T, f"forward M={M} N={N} K={K}")


# backward: one row range (small N) and several (partial sums reduced in order), many
# ranges (more than 16: grouped reduction), long K with N above one range's 2048 rows
BSHAPES = [(1, 300, 256), (2, 77, 512), (3, 1000, 1024), (1, 4096, 4096), (4, 2048, 4096), (1, 8192, 256),
           (1, 5000, 65536)]


@pytest.mark.parametrize("M,N,K", BSHAPES)
def test_gemv_q4_k_backward_vs_oracle(M, N, K):
    W = inputs.make_q4_k(N, K, seed=N * 3 + K)
    dy = inputs.randn((M, N), seed=M + 2)
    dxref, T = oracle.gemv_q4_k_backward(dy.numpy(), W.numpy(), K, nthreads=8)
    dx = w4a8.gemv_q4_k_backward(dy.cuda(), W.cuda(), K)
    torch.cuda.synchronize()
    _check(dx.cpu().numpy(), dxref, T, f"backward M={M} N={N} K={K}")


def test_backward_is_deterministic():
    M, N, K = 2, 2048, 4096
    W = inputs.make_q4_k(N, K, seed=1).cuda()
    dy = inputs.randn((M, N), seed=2).cuda()
    a = w4a8.gemv_q4_k_backward(dy, W, K)
    b = w4a8.gemv_q4_k_backward(dy, W, K)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_backward_workspace_too_small_is_rejected():
    M, N, K = 1, 4096, 4096
    need = w4a8.w4a8_q4_k_backward_workspace_bytes(M, N, K)
    assert need > 16  # several row ranges at this size
    W = torch.zeros(N, K // 256 * 144, dtype=torch.uint8, device="cuda")
    dy = torch.zeros(M, N, device="cuda")
    dx = torch.empty(M, K, device="cuda")
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(w4a8.W4A8Error) as e:
        w4a8.w4a8_gemv_q4_k_backward(dy, W, dx, ws)
    assert e.value.status == 3

"""Affine weights with 6- and 8-bit codes and with groups of 32 on the GPU, against the
oracle: the pack bit for bit (codes, scales, biases), the contraction element by element
within the tolerance of the 4-bit paths (|y - y_ref| <= 1e-5 * T) on the GEMV and on the
CTA-pair tensor-core kernel (with and without a split of K), with and without the output
epilogue, on ragged shapes; the scale range of the tensor path; 4-bit codes in groups of
32 on every kernel path."""
import numpy as np
import pytest
import torch

import block_quantized_w4a8_b200 as w4a8
import oracle
from block_quantized_w4a8_b200 import inputs

pytestmark = pytest.mark.gpu
TOL = 1e-5
PATHS = {"auto": w4a8.PATH_AUTO, "gemv": w4a8.PATH_GEMV, "gemm": w4a8.PATH_GEMM}


def as_np(t):
    return t.detach().cpu().numpy()


def check_tol(y, yref, T, what):
    err = np.abs(np.asarray(y, dtype=np.float64) - yref)
    bad = err > TOL * T
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside; worst {err.max()}"


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pack_nbit_bitwise(bits, group, dtype):
    N, K = 77, 1024
    w = inputs.randn((N, K), seed=bits * 10 + group)
    w[3, :group] = 0.25  # constant group: s = 0
    if dtype == "bf16":
        w = w.to(torch.bfloat16)
    rq, rs, rb = oracle.pack_affine(w.float().numpy(), group, bits=bits)
    q, s, b = w4a8.pack_affine_nbit(w.cuda(), group, bits)
    torch.cuda.synchronize()
    assert np.array_equal(as_np(q), rq.view(np.uint8).reshape(N, -1))
    assert np.array_equal(as_np(s).view(np.uint16), rs) and np.array_equal(as_np(b).view(np.uint16), rb)


# (M, N, K): single token, a few tokens, ragged N, K with a tail of 32-blocks that does not
# fill a lane's last unrolled step, more rows than one GEMV chunk (8); M > 64 takes CTA
# pairs (a padded pair for 130 rows, ragged N tiles, a split of K for 200 x 512 x 4096)
# where K/group is a multiple of 8, and the GEMV otherwise
SHAPES = [(1, 64, 128), (3, 300, 640), (8, 256, 1024), (13, 129, 384), (40, 200, 1280), (130, 96, 4096),
          (300, 333, 1024), (200, 512, 4096), (256, 160, 2048), (100, 64, 640)]


def _pair_ok(M, K, group, bits):
    return M > 64 and (K // group) % 8 == 0 and (K * bits // 8) % 16 == 0


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("bits", [6, 8])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_affine_nbit_vs_oracle(M, N, K, bits, group):
    if K % group:
        pytest.skip("K not a multiple of the group")
    wl = inputs.Workload("nbit", M=M, K=K, N=N, x_dtype="bf16", w_std=1.0, seed=M * 7 + N + bits)
    x, w = inputs.make(wl)
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group, bits=bits)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8, bits=bits)
    q, s, b = w4a8.pack_affine_nbit(w.cuda(), group, bits)
    paths = ["auto", "gemv"] + (["gemm"] if _pair_ok(M, K, group, bits) else [])
    for path in paths:
        y = as_np(w4a8.gemm_affine_nbit(x.cuda(), q, s, b, group, bits, path=PATHS[path]))
        assert w4a8.w4a8_last_device_error() == 0
        check_tol(y, yref, T, f"affine {bits}-bit gs{group} M={M} N={N} K={K} {path}")


@pytest.mark.parametrize("bits", [6, 8])
@pytest.mark.parametrize("M", [5, 300])
def test_gemm_affine_nbit_epilogue(bits, M):
    N, K, group = 300, 1024, 64
    wl = inputs.Workload("nbit_epi", M=M, K=K, N=N, seed=5 + bits)
    x, w = inputs.make(wl)
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group, bits=bits)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8, bits=bits)
    bias = inputs.randn((N,), seed=3, std=0.5)
    ref = oracle.epilogue(yref.astype(np.float32), bias.numpy(), out_bf16=True)
    q, s, b = w4a8.pack_affine_nbit(w.cuda(), group, bits)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = w4a8.workspace(M, N, K, group)
    w4a8.w4a8_gemm_affine_nbit(x.cuda(), q, s, b, y, ws, group, bits, bias=bias.cuda())
    torch.cuda.synchronize()
    yv = oracle.bf16_to_f32(as_np(y.view(torch.int16)).view(np.uint16)).astype(np.float64)
    rv = oracle.bf16_to_f32(ref).astype(np.float64)
    assert np.all(np.abs(yv - rv) <= TOL * T + np.abs(rv) * 2.0 ** -7)


@pytest.mark.parametrize("M,K", [(40, 1024), (200, 256)])
def test_gemm_affine_nbit_tensor_path_is_refused(M, K):
    """No tensor kernel for 6/8-bit codes at M <= 64, nor when K/group is not a multiple of
    8 (the scale rows' pitch): PATH_GEMM is refused there (AUTO takes the GEMV)."""
    x = torch.randn(M, K, device="cuda")
    q, s, b = w4a8.pack_affine_nbit(torch.randn(64, K, device="cuda"), 64, 8)
    with pytest.raises(w4a8.W4A8Error) as e:
        w4a8.gemm_affine_nbit(x, q, s, b, 64, 8, path=w4a8.PATH_GEMM)
    assert e.value.status == 2


@pytest.mark.parametrize("bits", [6, 8])
def test_wide_scale_outside_tensor_range_is_reported(bits):
    """A group scale above 32 cannot be split into the CTA-pair kernel's exact fp16 parts
    for 6/8-bit codes: W4A8_ERR_RANGE, while the GEMV path stays within tolerance."""
    M, N, K, group = 200, 128, 1024, 64
    x = inputs.randn((M, K), seed=51)
    w = inputs.randn((N, K), seed=52)
    w[9, :64] *= 4000.0  # scale near 4000 * 6 / 2^bits
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group, bits=bits)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8, bits=bits)
    q, s, b = w4a8.pack_affine_nbit(w.cuda(), group, bits)
    assert w4a8.w4a8_last_device_error() == 0
    check_tol(as_np(w4a8.gemm_affine_nbit(x.cuda(), q, s, b, group, bits, path=w4a8.PATH_GEMV)), yref, T, "gemv")
    assert w4a8.w4a8_last_device_error() == 0
    w4a8.gemm_affine_nbit(x.cuda(), q, s, b, group, bits, path=w4a8.PATH_GEMM)
    assert w4a8.w4a8_last_device_error() == 7  # W4A8_ERR_RANGE
    assert w4a8.w4a8_last_device_error() == 0


@pytest.mark.parametrize("bits", [6, 8])
@pytest.mark.parametrize("std,offset", [(1e-3, 0.0), (0.02, 500.0), (1.0, -3.0)])
def test_wide_bias_term_magnitudes(bits, std, offset):
    """Bias factors b + c*s near zero, in fp16's subnormal range and at large offsets on
    the CTA-pair kernel for 6/8-bit codes."""
    M, N, K, group = 300, 256, 1024, 64
    x = inputs.randn((M, K), seed=61)
    w = inputs.randn((N, K), seed=62, std=std) + offset
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group, bits=bits)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8, bits=bits)
    q, s, b = w4a8.pack_affine_nbit(w.cuda(), group, bits)
    y = as_np(w4a8.gemm_affine_nbit(x.cuda(), q, s, b, group, bits, path=w4a8.PATH_GEMM))
    assert w4a8.w4a8_last_device_error() == 0
    check_tol(y, yref, T, f"{bits}-bit std={std} offset={offset}")


def test_nbit_4bit_equals_affine_entry():
    """bits = 4 through w4a8_gemm_affine_nbit is the w4a8_gemm_affine computation."""
    M, N, K, group = 300, 256, 1024, 64
    x = inputs.randn((M, K), seed=1).cuda()
    q, s, b = w4a8.pack_affine_nbit(inputs.randn((N, K), seed=2).cuda(), group, 4)
    y1 = w4a8.gemm_affine_nbit(x, q, s, b, group, 4)
    y2 = w4a8.gemm_affine(x, q.view(torch.int32), s, b, group)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


# 4-bit codes in groups of 32 on every path: fused GEMV, prepared GEMV (long K), tokens as
# N (16/32/64-token tiles), CTA pairs (K/32 a multiple of 8), the single-CTA token-lane
# kernel (K/32 = 25, not a multiple of 8), CTA pairs with K split.
GS32 = [(1, 300, 256, "auto"), (5, 64, 32768, "gemv"), (20, 200, 640, "gemm"), (64, 128, 1024, "gemm"),
        (300, 333, 1024, "auto"), (130, 160, 800, "auto"), (200, 512, 4096, "auto")]


@pytest.mark.parametrize("M,N,K,path", GS32)
def test_affine_gs32_vs_oracle(M, N, K, path):
    group = 32
    wl = inputs.Workload("gs32", M=M, K=K, N=N, x_dtype="bf16", w_std=1.0, seed=M + N)
    x, w = inputs.make(wl)
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8)
    q, s, b = w4a8.pack_affine(w.cuda(), group)
    assert np.array_equal(as_np(q).view(np.uint32), rq)
    y = as_np(w4a8.gemm_affine(x.cuda(), q, s, b, group, path=PATHS[path]))
    assert w4a8.w4a8_last_device_error() == 0
    check_tol(y, yref, T, f"affine gs32 M={M} N={N} K={K} {path}")

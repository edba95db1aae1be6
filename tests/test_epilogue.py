"""Output epilogue (bias of a linear layer, f32 or bf16 output).

CPU: the oracle's epilogue against values fixed by IEEE 754 single-precision addition and
round-to-nearest-even narrowing to bf16 (worked out by hand below), and the C ABI's
rejection of bad epilogues before any device work. GPU: w4a8_gemm_epi /
w4a8_gemm_affine_epi against the oracle on every kernel path (GEMV fused and from a
prepared workspace, tokens-as-N GEMM, CTA-pair GEMM with and without a split of K, the
single-CTA token-lane GEMM), and without an epilogue bit-identical to w4a8_gemm_ex."""
import ctypes

import numpy as np
import pytest
import torch

import block_quantized_w4a8_b200 as w4a8
import oracle
from block_quantized_w4a8_b200 import inputs

TOL = 1e-5


# ------------------------------------------------------------------ oracle pins (CPU)
def test_bias_is_added_in_single_precision():
    one = np.array([[1.0]], np.float32)
    # 1 + 2^-24 is half an f32 ulp above 1: the tie goes to the even neighbour, 1.
    assert oracle.epilogue(one, np.array([2.0 ** -24], np.float32))[0, 0] == np.float32(1.0)
    # 1 + 3 * 2^-24 is halfway between 1 + 2^-23 (odd) and 1 + 2^-22 (even).
    assert oracle.epilogue(one, np.array([3 * 2.0 ** -24], np.float32))[0, 0] == np.float32(1 + 2.0 ** -22)
    # every row gets the same per-column bias
    y = oracle.epilogue(np.zeros((3, 2), np.float32), np.array([0.5, -2.0], np.float32))
    assert np.array_equal(y, np.array([[0.5, -2.0]] * 3, np.float32))


def test_bf16_output_rounds_to_nearest_even():
    v = np.array([[1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -20, 0.0]], np.float32)
    # bf16 keeps 7 fraction bits: 1 + 2^-8 is half an ulp above 1.0 (0x3F80, even), 1 + 3*2^-8
    # halfway between 0x3F81 and 0x3F82 (even), the last one just above half an ulp.
    assert list(oracle.epilogue(v, out_bf16=True)[0]) == [0x3F80, 0x3F82, 0xBF80, 0x3F81, 0x0000]


def test_bf16_output_overflow_nan_and_signed_zero():
    v = np.array([[np.finfo(np.float32).max, -np.finfo(np.float32).max, np.nan, -0.0]], np.float32)
    out = oracle.epilogue(v, out_bf16=True)[0]
    assert out[0] == 0x7F80 and out[1] == 0xFF80              # beyond the largest bf16: infinity
    assert (out[2] & 0x7F80) == 0x7F80 and (out[2] & 0x7F) != 0  # NaN stays NaN
    assert out[3] == 0x8000                                    # -0 without a bias stays -0
    z = oracle.epilogue(np.array([[-0.0]], np.float32), np.array([0.0], np.float32))
    assert z.view(np.uint32)[0, 0] == 0                        # -0 + 0 = +0 (IEEE)


def test_bf16_bias_is_widened_exactly():
    bias = np.array([0x3F81, 0xC2F7], np.uint16)  # 1 + 2^-7 and -(64 + 59.5)
    y = oracle.epilogue(np.zeros((1, 2), np.float32), bias, bias_bf16=True)
    assert y[0, 0] == np.float32(1 + 2.0 ** -7) and y[0, 1] == np.float32(-123.5)


# ------------------------------------------------------------------ C ABI (CPU)
FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case fails its checks first


def test_epilogue_argument_errors():
    from block_quantized_w4a8_b200 import build
    build.build()
    lib = w4a8.load_library()
    P = ctypes.c_void_p

    def call(bias=FAKE, bias_dtype=0, out_dtype=0, fn="w4a8_gemm_epi"):
        e = w4a8.Epilogue()
        e.bias, e.bias_dtype, e.out_dtype = bias, bias_dtype, out_dtype
        if fn == "w4a8_gemm_epi":
            return lib.w4a8_gemm_epi(8, 8, 32, P(FAKE), 0, P(FAKE), P(FAKE), ctypes.byref(e), P(FAKE), P(FAKE), 16, 0,
                                     P(0))
        return lib.w4a8_gemm_affine_epi(8, 8, 128, 64, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), ctypes.byref(e),
                                        P(FAKE), P(FAKE), 16, 0, P(0))

    assert call(out_dtype=5) == 2              # UNSUPPORTED output type
    assert call(bias_dtype=5) == 2             # UNSUPPORTED bias type
    assert call(bias=FAKE + 2) == 6            # f32 bias not 4-byte aligned
    assert call(bias=FAKE + 1, bias_dtype=1) == 6
    assert call(bias=FAKE + 2, bias_dtype=1) == 3   # bf16 bias 2-byte aligned: passes, then the small workspace
    assert call(fn="affine", out_dtype=7) == 2


# ------------------------------------------------------------------ GPU parity
def dev(t):
    return t.cuda()


def _check(y, ref, T, out_bf16, what):
    """|y - ref| <= TOL*T plus the output rounding: half an f32 ulp of the bias addition, or
    one bf16 ulp (a product within TOL*T of the oracle's may round to the other neighbour)."""
    if out_bf16:
        yv = oracle.bf16_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
        rv = oracle.bf16_to_f32(ref).astype(np.float64)
        slack = np.abs(rv) * 2.0 ** -7
    else:
        yv = y.cpu().numpy().astype(np.float64)
        rv = ref.astype(np.float64)
        slack = np.abs(rv) * 2.0 ** -23
    err = np.abs(yv - rv)
    bad = err > TOL * T + slack
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside; worst {err.max()}"


PATHS = {"gemv": w4a8.PATH_GEMV, "gemm": w4a8.PATH_GEMM, "auto": w4a8.PATH_AUTO}
# (M, N, K, path): GEMV fused (small x) and from a prepared workspace (large x), tokens as N,
# CTA pairs (padded pair, ragged tile), CTA pairs with K split, single-CTA token lanes.
# (5, 64, 32768) streams the activation (too large for shared memory); (200, 510, 4096)
# splits K with rows whose length is not a multiple of 4 (element-wise reduction stores).
CASES = [(1, 300, 256, "gemv"), (5, 160, 8192, "gemv"), (5, 64, 32768, "gemv"), (24, 200, 512, "gemm"),
         (300, 333, 1024, "auto"), (200, 512, 4096, "auto"), (200, 510, 4096, "auto"), (130, 257, 800, "auto")]
EPIS = [("f32", "bf16"), ("bf16", "f32"), (None, "bf16"), ("f32", "f32")]


@pytest.mark.gpu
@pytest.mark.parametrize("bias_t,out_t", EPIS)
@pytest.mark.parametrize("M,N,K,path", CASES)
def test_q4_0_epilogue_vs_oracle(M, N, K, path, bias_t, out_t):
    wl = inputs.Workload("epi", M=M, K=K, N=N, seed=M + N + K)
    x, w = inputs.make(wl)
    rqx, rdx, _ = oracle.quant_act_q8_0(x.float().numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd, nthreads=8)
    bias = inputs.randn((N,), seed=7, std=3.0)
    bias_np, bias_dev = None, None
    if bias_t == "f32":
        bias_np, bias_dev = bias.numpy(), dev(bias)
    elif bias_t == "bf16":
        bias_np = oracle.f32_to_bf16(bias.numpy())
        bias_dev = dev(bias.to(torch.bfloat16))
    out_bf16 = out_t == "bf16"
    ref = oracle.epilogue(yref.astype(np.float32), bias_np, bias_bf16=(bias_t == "bf16"), out_bf16=out_bf16)
    qs, d = w4a8.pack_q4_0(dev(w))
    ws = w4a8.workspace(M, N, K)
    y = torch.empty(M, N, dtype=torch.bfloat16 if out_bf16 else torch.float32, device="cuda")
    w4a8.w4a8_gemm_epi(dev(x), qs, d, y, ws, bias=bias_dev, path=PATHS[path])
    torch.cuda.synchronize()
    assert w4a8.w4a8_last_device_error() == 0
    _check(y, ref, T, out_bf16, f"M={M} N={N} K={K} {path} bias={bias_t} out={out_t}")


@pytest.mark.gpu
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("M,N,K,path", [(3, 200, 1024, "gemv"), (32, 256, 1024, "gemm"), (300, 333, 1024, "auto")])
def test_affine_epilogue_vs_oracle(M, N, K, path, group):
    wl = inputs.Workload("epi_aff", M=M, K=K, N=N, seed=M + K)
    x, w = inputs.make(wl)
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8)
    bias = inputs.randn((N,), seed=11, std=1.0)
    ref = oracle.epilogue(yref.astype(np.float32), bias.numpy(), out_bf16=True)
    q, s, b = w4a8.pack_affine(dev(w), group)
    ws = w4a8.workspace(M, N, K, group)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    w4a8.w4a8_gemm_affine_epi(dev(x), q, s, b, y, ws, group, bias=dev(bias), path=PATHS[path])
    torch.cuda.synchronize()
    assert w4a8.w4a8_last_device_error() == 0
    _check(y, ref, T, True, f"affine gs{group} M={M} N={N} K={K} {path}")


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,path", CASES)
def test_no_epilogue_is_bitwise_the_plain_call(M, N, K, path):
    wl = inputs.Workload("epi0", M=M, K=K, N=N, seed=3)
    x, w = inputs.make(wl)
    qs, d = w4a8.pack_q4_0(dev(w))
    ws = w4a8.workspace(M, N, K)
    ya = torch.empty(M, N, device="cuda")
    yb = torch.empty(M, N, device="cuda")
    w4a8.w4a8_gemm_ex(dev(x), qs, d, ya, ws, PATHS[path])
    w4a8.w4a8_gemm_epi(dev(x), qs, d, yb, ws, bias=None, path=PATHS[path])
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)

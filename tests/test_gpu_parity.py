"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Codes, scales and block sums must be bit-exact; matmul outputs must satisfy
|y - y_ref| <= 1e-5 * T elementwise, T = sum over blocks of |d_w * d_x * D| (the oracle's
exact f64 terms), and y must be exactly 0 where T is 0. Small shapes are compared in
full (several tiles in every dimension plus ragged tails); the full-size workloads are
compared on sampled outputs that the oracle computes one by one, in the launch
configuration the benchmark times.
"""
import os

import numpy as np
import pytest
import torch

import block_quantized_w4a8_b200 as w4a8
import oracle
from block_quantized_w4a8_b200 import inputs
from tests import refdecode as ref

pytestmark = pytest.mark.gpu
TOL = 1e-5
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
PATHS = {"auto": w4a8.PATH_AUTO, "gemv": w4a8.PATH_GEMV, "gemm": w4a8.PATH_GEMM}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    w4a8.load_library()
    yield
    assert w4a8.w4a8_last_device_error() == 0, "a kernel reported a bounded-wait timeout"


def dev(t):
    return t.contiguous().cuda()


def as_np(t):
    return t.cpu().numpy()


def check_tol(y, yref, T, what=""):
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - yref)
    bad = err > TOL * T
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"y={y[tuple(i)]!r} ref={yref[tuple(i)]!r} T={T[tuple(i)]!r}")
    nz = T > 0
    return float((err[nz] / T[nz]).max()) if nz.any() else 0.0


# ------------------------------------------------------------------ act quant
@pytest.mark.parametrize("M,K,dtype", [(64, 384, "f32"), (1, 4096, "f32"), (37, 160, "bf16"), (300, 800, "f32"),
                                       (5, 14336, "bf16")])
def test_quant_act_bit_exact(M, K, dtype):
    x = inputs.randn((M, K), seed=M * 7 + K)
    x[0, :32] = 0.0
    if M > 2:
        x[2, 32:64] = torch.arange(32, dtype=torch.float32) - 15.5  # exact half-way products
    xt = x.to(torch.bfloat16) if dtype == "bf16" else x
    qx, dx, sx = w4a8.quant_act_q8_0(dev(xt))
    rq, rd, rs = oracle.quant_act_q8_0(xt.float().numpy())
    assert np.array_equal(as_np(qx), rq)
    assert np.array_equal(as_np(dx).view(np.uint32), rd.view(np.uint32))
    assert np.array_equal(as_np(sx), rs)


def test_quant_act_golden_rounding():
    g = ref.read_golden(os.path.join(GOLDEN, "q8_0_rounding.txt"))
    x = torch.tensor([[float(v) for v in g["x"]]], dtype=torch.float32)
    qx, dx, sx = w4a8.quant_act_q8_0(dev(x))
    assert [int(v) for v in as_np(qx)[0]] == [int(v) for v in g["q"]]
    assert int(as_np(sx)[0, 0]) == int(g["sum"][0])


# ------------------------------------------------------------------ weight packs
@pytest.mark.parametrize("N,K,dtype,std", [(1536, 384, "f32", 0.02), (4096, 4096, "f32", 0.02), (333, 800, "bf16", 1.0),
                                           (64, 14336, "f32", 1.0)])
def test_pack_q4_0_bit_exact(N, K, dtype, std):
    w = inputs.randn((N, K), seed=N + K, std=std)
    w[1, :32] = 0.0
    w[2, 32] = 0.5
    w[2, 33] = -0.5
    wt = w.to(torch.bfloat16) if dtype == "bf16" else w
    qs, d = w4a8.pack_q4_0(dev(wt))
    rqs, rd = oracle.pack_q4_0(wt.float().numpy())
    assert np.array_equal(as_np(qs), rqs)
    assert np.array_equal(as_np(d).view(np.uint16), rd)


def test_pack_q4_0_golden_block():
    g = ref.read_golden(os.path.join(GOLDEN, "q4_0_block_layout.txt"))
    w = torch.tensor([[float(v) for v in g["x"]]], dtype=torch.float32)
    qs, d = w4a8.pack_q4_0(dev(w))
    assert [int(b) for b in as_np(qs)[0]] == [int(v, 16) for v in g["bytes"]]
    assert int(as_np(d).view(np.uint16)[0, 0]) == int(g["scale_fp16_bits"][0], 16)


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("N,K,dtype", [(512, 1024, "f32"), (4096, 4096, "bf16"), (33, 384, "f32")])
def test_pack_affine_bit_exact(group, N, K, dtype):
    w = inputs.randn((N, K), seed=N * 3 + group)
    w[1, :group] = 0.25
    wt = w.to(torch.bfloat16) if dtype == "bf16" else w
    q, s, b = w4a8.pack_affine(dev(wt), group)
    rq, rs, rb = oracle.pack_affine(wt.float().numpy(), group)
    assert np.array_equal(as_np(q).view(np.uint32), rq)
    assert np.array_equal(as_np(s).view(np.uint16), rs)
    assert np.array_equal(as_np(b).view(np.uint16), rb)


# ------------------------------------------------------------------ Q4_0 matmul, full compare
# M > 64 with K a multiple of 256 runs on CTA pairs: (300, 333, 1024) has an odd token-tile
# count (padded to a pair) and a ragged weight tile, (200, 512, 4096) splits K over the
# pairs; the other M > 64 shapes take the single-CTA kernel (scale rows not 16-B aligned).
SHAPES = [(1, 1, 32), (1, 4096, 4096), (2, 333, 800), (5, 1536, 384), (8, 200, 256), (17, 96, 640),
          (32, 520, 1056), (64, 1536, 384), (300, 333, 800), (129, 128, 128), (130, 257, 4128), (3, 64, 32768),
          (300, 333, 1024), (200, 512, 4096),
          # bulk-copy GEMV: fewer rows than SMs, rows not a multiple of the SM count, long K,
          # several stage refills per CTA, eight tokens at the sweep's K
          (1, 100, 2048), (6, 1000, 2048), (1, 1000, 14336), (4, 2000, 4096), (8, 300, 8192)]


def _q4_0_case(M, N, K, x_dtype="f32", w_std=0.02, seed=0):
    wl = inputs.Workload("case", M=M, K=K, N=N, x_dtype=x_dtype, w_std=w_std, seed=seed)
    x, w = inputs.make(wl)
    rqx, rdx, _ = oracle.quant_act_q8_0(x.float().numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    return x, w, rqx, rdx, rqs, rd


@pytest.mark.parametrize("path", ["gemv", "gemm", "auto"])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_q4_0_vs_oracle(M, N, K, path):
    x, w, rqx, rdx, rqs, rd = _q4_0_case(M, N, K, seed=M + N)
    yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd, nthreads=8)
    qs, d = w4a8.pack_q4_0(dev(w))
    y = w4a8.gemm(dev(x), qs, d, path=PATHS[path])
    torch.cuda.synchronize()
    check_tol(as_np(y), yref, T, f"M={M} N={N} K={K} {path}")


@pytest.mark.parametrize("M,path", [(256, "gemm"), (40, "gemm"), (3, "gemv")])
def test_long_k_same_sign_within_tolerance(M, path):
    """K = 14336 with x >= 0 and W >= 0: every block term has the same sign, so |y| is the
    sum of |terms| and an f32 chain over all 448 blocks would show its full rounding error
    (up to 448 * 2^-24 = 2.7e-5 of it). The 1e-5 bound holds here as at K = 4096: the
    tensor-core path splits K so that no chain is longer than 128 blocks (M = 256: CTA
    pairs; M = 40: tokens as the MMA's N), and the GEMV's chains are short."""
    N, K = 128, 14336
    x = inputs.randn((M, K), seed=31).abs()
    w = inputs.randn((N, K), seed=32, std=0.02).abs()
    rqx, rdx, _ = oracle.quant_act_q8_0(x.numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd, nthreads=8)
    assert np.all(np.abs(yref) >= 0.999999 * T)  # same-sign terms: |y| = T
    qs, d = w4a8.pack_q4_0(dev(w))
    y = w4a8.gemm(dev(x), qs, d, path=PATHS[path])
    torch.cuda.synchronize()
    check_tol(as_np(y), yref, T, f"M={M} K={K} {path}")


def test_gemm_bf16_input_and_paths_agree():
    x, w, rqx, rdx, rqs, rd = _q4_0_case(48, 640, 1024, x_dtype="bf16", w_std=1.0, seed=5)
    yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd, nthreads=8)
    qs, d = w4a8.pack_q4_0(dev(w))
    ya = as_np(w4a8.gemm(dev(x), qs, d, path=w4a8.PATH_GEMV))
    yb = as_np(w4a8.gemm(dev(x), qs, d, path=w4a8.PATH_GEMM))
    check_tol(ya, yref, T, "gemv bf16")
    check_tol(yb, yref, T, "gemm bf16")
    assert np.all(np.abs(ya.astype(np.float64) - yb) <= 2 * TOL * T)


def test_gemm_degenerate_inputs_give_exact_zero():
    M, N, K = 130, 160, 256
    x = torch.zeros(M, K)
    w = inputs.randn((N, K), seed=1, std=0.02)
    qs, d = w4a8.pack_q4_0(dev(w))
    for path in (w4a8.PATH_GEMV, w4a8.PATH_GEMM):
        assert torch.count_nonzero(w4a8.gemm(dev(x), qs, d, path=path)).item() == 0
    qs0, d0 = w4a8.pack_q4_0(dev(torch.zeros(N, K)))
    x1 = inputs.randn((M, K), seed=2)
    for path in (w4a8.PATH_GEMV, w4a8.PATH_GEMM):
        assert torch.count_nonzero(w4a8.gemm(dev(x1), qs0, d0, path=path)).item() == 0


def test_gemm_is_deterministic_and_ignores_workspace_contents():
    M, N, K = 200, 384, 1024
    x, w, *_ = _q4_0_case(M, N, K, seed=3)
    qs, d = w4a8.pack_q4_0(dev(w))
    for path in (w4a8.PATH_GEMV, w4a8.PATH_GEMM):
        ws = w4a8.workspace(M, N, K)
        ws.random_(0, 256)
        y1 = w4a8.gemm(dev(x), qs, d, path=path, ws=ws)
        ws.random_(0, 256)
        y2 = w4a8.gemm(dev(x), qs, d, path=path, ws=ws)
        assert torch.equal(y1, y2)


@pytest.mark.parametrize("M", [40, 130])
def test_scale_outside_tensor_core_range_is_reported(M):
    """A Q4_0 block scale above 2720 cannot be held exactly by the fp16 weight operand of
    the CTA-pair and single-CTA tensor-core kernels (M = 130): that path reports
    W4A8_ERR_RANGE through the device status word. The GEMV path and the int8 tensor-core
    kernel (M = 40: 64-token tiles, K a multiple of 256) have no such limit and stay within
    tolerance."""
    N, K = 128, 256
    x, w, *_ = _q4_0_case(M, N, K, seed=21)
    w[5, :32] *= 100000.0 / float(w[5, :32].abs().max())  # block scale 12500
    rqs, rd = oracle.pack_q4_0(w.numpy())
    rqx, rdx, _ = oracle.quant_act_q8_0(x.numpy())
    yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd, nthreads=8)
    qs, d = w4a8.pack_q4_0(dev(w))
    assert w4a8.w4a8_last_device_error() == 0
    check_tol(as_np(w4a8.gemm(dev(x), qs, d, path=w4a8.PATH_GEMV)), yref, T, "gemv, large scale")
    assert w4a8.w4a8_last_device_error() == 0
    y = w4a8.gemm(dev(x), qs, d, path=w4a8.PATH_GEMM)
    if M <= 64:
        check_tol(as_np(y), yref, T, "int8 tensor path, large scale")
        assert w4a8.w4a8_last_device_error() == 0
    else:
        assert w4a8.w4a8_last_device_error() == 7  # W4A8_ERR_RANGE, read and cleared
        assert w4a8.w4a8_last_device_error() == 0


def test_empty_input_is_rejected():
    qs = torch.zeros(8, 16, dtype=torch.uint8, device="cuda")
    d = torch.zeros(8, 1, dtype=torch.int16, device="cuda")
    x = torch.zeros(0, 32, device="cuda")
    y = torch.zeros(0, 8, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(w4a8.W4A8Error) as e:
        w4a8.w4a8_gemm(x, qs, d, y, ws)
    assert e.value.status == 1


# ------------------------------------------------------------------ full-size workloads, sampled
FULL = [inputs.MINILM, inputs.DECODE, inputs.PREFILL,
        inputs.Workload("mlp_m16_k4096_n14336", M=16, K=4096, N=14336),
        inputs.Workload("mlp_m256_k14336_n4096", M=256, K=14336, N=4096),
        inputs.Workload("mlp_m4096_k8192_n2048", M=4096, K=8192, N=2048)]


@pytest.mark.parametrize("wl", FULL, ids=lambda w: w.name)
def test_full_size_sampled(wl):
    x, w = inputs.make(wl)
    qs, d = w4a8.pack_q4_0(dev(w))
    y = as_np(w4a8.gemm(dev(x), qs, d))           # AUTO: the path the benchmark times
    rqx, rdx, _ = oracle.quant_act_q8_0(x.float().numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    assert np.array_equal(as_np(qs), rqs) and np.array_equal(as_np(d).view(np.uint16), rd)
    ms, ns = inputs.sample_indices(wl.M, wl.N, 3000)
    yref, T = oracle.gemm_q4_0_sampled(rqx, rdx, rqs, rd, ms, ns)
    check_tol(y[ms, ns], yref, T, wl.name)


# Every K x N of the MLP sweep at M = 1, 8, 64 and 1024 (GEMV, int8 tensor kernel at 8
# and 64 tokens, CTA pairs at 1024), through AUTO, on sampled outputs.
SWEEP_FULL = [inputs.Workload(f"sweep_m{M}_k{K}_n{N}", M=M, K=K, N=N)
              for K, N in inputs.SWEEP_SHAPES for M in (1, 8, 64, 1024)]


@pytest.mark.parametrize("wl", SWEEP_FULL, ids=lambda w: w.name)
def test_sweep_full_size_sampled(wl):
    x, w = inputs.make(wl)
    qs, d = w4a8.pack_q4_0(dev(w))
    y = as_np(w4a8.gemm(dev(x), qs, d))
    rqx, rdx, _ = oracle.quant_act_q8_0(x.float().numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    ms, ns = inputs.sample_indices(wl.M, wl.N, 1000, seed=wl.M + wl.K)
    yref, T = oracle.gemm_q4_0_sampled(rqx, rdx, rqs, rd, ms, ns)
    check_tol(y[ms, ns], yref, T, wl.name)


CROSSOVER = [inputs.Workload(f"crossover_m{M}_k{K}_n{N}", M=M, K=K, N=N, seed=M + N)
             for K, N in inputs.SWEEP_SHAPES + [(4096, 4096)] for M in (2, 4, 5)]


@pytest.mark.parametrize("wl", CROSSOVER, ids=lambda w: w.name)
def test_dispatch_crossover_sampled(wl):
    """At the GEMV / int8-kernel crossover (M = 2..5) the AUTO call agrees with the
    oracle, and with the path the dispatch rule names forced explicitly: the two paths
    give the same result up to the tolerance, whichever the rule picks."""
    x, w = inputs.make(wl)
    qs, d = w4a8.pack_q4_0(dev(w))
    rqx, rdx, _ = oracle.quant_act_q8_0(x.float().numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    ms, ns = inputs.sample_indices(wl.M, wl.N, 1000, seed=wl.M * 7 + wl.K)
    yref, T = oracle.gemm_q4_0_sampled(rqx, rdx, rqs, rd, ms, ns)
    chosen = w4a8.w4a8_gemm_path(wl.M, wl.N, wl.K)
    for path in ("auto", "gemv", "gemm"):
        y = as_np(w4a8.gemm(dev(x), qs, d, path=PATHS[path]))
        check_tol(y[ms, ns], yref, T, f"{wl.name} {path} (auto: {chosen})")
        assert w4a8.w4a8_last_device_error() == 0


# ------------------------------------------------------------------ affine
AFFINE_SHAPES = [(1, 64, 128), (3, 300, 640), (8, 256, 1024), (20, 128, 640), (32, 256, 1024), (64, 1536, 384),
                 (200, 333, 1280), (130, 128, 4096), (300, 333, 1024), (200, 512, 4096)]


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("path", ["gemv", "gemm"])
@pytest.mark.parametrize("M,N,K", AFFINE_SHAPES)
def test_gemm_affine_vs_oracle(M, N, K, path, group):
    if K % group:
        pytest.skip("K not a multiple of the group")
    wl = inputs.Workload("aff", M=M, K=K, N=N, x_dtype="bf16", w_std=1.0, seed=M * 5 + N)
    x, w = inputs.make(wl)
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8)
    q, s, b = w4a8.pack_affine(dev(w), group)
    y = as_np(w4a8.gemm_affine(dev(x), q, s, b, group, path=PATHS[path]))
    check_tol(y, yref, T, f"affine gs{group} M={M} N={N} K={K} {path}")


@pytest.mark.parametrize("wl", [inputs.AFFINE_GS64, inputs.AFFINE_GS128], ids=lambda w: w.name)
def test_affine_full_size_sampled(wl):
    x, w = inputs.make(wl)
    q, s, b = w4a8.pack_affine(dev(w), wl.group)
    y = as_np(w4a8.gemm_affine(dev(x), q, s, b, wl.group))
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), wl.group)
    assert np.array_equal(as_np(q).view(np.uint32), rq)
    ms, ns = inputs.sample_indices(wl.M, wl.N, 3000)
    yref, T = oracle.gemm_affine_sampled(rqx, rdx, rsx, rq, rs, rb, wl.group, ms, ns)
    check_tol(y[ms, ns], yref, T, wl.name)


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("std,offset", [(1.0, 0.0), (1e-4, 0.0), (0.02, 3000.0), (0.01, -0.05), (1e-3, 2e-5)])
def test_affine_bias_term_magnitudes(std, offset, group):
    """The CTA-pair kernel (128-token tiles, K/group a multiple of 8) carries the factor of
    the group bias term, b + 8s, as two fp16 MMA operands (22 bits of it): weights whose
    groups put that factor far below or above the codes' term (tiny weights, a large or a
    small common offset, a factor near zero or in fp16's subnormal range) stay within the
    tolerance of the oracle, as on the GEMV path."""
    M, N, K = 300, 256, 1024
    x = inputs.randn((M, K), seed=31)
    w = inputs.randn((N, K), seed=32, std=std) + offset
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8)
    q, s, b = w4a8.pack_affine(dev(w), group)
    for path in ("gemm", "gemv"):
        y = as_np(w4a8.gemm_affine(dev(x), q, s, b, group, path=PATHS[path]))
        assert w4a8.w4a8_last_device_error() == 0
        check_tol(y, yref, T, f"affine gs{group} std={std} offset={offset} {path}")


def test_affine_bias_factor_outside_fp16_is_reported():
    """A group whose b + 8s exceeds fp16's range cannot be an MMA operand of the CTA-pair
    kernel: it reports W4A8_ERR_RANGE, while the GEMV path stays within tolerance."""
    M, N, K, group = 300, 128, 1024, 64
    x = inputs.randn((M, K), seed=33)
    w = inputs.randn((N, K), seed=34)
    w[7, 64:128] += 70000.0  # one group of one row: b + 8s near 7e4
    rqx, rdx, rsx = oracle.quant_act_q8_0(x.numpy())
    rq, rs, rb = oracle.pack_affine(w.numpy(), group)
    yref, T = oracle.gemm_affine(rqx, rdx, rsx, rq, rs, rb, group, nthreads=8)
    q, s, b = w4a8.pack_affine(dev(w), group)
    assert w4a8.w4a8_last_device_error() == 0
    check_tol(as_np(w4a8.gemm_affine(dev(x), q, s, b, group, path=w4a8.PATH_GEMV)), yref, T, "gemv, large bias")
    assert w4a8.w4a8_last_device_error() == 0
    w4a8.gemm_affine(dev(x), q, s, b, group, path=w4a8.PATH_GEMM)
    assert w4a8.w4a8_last_device_error() == 7  # W4A8_ERR_RANGE
    assert w4a8.w4a8_last_device_error() == 0


def test_affine_bias_minus_8s_matches_q4_0_on_gpu():
    """Cross-format invariant on the GPU: affine codes with bias = -8*scale reproduce the
    Q4_0 matmul with d = scale and the same codes."""
    rng = np.random.default_rng(12)
    M, N, K, group = 160, 256, 512, 64
    codes = rng.integers(0, 16, size=(N, K))
    scale = (2.0 ** rng.integers(-8, -4, size=(N, K // group))).astype(np.float32)
    words = (codes.reshape(N, K // 8, 8).astype(np.uint64) << (4 * np.arange(8, dtype=np.uint64))).sum(axis=2).astype(np.uint32)
    s_bits = torch.from_numpy(scale).to(torch.bfloat16).view(torch.int16)
    b_bits = torch.from_numpy(-8 * scale).to(torch.bfloat16).view(torch.int16)
    blocks = codes.reshape(N, K // 32, 32)
    qs = (blocks[:, :, :16] | (blocks[:, :, 16:] << 4)).reshape(N, K // 2).astype(np.uint8)
    d_bits = np.repeat(scale, group // 32, axis=1).astype(np.float16).view(np.int16)
    x = dev(inputs.randn((M, K), seed=13))
    for path in (w4a8.PATH_GEMV, w4a8.PATH_GEMM):
        ya = w4a8.gemm_affine(x, dev(torch.from_numpy(words.view(np.int32))), dev(s_bits), dev(b_bits), group,
                              path=path)
        yq = w4a8.gemm(x, dev(torch.from_numpy(qs)), dev(torch.from_numpy(d_bits)), path=path)
        rqx, rdx, _ = oracle.quant_act_q8_0(as_np(x))
        _, T = oracle.gemm_q4_0(rqx, rdx, qs, d_bits.view(np.uint16), nthreads=8)
        assert np.all(np.abs(as_np(ya).astype(np.float64) - as_np(yq)) <= 2 * TOL * T)

"""Pins for the oracle's affine 6- and 8-bit codes and groups of 32 (no GPU): hand-worked
bit-stream layouts, exact grids, brute force over every code, an independent numpy
decoder, the split of an 8-bit code into two 4-bit codes, and the accuracy rows of the
MLX affine page for 6 and 8 bits."""
import os

import numpy as np
import pytest
import torch

import oracle
from block_quantized_w4a8_b200 import inputs
from tests import refdecode as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = [4, 6, 8]
GROUPS = [32, 64, 128]


def _hex(vals):
    return [int(v, 16) for v in vals]


def test_affine_nbit_golden_layout():
    g = ref.read_golden(os.path.join(GOLDEN, "affine_nbit_layout.txt"))
    # 6-bit grid: codes 0..63 in order
    w6 = (-1.0 + np.arange(64) / 32.0).astype(np.float32)[None, :]
    q, s, b = oracle.pack_affine(w6, 64, bits=6)
    assert q.dtype == np.uint8 and q.shape == (1, 48)
    assert list(q[0, :6]) == _hex(g["six_first_bytes"])
    assert int(s[0, 0]) == _hex(g["six_scale_bf16_bits"])[0] and int(b[0, 0]) == _hex(g["six_bias_bf16_bits"])[0]
    # 8-bit grid in a group of 32
    codes8 = np.array([0, 255] + list(range(1, 31)))
    q, s, b = oracle.pack_affine((2.0 + codes8 / 64.0).astype(np.float32)[None, :], 32, bits=8)
    assert list(q[0, :4]) == _hex(g["eight_first_bytes"]) and list(q[0]) == list(codes8)
    assert int(s[0, 0]) == _hex(g["eight_scale_bf16_bits"])[0] and int(b[0, 0]) == _hex(g["eight_bias_bf16_bits"])[0]
    # a given 6-bit code sequence (the group holds codes 0 and 63, so s and b are exact)
    c = np.array([int(v) for v in g["six_codes"]] + [5] * 24)
    q, _, _ = oracle.pack_affine((-2.0 + c / 16.0).astype(np.float32)[None, :], 32, bits=6)
    assert list(q[0, :6]) == _hex(g["six_code_bytes"])


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("bits", BITS)
def test_affine_nbit_grid_round_trip_and_invariants(bits, group):
    rng = np.random.default_rng(100 + bits + group)
    qmax = (1 << bits) - 1
    N, K = 8, 512
    codes = rng.integers(0, qmax + 1, size=(N, K))
    codes[:, ::group] = 0
    codes[:, 1::group] = qmax
    s = (2.0 ** rng.integers(-8, -2, size=(N, K // group))).astype(np.float32)
    b = (-(2.0 ** rng.integers(-3, 2, size=(N, K // group)))).astype(np.float32)
    w = (np.repeat(s, group, 1) * codes + np.repeat(b, group, 1)).astype(np.float32)
    q, sb, bb = oracle.pack_affine(w, group, bits=bits)
    assert np.array_equal(ref.affine_codes_bits(q, bits), codes)
    assert np.array_equal(ref.bf16_bits_to_f64(sb), s.astype(np.float64))
    assert np.array_equal(ref.bf16_bits_to_f64(bb), b.astype(np.float64))
    if bits == 4:  # the 4-bit bit stream is the word layout
        assert np.array_equal(ref.affine_codes(q), codes)
    # random weights: codes in range, constant group gives s = 0, codes 0, w = b
    w2 = inputs.randn((8, 512), seed=8 + bits).numpy()
    w2[2, :group] = 0.375
    q2, s2, b2 = oracle.pack_affine(w2, group, bits=bits)
    c2 = ref.affine_codes_bits(q2, bits)
    assert c2.min() >= 0 and c2.max() <= qmax and c2.max() == qmax
    assert ref.bf16_bits_to_f64(s2)[2, 0] == 0 and np.all(c2[2, :group] == 0)
    assert ref.bf16_bits_to_f64(b2)[2, 0] == 0.375
    # each code is a nearest grid point of s*q + b (brute force over all 2^bits codes)
    sv = np.repeat(ref.bf16_bits_to_f64(s2), group, 1)
    bv = np.repeat(ref.bf16_bits_to_f64(b2), group, 1)
    err = np.abs(w2[..., None] - (sv[..., None] * np.arange(qmax + 1) + bv[..., None]))
    chosen = np.take_along_axis(err, c2[..., None], 2)[..., 0]
    assert np.all(chosen <= err.min(axis=2) + 1e-6 * sv + 1e-30)


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (3, 2, 256), (5, 6, 384)])
def test_gemm_affine_nbit_brute_force(bits, group, M, N, K):
    if K % group:
        pytest.skip("K not a multiple of the group")
    x = inputs.randn((M, K), seed=30 + M + bits).numpy()
    w = inputs.randn((N, K), seed=40 + N + bits).numpy()
    qx, dx, sx = oracle.quant_act_q8_0(x)
    q, s, b = oracle.pack_affine(w, group, bits=bits)
    y, T = oracle.gemm_affine(qx, dx, sx, q, s, b, group, bits=bits)
    want = ref.q8_0_values(qx, dx) @ ref.affine_weights_bits(q, s, b, group, bits).T
    assert np.all(np.abs(y - want) <= 1e-12 * T + 1e-300)
    ms, ns = np.repeat(np.arange(M), N), np.tile(np.arange(N), M)
    ys, Ts = oracle.gemm_affine_sampled(qx, dx, sx, q, s, b, group, ms, ns, bits=bits)
    assert np.array_equal(ys, y.reshape(-1)) and np.array_equal(Ts, T.reshape(-1))


@pytest.mark.parametrize("bits", [6, 8])
def test_wide_code_is_two_4bit_codes(bits):
    """q = 16h + l: the affine matmul with codes q, scale s and bias b equals the sum of
    two 4-bit affine matmuls, codes h with scale 16s and bias b plus codes l with scale s
    and bias 0 (every scale exact in bf16)."""
    rng = np.random.default_rng(bits)
    M, N, K, group = 3, 5, 256, 64
    codes = rng.integers(0, 1 << bits, size=(N, K))
    s = (2.0 ** rng.integers(-7, -3, size=(N, K // group))).astype(np.float32)
    b = rng.choice([-1.0, -0.5, 0.25], size=(N, K // group)).astype(np.float32)
    codes[:, ::group], codes[:, 1::group] = 0, (1 << bits) - 1  # the grid's ends: s and b exact
    w = (np.repeat(s, group, 1) * codes + np.repeat(b, group, 1)).astype(np.float32)
    q, sb, bb = oracle.pack_affine(w, group, bits=bits)
    x = inputs.randn((M, K), seed=77).numpy()
    qx, dx, sx = oracle.quant_act_q8_0(x)
    y, T = oracle.gemm_affine(qx, dx, sx, q, sb, bb, group, bits=bits)

    def words(c):
        return (c.reshape(N, K // 8, 8).astype(np.uint64) << (4 * np.arange(8, dtype=np.uint64))).sum(2).astype(np.uint32)

    def bf16(v):
        return torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    yh, _ = oracle.gemm_affine(qx, dx, sx, words(codes >> 4), bf16(16 * s), bb, group)
    yl, _ = oracle.gemm_affine(qx, dx, sx, words(codes & 15), sb, bf16(np.zeros_like(s)), group)
    assert np.all(np.abs(y - (yh + yl)) <= 1e-12 * T)


@pytest.mark.parametrize("bits,group", [(6, 64), (8, 64), (8, 128)])
def test_affine_nbit_accuracy_matches_mlx_table(bits, group):
    """Relative RMS error against the f32 matmul of the unquantised inputs, on the MLX
    accuracy setup (M=1024, K=N=4096, normal x and w, bf16); 64 of the 1024 rows. The
    page's "qqmm" figure adds its own int8 quantisation of x and bf16 arithmetic to the
    weight error, its "quantized_matmul" figure has the weight error and bf16 arithmetic
    only; the oracle (f64 arithmetic, one x scale per 32-block) falls between the two."""
    rows = {(r[0], r[1]): (float(r[2]), float(r[3])) for r in
            ref.read_golden(os.path.join(GOLDEN, "affine_accuracy_nbit.txt"))["rows"]}
    wl = inputs.AFFINE_GS64 if group == 64 else inputs.AFFINE_GS128
    x, w = inputs.make(wl)
    x = x[:64]
    w = w.to(torch.bfloat16).float()
    qx, dx, sx = oracle.quant_act_q8_0(x.float().numpy())
    q, s, b = oracle.pack_affine(w.numpy(), group, bits=bits)
    y, _ = oracle.gemm_affine(qx, dx, sx, q, s, b, group, nthreads=8, bits=bits)
    exact = x.double().numpy() @ w.double().numpy().T
    rel = 100 * np.sqrt(np.mean((y - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    qq, qm = rows[(str(bits), str(group))]
    assert 0.9 * qm <= rel <= 1.05 * qq, (rel, qm, qq)

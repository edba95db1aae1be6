"""Pins for the CPU oracle (no GPU). Each test checks the oracle against something
other than itself: hand-worked golden blocks, exact grids, brute force over all codes,
textbook integer matmuls, dequantise-then-f64 matmuls through independent decoders,
torch/numpy conversions, and the accuracy table of the MLX affine page."""
import os

import numpy as np
import pytest
import torch

import oracle
from block_quantized_w4a8_b200 import inputs
from tests import refdecode as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ O1 conversions
def _structured_f32(drop_bits: int) -> np.ndarray:
    """Every sign/exponent/top-fraction pattern combined with the low-bit patterns that
    decide rounding when `drop_bits` bits are dropped (ties, just below, just above)."""
    lows = np.array([0, 1, (1 << (drop_bits - 1)) - 1, 1 << (drop_bits - 1), (1 << (drop_bits - 1)) + 1,
                     (1 << drop_bits) - 1], dtype=np.uint64)
    highs = np.arange(1 << (32 - drop_bits), dtype=np.uint64) << np.uint64(drop_bits)
    bits = (highs[:, None] | lows[None, :]).reshape(-1).astype(np.uint32)
    f = bits.view(np.float32)
    return f[np.isfinite(f)]


def test_f32_to_f16_matches_torch_structured_and_random():
    f = _structured_f32(13)
    rnd = np.random.default_rng(0).integers(0, 2**32, size=4_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    f = np.concatenate([f, rnd[np.isfinite(rnd)]])
    got = oracle.f32_to_f16(f)
    want = torch.from_numpy(f.copy()).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_f32_to_bf16_matches_torch_structured_and_random():
    f = _structured_f32(16)
    rnd = np.random.default_rng(1).integers(0, 2**32, size=4_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    f = np.concatenate([f, rnd[np.isfinite(rnd)]])
    got = oracle.f32_to_bf16(f)
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_widening_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    h = oracle.f16_to_f32(bits)
    want_h = bits.view(np.float16).astype(np.float32)
    fin = np.isfinite(want_h)
    assert np.array_equal(h[fin].view(np.uint32), want_h[fin].view(np.uint32))
    assert np.all(np.isnan(h[~fin]) == np.isnan(want_h[~fin]))
    b = oracle.bf16_to_f32(bits)
    want_b = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    fin = np.isfinite(want_b)
    assert np.array_equal(b[fin].view(np.uint32), want_b[fin].view(np.uint32))


# ------------------------------------------------------------------ O2 Q4_0 pack
def test_q4_0_golden_block():
    g = ref.read_golden(os.path.join(GOLDEN, "q4_0_block_layout.txt"))
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)[None, :]
    qs, d = oracle.pack_q4_0(x)
    assert [int(b) for b in qs[0]] == [int(v, 16) for v in g["bytes"]]
    assert int(d[0, 0]) == int(g["scale_fp16_bits"][0], 16)


def test_q4_0_grid_round_trip():
    rng = np.random.default_rng(2)
    N, K = 16, 256
    codes = rng.integers(0, 16, size=(N, K))
    codes[:, ::32] = 0  # every block reaches code 0 (the element that sets the scale)
    # fp16-representable scales of both signs and several binades
    d16 = (rng.choice([-1, 1], size=(N, K // 32)) * rng.integers(1024, 2048, size=(N, K // 32))
           * 2.0 ** rng.integers(-20, -8, size=(N, K // 32))).astype(np.float32)
    assert np.array_equal(d16.astype(np.float16).astype(np.float32), d16)
    w = (np.repeat(d16, 32, axis=1) * (codes - 8)).astype(np.float32)
    qs, d = oracle.pack_q4_0(w)
    assert np.array_equal(ref.q4_0_codes(qs), codes)
    assert np.array_equal(ref.fp16_bits_to_f64(d), d16.astype(np.float64))
    assert np.array_equal(ref.q4_0_weights(qs, d), w.astype(np.float64))


def test_q4_0_invariants_and_brute_force_nearest_code():
    x = inputs.randn((64, 512), seed=3, std=0.02).numpy()
    x[5, 32:64] = 0.0                               # an all-zero block
    x[7, 64] = 0.05; x[7, 65] = -0.05              # +a then -a: first wins, -a clamps to 15
    qs, d = oracle.pack_q4_0(x)
    codes = ref.q4_0_codes(qs)
    assert codes.min() >= 0 and codes.max() <= 15
    xb = x.reshape(64, 16, 32)
    cb = codes.reshape(64, 16, 32)
    first = np.argmax(np.abs(xb), axis=2)          # numpy returns the first maximum
    nz = np.abs(xb).max(axis=2) > 0
    assert np.all(np.take_along_axis(cb, first[..., None], 2)[..., 0][nz] == 0)
    assert np.all(cb[5, 1] == 8) and ref.fp16_bits_to_f64(d)[5, 1] == 0.0
    assert cb[7, 2, 0] == 0 and cb[7, 2, 1] == 15
    # brute force: each code is a nearest grid point under the f32 block scale
    mx = np.take_along_axis(xb, first[..., None], 2)
    d32 = (mx / np.float32(-8.0)).astype(np.float64)
    grid = d32[..., None] * (np.arange(16) - 8)
    err = np.abs(xb.astype(np.float64)[..., None] - grid)
    chosen = np.take_along_axis(err, cb[..., None], 3)[..., 0]
    best = err.min(axis=3)
    clamp = (xb.astype(np.float64) / np.where(d32 == 0, 1, d32)) > 7.5   # past the top code
    ok = (chosen <= best + 1e-6 * np.abs(d32)) | clamp
    assert np.all(ok[nz])
    # error bound with the stored fp16 scale
    wq = ref.q4_0_weights(qs, d).reshape(64, 16, 32)
    bound = np.abs(d32) / 2 * (1 + 2**-20) + 8 * np.abs(d32 - ref.fp16_bits_to_f64(d)[..., None]) + 1e-30
    assert np.all((np.abs(xb - wq) <= bound) | clamp)


# ------------------------------------------------------------------ O3 Q8_0 quant
def test_q8_0_golden_half_away_rounding():
    g = ref.read_golden(os.path.join(GOLDEN, "q8_0_rounding.txt"))
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)[None, :]
    qx, dx, sx = oracle.quant_act_q8_0(x)
    assert [int(v) for v in qx[0]] == [int(v) for v in g["q"]]
    assert sx[0, 0] == int(g["sum"][0]) and dx[0, 0] == float(g["scale"][0])


def test_q8_0_invariants_and_brute_force():
    x = inputs.randn((32, 1024), seed=4).numpy()
    x[3, :32] = 0.0
    qx, dx, sx = oracle.quant_act_q8_0(x)
    xb = x.reshape(32, 32, 32).astype(np.float64)
    qb = qx.reshape(32, 32, 32).astype(np.int64)
    amax_i = np.argmax(np.abs(xb), axis=2)
    top = np.take_along_axis(qb, amax_i[..., None], 2)[..., 0]
    sgn = np.sign(np.take_along_axis(xb, amax_i[..., None], 2)[..., 0])
    nz = np.abs(xb).max(axis=2) > 0
    assert np.all(top[nz] == 127 * sgn[nz])
    assert np.all(qb[3, 0] == 0) and dx[3, 0] == 0 and sx[3, 0] == 0
    assert np.array_equal(sx, qb.sum(axis=2))
    d = dx.astype(np.float64)[..., None]
    # brute force over all 255 codes: the chosen code is a nearest one
    grid = d[..., None] * np.arange(-127, 128)[None, None, None, :]
    err = np.abs(xb[..., None] - grid)
    chosen = np.take_along_axis(err, (qb + 127)[..., None], 3)[..., 0]
    assert np.all(chosen <= err.min(axis=3) + 1e-6 * d)
    assert np.all(np.abs(xb - d * qb) <= d / 2 * (1 + 2**-20) + 1e-30)


def test_q8_0_bf16_input_is_widened_exactly():
    xb = inputs.randn((4, 256), seed=5).to(torch.bfloat16)
    a = oracle.quant_act_q8_0(xb.float().numpy())
    b = oracle.quant_act_q8_0(xb.to(torch.float64).numpy().astype(np.float32))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# ------------------------------------------------------------------ O4 contraction
@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (2, 3, 64), (3, 2, 96), (5, 7, 160), (4, 9, 352)])
def test_gemm_q4_0_brute_force_dequantised_f64(M, N, K):
    x = inputs.randn((M, K), seed=10 + M).numpy()
    w = inputs.randn((N, K), seed=20 + N, std=0.02).numpy()
    qx, dx, sx = oracle.quant_act_q8_0(x)
    qs, d = oracle.pack_q4_0(w)
    y, T = oracle.gemm_q4_0(qx, dx, qs, d)
    want = ref.q8_0_values(qx, dx) @ ref.q4_0_weights(qs, d).T
    assert np.all(np.abs(y - want) <= 1e-12 * T + 1e-300)
    # T is the sum of |block terms|: never below |y|
    assert np.all(T >= np.abs(y))


def test_gemm_q4_0_unit_scales_is_integer_matmul():
    rng = np.random.default_rng(6)
    M, N, K = 6, 5, 128
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    codes = rng.integers(0, 16, size=(N, K))
    blocks = codes.reshape(N, K // 32, 32)
    qs = (blocks[:, :, :16] | (blocks[:, :, 16:] << 4)).reshape(N, K // 2).astype(np.uint8)
    d = np.full((N, K // 32), 0x3C00, dtype=np.uint16)  # fp16 1.0
    dx = np.ones((M, K // 32), dtype=np.float32)
    y, _ = oracle.gemm_q4_0(qx, dx, qs, d)
    want = qx.astype(np.int64) @ (codes - 8).T.astype(np.int64)
    assert np.array_equal(y, want.astype(np.float64))


def test_gemm_q4_0_sampled_and_threads_match_full():
    wl = inputs.MINILM
    x, w = inputs.make(wl, M=16, N=96)
    qx, dx, _ = oracle.quant_act_q8_0(x.numpy())
    qs, d = oracle.pack_q4_0(w.numpy())
    y1, T1 = oracle.gemm_q4_0(qx, dx, qs, d, nthreads=1)
    y4, T4 = oracle.gemm_q4_0(qx, dx, qs, d, nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(T1, T4)
    ms, ns = inputs.sample_indices(16, 96, 50)
    ys, Ts = oracle.gemm_q4_0_sampled(qx, dx, qs, d, ms, ns)
    assert np.array_equal(ys, y1[ms, ns]) and np.array_equal(Ts, T1[ms, ns])


def test_f32_block_rescale_meets_tolerance():
    """Plain sequential f32 per-block rescaling stays within 1e-5 * sum|terms|."""
    x, w = inputs.make(inputs.MINILM)
    qx, dx, _ = oracle.quant_act_q8_0(x.numpy())
    qs, d = oracle.pack_q4_0(w.numpy())
    y, T = oracle.gemm_q4_0(qx, dx, qs, d, nthreads=8)
    y32 = oracle.gemm_q4_0_f32(qx, dx, qs, d)
    assert np.all(np.abs(y32 - y) <= 1e-5 * T)


def test_q4_0_accuracy_band_minilm_shape():
    x, w = inputs.make(inputs.MINILM)
    qx, dx, _ = oracle.quant_act_q8_0(x.numpy())
    qs, d = oracle.pack_q4_0(w.numpy())
    y, _ = oracle.gemm_q4_0(qx, dx, qs, d, nthreads=8)
    exact = x.double().numpy() @ w.double().numpy().T
    rel = np.sqrt(np.mean((y - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    cos = np.sum(y * exact) / np.linalg.norm(y) / np.linalg.norm(exact)
    assert 0.05 < rel < 0.12, rel
    assert cos > 0.99


# ------------------------------------------------------------------ O5 affine pack
def test_affine_golden_grid():
    g = ref.read_golden(os.path.join(GOLDEN, "affine_grid.txt"))
    codes = np.arange(64) % 16
    w = (-1.0 + 0.125 * codes).astype(np.float32)[None, :]
    q, s, b = oracle.pack_affine(w, 64)
    assert [int(v) for v in q[0]] == [int(v, 16) for v in g["words"]]
    assert int(s[0, 0]) == int(g["scale_bf16_bits"][0], 16)
    assert int(b[0, 0]) == int(g["bias_bf16_bits"][0], 16)


@pytest.mark.parametrize("group", [64, 128])
def test_affine_grid_round_trip_and_invariants(group):
    rng = np.random.default_rng(7)
    N, K = 8, 512
    codes = rng.integers(0, 16, size=(N, K))
    codes[:, ::group] = 0
    codes[:, 1::group] = 15
    s = (2.0 ** rng.integers(-6, 0, size=(N, K // group))).astype(np.float32)
    b = (-(2.0 ** rng.integers(-3, 2, size=(N, K // group)))).astype(np.float32)
    w = (np.repeat(s, group, 1) * codes + np.repeat(b, group, 1)).astype(np.float32)
    q, sb, bb = oracle.pack_affine(w, group)
    assert np.array_equal(ref.affine_codes(q), codes)
    assert np.array_equal(ref.bf16_bits_to_f64(sb), s.astype(np.float64))
    assert np.array_equal(ref.bf16_bits_to_f64(bb), b.astype(np.float64))
    # random weights: codes in range, constant group gives s = 0, codes 0, w = b
    w2 = inputs.randn((8, 512), seed=8).numpy()
    w2[2, :group] = 0.375
    q2, s2, b2 = oracle.pack_affine(w2, group)
    c2 = ref.affine_codes(q2)
    assert c2.min() >= 0 and c2.max() <= 15
    assert ref.bf16_bits_to_f64(s2)[2, 0] == 0 and np.all(c2[2, :group] == 0)
    assert ref.bf16_bits_to_f64(b2)[2, 0] == 0.375
    # each code is a nearest grid point of s*q + b (brute force over the 16 codes)
    sv = np.repeat(ref.bf16_bits_to_f64(s2), group, 1)
    bv = np.repeat(ref.bf16_bits_to_f64(b2), group, 1)
    err = np.abs(w2[..., None] - (sv[..., None] * np.arange(16) + bv[..., None]))
    chosen = np.take_along_axis(err, c2[..., None], 2)[..., 0]
    assert np.all(chosen <= err.min(axis=2) + 1e-6 * sv + 1e-30)


# ------------------------------------------------------------------ O6 affine contraction
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (3, 2, 256), (5, 6, 384)])
def test_gemm_affine_brute_force(group, M, N, K):
    if K % group:
        pytest.skip("K not a multiple of the group")
    x = inputs.randn((M, K), seed=30 + M).numpy()
    w = inputs.randn((N, K), seed=40 + N).numpy()
    qx, dx, sx = oracle.quant_act_q8_0(x)
    q, s, b = oracle.pack_affine(w, group)
    y, T = oracle.gemm_affine(qx, dx, sx, q, s, b, group)
    want = ref.q8_0_values(qx, dx) @ ref.affine_weights(q, s, b, group).T
    assert np.all(np.abs(y - want) <= 1e-12 * T + 1e-300)


def test_affine_with_bias_minus_8s_equals_q4_0():
    """An affine group with bias = -8*scale holds the same weights as Q4_0 blocks with
    d = scale and the same codes, so the two contractions agree."""
    rng = np.random.default_rng(9)
    M, N, K, group = 4, 6, 256, 64
    codes = rng.integers(0, 16, size=(N, K))
    scale = (2.0 ** rng.integers(-8, -4, size=(N, K // group))).astype(np.float32)
    x = inputs.randn((M, K), seed=11).numpy()
    qx, dx, sx = oracle.quant_act_q8_0(x)
    words = (codes.reshape(N, K // 8, 8) << (4 * np.arange(8))).sum(axis=2).astype(np.uint32)
    s_bits = torch.from_numpy(scale).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    b_bits = torch.from_numpy(-8 * scale).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ya, Ta = oracle.gemm_affine(qx, dx, sx, words, s_bits, b_bits, group)
    blocks = codes.reshape(N, K // 32, 32)
    qs = (blocks[:, :, :16] | (blocks[:, :, 16:] << 4)).reshape(N, K // 2).astype(np.uint8)
    d_bits = np.repeat(scale, group // 32, axis=1).astype(np.float16).view(np.uint16)
    yq, Tq = oracle.gemm_q4_0(qx, dx, qs, d_bits)
    assert np.all(np.abs(ya - yq) <= 1e-12 * Tq)


@pytest.mark.parametrize("group", [64, 128])
def test_affine_accuracy_matches_mlx_table(group):
    """Relative RMS error against the f32 matmul of the unquantised inputs, on the MLX
    accuracy setup (M=1024, K=N=4096, normal x and w, bf16); 64 of the 1024 rows."""
    rows = {r[0]: float(r[1]) for r in ref.read_golden(os.path.join(GOLDEN, "affine_accuracy.txt"))["rows"]}
    wl = inputs.AFFINE_GS64 if group == 64 else inputs.AFFINE_GS128
    x, w = inputs.make(wl)
    x = x[:64]
    w = w.to(torch.bfloat16).float()
    qx, dx, sx = oracle.quant_act_q8_0(x.float().numpy())
    q, s, b = oracle.pack_affine(w.numpy(), group)
    y, _ = oracle.gemm_affine(qx, dx, sx, q, s, b, group, nthreads=8)
    exact = x.double().numpy() @ w.double().numpy().T
    rel = 100 * np.sqrt(np.mean((y - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    page = rows[str(group)]
    assert abs(rel - page) < 0.6, (rel, page)

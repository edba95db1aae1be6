"""Pins for the oracle's Q4_K GEMV and its input-gradient backward (no GPU): the hand-worked
scale packing, brute force over every 6-bit scale and min, an independent numpy decoder of
the super-block layout, f64 matmuls of the decoded weights, the adjoint identity between
the forward and the backward, and the integer special case."""
import os

import numpy as np
import pytest

import oracle
from block_quantized_w4a8_b200 import inputs
from tests import refdecode as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pack_scales(sc, m):
    """Inverse of the scale packing, written from the layout (for the brute-force pin)."""
    s = np.zeros(12, dtype=np.int64)
    for j in range(4):
        s[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        s[j + 4] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        s[j + 8] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    return s.astype(np.uint8)


def test_q4_k_scales_golden():
    g = ref.read_golden(os.path.join(GOLDEN, "q4_k_scales.txt"))
    s = np.array([int(v, 16) for v in g["bytes"]], dtype=np.uint8)
    sc, m = oracle.q4_k_unpack_scales(s)
    assert list(sc) == [int(v) for v in g["sc"]] and list(m) == [int(v) for v in g["m"]]
    rsc, rm = ref.q4_k_scales(s)
    assert list(rsc) == list(sc) and list(rm) == list(m)


def test_q4_k_scales_round_trip_every_value():
    """Every 6-bit value in every one of the 16 slots survives pack -> unpack."""
    rng = np.random.default_rng(4)
    for v in range(64):
        for slot in range(16):
            sc = rng.integers(0, 64, 8)
            m = rng.integers(0, 64, 8)
            (sc if slot < 8 else m)[slot % 8] = v
            got_sc, got_m = oracle.q4_k_unpack_scales(_pack_scales(sc, m))
            assert np.array_equal(got_sc, sc) and np.array_equal(got_m, m)


def test_q4_k_dequant_matches_independent_decoder():
    N, K = 7, 768
    W = inputs.make_q4_k(N, K, seed=5).numpy()
    assert np.array_equal(oracle.dequant_q4_k(W, N, K), ref.q4_k_weights(W, N, K))


def test_q4_k_dequant_hand_block():
    """One super-block built by hand: d = 1, dmin = 0.5, sc = 1..8, m = 0..7, low nibble of
    qs[l] = l % 16, high nibble = 15 - l % 16."""
    blk = np.zeros(144, dtype=np.uint8)
    blk[0:2] = np.array([1.0], np.float16).view(np.uint8)
    blk[2:4] = np.array([0.5], np.float16).view(np.uint8)
    blk[4:16] = _pack_scales(np.arange(1, 9), np.arange(8))
    lo = np.arange(128) % 16
    blk[16:] = (lo | ((15 - lo) << 4)).astype(np.uint8)
    w = oracle.dequant_q4_k(blk, 1, 256)[0]
    # element 64i + l: sub-block 2i, code l % 16 (l < 32); 64i + 32 + l: sub-block 2i + 1, 15 - l % 16
    assert w[0] == 0.0 and w[5] == 1 * 5 - 0.0
    assert w[32 + 3] == 2 * 12 - 0.5 * 1            # sub-block 1: sc 2, m 1, code 15 - 3
    assert w[64 + 17] == 3 * 1 - 0.5 * 2            # sub-block 2: code (32 + 17) % 16 = 1
    assert w[255] == 8 * (15 - 15) - 0.5 * 7        # sub-block 7: qs[127] high nibble = 15 - 15


@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (2, 3, 512), (3, 5, 768)])
def test_gemv_q4_k_brute_force(M, N, K):
    W = inputs.make_q4_k(N, K, seed=M + N).numpy()
    x = inputs.randn((M, K), seed=9).numpy()
    y, T = oracle.gemv_q4_k(x, W, N)
    want = x.astype(np.float64) @ ref.q4_k_weights(W, N, K).T
    assert np.all(np.abs(y - want) <= 1e-12 * T)


@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (2, 3, 512), (3, 5, 768)])
def test_gemv_q4_k_backward_brute_force(M, N, K):
    W = inputs.make_q4_k(N, K, seed=M * N).numpy()
    dy = inputs.randn((M, N), seed=10).numpy()
    dx, T = oracle.gemv_q4_k_backward(dy, W, K)
    want = dy.astype(np.float64) @ ref.q4_k_weights(W, N, K)
    assert np.all(np.abs(dx - want) <= 1e-12 * T)


def test_backward_is_the_adjoint_of_the_forward():
    """u . (x W^T) == (u W) . x for the same Q4_K W (sums in f64)."""
    N, K = 37, 512
    W = inputs.make_q4_k(N, K, seed=12).numpy()
    x = inputs.randn((1, K), seed=13).numpy()
    u = inputs.randn((1, N), seed=14).numpy()
    y, Ty = oracle.gemv_q4_k(x, W, N)
    dx, Tx = oracle.gemv_q4_k_backward(u, W, K)
    lhs = float(u[0].astype(np.float64) @ y[0])
    rhs = float(dx[0] @ x[0].astype(np.float64))
    assert abs(lhs - rhs) <= 1e-12 * float(np.abs(u[0]) @ Ty[0])


def test_q4_k_unit_scales_is_integer_matmul():
    """d = 1, dmin = 0, every sc = 1: the weights are the codes, so with integer x the
    forward is an integer matmul."""
    N, K = 6, 512
    W = inputs.make_q4_k(N, K, seed=15).numpy().reshape(N, K // 256, 144)
    W[..., 0:2] = np.array([1.0], np.float16).view(np.uint8)
    W[..., 2:4] = 0
    W[..., 4:16] = _pack_scales(np.ones(8, np.int64), np.zeros(8, np.int64))
    W = W.reshape(N, -1)
    codes = np.concatenate([W.reshape(N, K // 256, 144)[..., 16:].reshape(N, K // 256, 4, 32) & 15,
                            W.reshape(N, K // 256, 144)[..., 16:].reshape(N, K // 256, 4, 32) >> 4],
                           axis=-1).reshape(N, K).astype(np.int64)
    x = np.random.default_rng(3).integers(-50, 50, size=(2, K))
    y, _ = oracle.gemv_q4_k(x.astype(np.float32), W, N)
    assert np.array_equal(y, (x @ codes.T).astype(np.float64))


def test_oracle_agrees_with_the_pages_f32_sequence():
    """The page's scalar GEMV in f32 (d1 = d*sc, m1 = dmin*m, w = d1*q - m1, then
    sum += w * x element after element), written here with numpy float32 and a sequential
    accumulation, is within the f32 bound (K + 2) * 2^-24 * T of the oracle's f64 result."""
    N, K = 9, 1024
    W = inputs.make_q4_k(N, K, seed=31).numpy()
    x = inputs.randn((1, K), seed=32).numpy().astype(np.float32)
    b = W.reshape(N, K // 256, 144)
    d = b[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float32)
    dmin = b[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float32)
    sc, m = ref.q4_k_scales(b[..., 4:16])
    qs = b[..., 16:].reshape(N, K // 256, 4, 32).astype(np.int64)
    codes = np.concatenate([qs & 15, qs >> 4], axis=-1).reshape(N, K // 256, 256).astype(np.float32)
    sub = np.arange(256) // 32
    d1 = (d[..., None] * sc[..., sub].astype(np.float32)).astype(np.float32)
    m1 = (dmin[..., None] * m[..., sub].astype(np.float32)).astype(np.float32)
    w = (d1 * codes).astype(np.float32) - m1                      # f32 subtraction, rounded
    terms = (w.reshape(N, K) * x[0][None, :]).astype(np.float32)  # f32 products, rounded
    y32 = np.add.accumulate(terms, axis=1, dtype=np.float32)[:, -1].astype(np.float64)
    y, T = oracle.gemv_q4_k(x, W, N)
    assert np.all(np.abs(y32 - y[0]) <= (K + 2) * 2.0 ** -24 * T[0])

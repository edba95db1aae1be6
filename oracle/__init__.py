"""Scalar CPU oracle for the block-quantized W4A8 matmul (Q4_0 x Q8_0) and its affine
4-, 6- and 8-bit variants.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference leg are the only callers. The CUDA library never imports,
links or runs anything here, and nothing here touches the CUDA library.

The arithmetic lives in ``oracle.cpp`` (plain scalar C++, built with
``-O2 -ffp-contract=off``); this module only marshals numpy arrays to it.

Functions and the definitions they follow (see the header of ``oracle.cpp``):

* ``f32_to_f16`` / ``f32_to_bf16`` / ``f16_to_f32`` / ``bf16_to_f32`` -- IEEE 754
  round-to-nearest-even narrowing and exact widening.
* ``pack_q4_0`` -- Q4_0 weights (tract PR #2432, "The kernel": 4-bit N x K weight,
  per-32-block scale), d = mx/-8, q = min(15, trunc(x/d + 8.5)).
* ``quant_act_q8_0`` -- Q8_0 activations (tract PR #2432, "Pipeline": activation to int8
  per block), d = amax/127 in f32, q = round-half-away(x * (1/d)).
* ``gemm_q4_0`` -- y = x . W^T as sum over blocks of d_w * d_x * (exact int block dot),
  in f64 (each term exact), plus T = sum of |terms| (the tolerance scale).
* ``pack_affine`` / ``gemm_affine`` -- MLX PR #4802 "mx.qqmm ... mode=affine": codes
  q in [0, 2^bits - 1] (bits 4, 6 or 8), per-group (32, 64 or 128) bf16 scale
  (max-min)/(2^bits - 1) and bias min; the contraction runs on the original codes and
  applies d_x * (s * sum q q_x + b * sum q_x) per block. Codes of a row are a
  little-endian bit stream (4 bits: eight codes per 32-bit word, element k at bits
  4*(k%8) of word k/8).
* ``q4_k_unpack_scales`` / ``dequant_q4_k`` / ``gemv_q4_k`` / ``gemv_q4_k_backward`` --
  C-Kernel-Engine gemm_kernels_q4k.c ("GEMV: y = W @ x", "Backward Pass: Gradient w.r.t.
  Input"): Q4_K super-blocks of 256 (w = d*sc*q - dmin*m per 32-element sub-block) with
  FP32 activations, y = x W^T and dX = dY W, in f64 with T = sum of |terms|.
* ``epilogue`` -- the output of a linear layer: the optional per-column bias added to
  every row of the f32 product in f32 (C-Kernel-Engine gemm_kernels_q4k.c, "Engine-
  compatible wrapper: GEMM_NT with Q4_K weights"), then f32 or bf16 (nearest even).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.cpp`` into ``liboracle.so`` (g++, -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-pthread", _SRC, "-o", _LIB_PATH + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    sigs = {
        "orc_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float]),
        "orc_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
        "orc_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "orc_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "orc_f32_to_f16_array": (None, [P, P, I64]),
        "orc_f32_to_bf16_array": (None, [P, P, I64]),
        "orc_f16_to_f32_array": (None, [P, P, I64]),
        "orc_bf16_to_f32_array": (None, [P, P, I64]),
        "orc_pack_q4_0": (None, [P, I, I, P, P]),
        "orc_dequant_q4_0": (None, [P, P, I, I, P]),
        "orc_quant_act_q8_0": (None, [P, I, I, P, P, P]),
        "orc_dequant_q8_0": (None, [P, P, I, I, P]),
        "orc_gemm_q4_0": (None, [I, I, I, P, P, P, P, P, P, I]),
        "orc_gemm_q4_0_sampled": (None, [I, I, P, P, P, P, P, P, P, P]),
        "orc_gemm_q4_0_f32": (None, [I, I, I, P, P, P, P, P]),
        "orc_pack_affine_bits": (None, [P, I, I, I, I, P, P, P]),
        "orc_q4_k_unpack_scales": (None, [P, P, P]),
        "orc_dequant_q4_k": (None, [P, I, I, P]),
        "orc_gemv_q4_k": (None, [I, I, I, P, P, P, P, I]),
        "orc_gemv_q4_k_backward": (None, [I, I, I, P, P, P, P, I]),
        "orc_dequant_affine_bits": (None, [P, P, P, I, I, I, I, P]),
        "orc_gemm_affine_bits": (None, [I, I, I, I, I, P, P, P, P, P, P, P, P, I]),
        "orc_gemm_affine_bits_sampled": (None, [I, I, I, I, P, P, P, P, P, P, P, P, P, P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


# ----------------------------------------------------------------------------- O1
def f32_to_f16(a) -> np.ndarray:
    a = _f32(a)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().orc_f32_to_f16_array(_p(a), _p(out), a.size)
    return out


def f32_to_bf16(a) -> np.ndarray:
    a = _f32(a)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().orc_f32_to_bf16_array(_p(a), _p(out), a.size)
    return out


def f16_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(np.asarray(h, dtype=np.uint16))
    out = np.empty(h.shape, dtype=np.float32)
    _load().orc_f16_to_f32_array(_p(h), _p(out), h.size)
    return out


def bf16_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(np.asarray(h, dtype=np.uint16))
    out = np.empty(h.shape, dtype=np.float32)
    _load().orc_bf16_to_f32_array(_p(h), _p(out), h.size)
    return out


# ----------------------------------------------------------------------------- O2
def pack_q4_0(w) -> tuple[np.ndarray, np.ndarray]:
    """W (N, K) f32 -> (qs uint8 (N, K/2), d fp16 bits uint16 (N, K/32))."""
    w = _f32(w)
    N, K = w.shape
    assert K % 32 == 0
    qs = np.empty((N, K // 2), dtype=np.uint8)
    d = np.empty((N, K // 32), dtype=np.uint16)
    _load().orc_pack_q4_0(_p(w), N, K, _p(qs), _p(d))
    return qs, d


def dequant_q4_0(qs: np.ndarray, d: np.ndarray) -> np.ndarray:
    N, K2 = qs.shape
    K = 2 * K2
    out = np.empty((N, K), dtype=np.float64)
    _load().orc_dequant_q4_0(_p(np.ascontiguousarray(qs)), _p(np.ascontiguousarray(d)), N, K, _p(out))
    return out


# ----------------------------------------------------------------------------- O3
def quant_act_q8_0(x) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """x (M, K) f32 -> (qx int8 (M, K), dx f32 (M, K/32), sx int32 (M, K/32))."""
    x = _f32(x)
    M, K = x.shape
    assert K % 32 == 0
    qx = np.empty((M, K), dtype=np.int8)
    dx = np.empty((M, K // 32), dtype=np.float32)
    sx = np.empty((M, K // 32), dtype=np.int32)
    _load().orc_quant_act_q8_0(_p(x), M, K, _p(qx), _p(dx), _p(sx))
    return qx, dx, sx


def dequant_q8_0(qx: np.ndarray, dx: np.ndarray) -> np.ndarray:
    M, K = qx.shape
    out = np.empty((M, K), dtype=np.float64)
    _load().orc_dequant_q8_0(_p(np.ascontiguousarray(qx)), _p(np.ascontiguousarray(dx)), M, K, _p(out))
    return out


# ----------------------------------------------------------------------------- O4
def gemm_q4_0(qx, dx, qs, d, nthreads: int = 1) -> tuple[np.ndarray, np.ndarray]:
    """-> (y f64 (M, N), T f64 (M, N)) with T = sum over blocks of |term|."""
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    dx = np.ascontiguousarray(dx, dtype=np.float32)
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    d = np.ascontiguousarray(d, dtype=np.uint16)
    M, K = qx.shape
    N = qs.shape[0]
    assert qs.shape[1] * 2 == K and d.shape == (N, K // 32) and dx.shape == (M, K // 32)
    y = np.empty((M, N), dtype=np.float64)
    T = np.empty((M, N), dtype=np.float64)
    _load().orc_gemm_q4_0(M, N, K, _p(qx), _p(dx), _p(qs), _p(d), _p(y), _p(T), int(nthreads))
    return y, T


def gemm_q4_0_sampled(qx, dx, qs, d, ms, ns) -> tuple[np.ndarray, np.ndarray]:
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    dx = np.ascontiguousarray(dx, dtype=np.float32)
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    d = np.ascontiguousarray(d, dtype=np.uint16)
    ms = np.ascontiguousarray(ms, dtype=np.int32)
    ns = np.ascontiguousarray(ns, dtype=np.int32)
    K = qx.shape[1]
    y = np.empty(ms.shape, dtype=np.float64)
    T = np.empty(ms.shape, dtype=np.float64)
    _load().orc_gemm_q4_0_sampled(K, ms.size, _p(ms), _p(ns), _p(qx), _p(dx), _p(qs), _p(d), _p(y), _p(T))
    return y, T


def gemm_q4_0_f32(qx, dx, qs, d) -> np.ndarray:
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    dx = np.ascontiguousarray(dx, dtype=np.float32)
    qs = np.ascontiguousarray(qs, dtype=np.uint8)
    d = np.ascontiguousarray(d, dtype=np.uint16)
    M, K = qx.shape
    N = qs.shape[0]
    y = np.empty((M, N), dtype=np.float32)
    _load().orc_gemm_q4_0_f32(M, N, K, _p(qx), _p(dx), _p(qs), _p(d), _p(y))
    return y


# ----------------------------------------------------------------------------- O5
def _codes_bytes(q) -> np.ndarray:
    """The packed codes as the rows' little-endian byte streams (a 4-bit u32 word array is
    the same bytes on a little-endian host)."""
    q = np.ascontiguousarray(q)
    return q.view(np.uint8).reshape(q.shape[0], -1)


def pack_affine(w, group: int, bits: int = 4) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """W (N, K) f32 -> (codes, scale bf16 bits (N, K/g), bias bf16 bits (N, K/g)). The codes
    are uint32 (N, K/8) words for 4 bits, else uint8 (N, K*bits/8) bytes."""
    w = _f32(w)
    N, K = w.shape
    assert bits in (4, 6, 8) and K % group == 0 and group % 32 == 0
    q = np.empty((N, K * bits // 8), dtype=np.uint8)
    s = np.empty((N, K // group), dtype=np.uint16)
    b = np.empty((N, K // group), dtype=np.uint16)
    _load().orc_pack_affine_bits(_p(w), N, K, int(group), int(bits), _p(q), _p(s), _p(b))
    if bits == 4:
        q = q.view(np.uint32)
    return q, s, b


def dequant_affine(q, scale, bias, group: int, bits: int = 4) -> np.ndarray:
    q = _codes_bytes(q)
    N = q.shape[0]
    K = q.shape[1] * 8 // bits
    out = np.empty((N, K), dtype=np.float64)
    _load().orc_dequant_affine_bits(_p(q), _p(np.ascontiguousarray(scale, dtype=np.uint16)),
                                    _p(np.ascontiguousarray(bias, dtype=np.uint16)), N, K, int(group), int(bits),
                                    _p(out))
    return out


# ----------------------------------------------------------------------------- O6
def gemm_affine(qx, dx, sx, q, scale, bias, group: int, nthreads: int = 1, bits: int = 4
                ) -> tuple[np.ndarray, np.ndarray]:
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    dx = np.ascontiguousarray(dx, dtype=np.float32)
    sx = np.ascontiguousarray(sx, dtype=np.int32)
    q = _codes_bytes(q)
    scale = np.ascontiguousarray(scale, dtype=np.uint16)
    bias = np.ascontiguousarray(bias, dtype=np.uint16)
    M, K = qx.shape
    N = q.shape[0]
    assert q.shape[1] * 8 == K * bits and scale.shape == (N, K // group) and bias.shape == scale.shape
    y = np.empty((M, N), dtype=np.float64)
    T = np.empty((M, N), dtype=np.float64)
    _load().orc_gemm_affine_bits(M, N, K, int(group), int(bits), _p(qx), _p(dx), _p(sx), _p(q), _p(scale),
                                 _p(bias), _p(y), _p(T), int(nthreads))
    return y, T


def gemm_affine_sampled(qx, dx, sx, q, scale, bias, group: int, ms, ns, bits: int = 4
                        ) -> tuple[np.ndarray, np.ndarray]:
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    dx = np.ascontiguousarray(dx, dtype=np.float32)
    sx = np.ascontiguousarray(sx, dtype=np.int32)
    q = _codes_bytes(q)
    ms = np.ascontiguousarray(ms, dtype=np.int32)
    ns = np.ascontiguousarray(ns, dtype=np.int32)
    K = qx.shape[1]
    assert q.shape[1] * 8 == K * bits
    y = np.empty(ms.shape, dtype=np.float64)
    T = np.empty(ms.shape, dtype=np.float64)
    _load().orc_gemm_affine_bits_sampled(K, int(group), int(bits), ms.size, _p(ms), _p(ns), _p(qx), _p(dx),
                                         _p(sx), _p(q), _p(np.ascontiguousarray(scale, dtype=np.uint16)),
                                         _p(np.ascontiguousarray(bias, dtype=np.uint16)), _p(y), _p(T))
    return y, T


# ----------------------------------------------------------------------------- O7 Q4_K
def q4_k_unpack_scales(s) -> tuple[np.ndarray, np.ndarray]:
    """The 12 packed scale bytes of a Q4_K super-block -> (sc[8], m[8]), 6 bits each."""
    s = np.ascontiguousarray(s, dtype=np.uint8)
    assert s.shape == (12,)
    sc = np.empty(8, dtype=np.uint8)
    m = np.empty(8, dtype=np.uint8)
    _load().orc_q4_k_unpack_scales(_p(s), _p(sc), _p(m))
    return sc, m


def dequant_q4_k(W, N: int, K: int) -> np.ndarray:
    """Q4_K weights (N rows x K/256 super-blocks of 144 bytes) -> f64 (N, K)."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    assert W.size == N * (K // 256) * 144
    out = np.empty((N, K), dtype=np.float64)
    _load().orc_dequant_q4_k(_p(W), N, K, _p(out))
    return out


def gemv_q4_k(x, W, N: int, nthreads: int = 1) -> tuple[np.ndarray, np.ndarray]:
    """y = x . W^T for FP32 x (M, K) and Q4_K W (N rows); f64 y (M, N) and T."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.uint8)
    M, K = x.shape
    assert K % 256 == 0 and W.size == N * (K // 256) * 144
    y = np.empty((M, N), dtype=np.float64)
    T = np.empty((M, N), dtype=np.float64)
    _load().orc_gemv_q4_k(M, N, K, _p(x), _p(W), _p(y), _p(T), int(nthreads))
    return y, T


def gemv_q4_k_backward(dy, W, K: int, nthreads: int = 1) -> tuple[np.ndarray, np.ndarray]:
    """dX = dY . W for FP32 dY (M, N) and Q4_K W (N rows, K columns); f64 dX (M, K) and T."""
    dy = np.ascontiguousarray(dy, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.uint8)
    M, N = dy.shape
    assert K % 256 == 0 and W.size == N * (K // 256) * 144
    dx = np.empty((M, K), dtype=np.float64)
    T = np.empty((M, K), dtype=np.float64)
    _load().orc_gemv_q4_k_backward(M, N, K, _p(dy), _p(W), _p(dx), _p(T), int(nthreads))
    return dx, T


def epilogue(p, bias=None, bias_bf16: bool = False, out_bf16: bool = False) -> np.ndarray:
    """Output epilogue: y[m][n] = f32(p[m][n]) + f32(bias[n]) with one f32 rounding
    (C-Kernel-Engine gemm_kernels_q4k.c, "Engine-compatible wrapper: GEMM_NT with Q4_K
    weights": after the product, ``row[j] += bias[j]`` for every row), no addition when
    ``bias`` is None; a bf16 output is that value narrowed to bf16 with round-to-nearest-even
    (returned as uint16 bit patterns). ``bias`` is f32 values, or bf16 bit patterns when
    ``bias_bf16``."""
    y = np.asarray(p, dtype=np.float32)
    if bias is not None:
        b = bf16_to_f32(bias) if bias_bf16 else np.asarray(bias, dtype=np.float32)
        y = (y + b.reshape(1, -1)).astype(np.float32)  # IEEE single-precision addition
    if out_bf16:
        return f32_to_bf16(y)
    return y

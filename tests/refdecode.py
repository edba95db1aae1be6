"""Independent numpy decoders of the packed formats, used only to pin the oracle.

They restate the storage layouts from the format definitions (not from the oracle's
code) so that a layout or indexing mistake in the oracle shows up as a mismatch:

* Q4_0: row n, block b = 16 bytes at n*K/2 + 16b; byte j low nibble = element 32b+j,
  high nibble = element 32b+j+16; w = fp16(d) * (q - 8).
* Q8_0: x = d * q with one f32 d per 32-block.
* affine: element k of row n at bits 4*(k%8) of uint32 word k/8; w = s*q + b with bf16
  s and b per group.
* affine with `bits`-bit codes: the row's bytes read as one little-endian bit stream,
  element k = bits [bits*k, bits*k + bits).
"""
import numpy as np
import torch


def q4_0_codes(qs: np.ndarray) -> np.ndarray:
    N, K2 = qs.shape
    blocks = qs.reshape(N, K2 // 16, 16)
    lo = blocks & 0x0F
    hi = blocks >> 4
    return np.concatenate([lo, hi], axis=2).reshape(N, K2 * 2).astype(np.int64)


def fp16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def q4_0_weights(qs: np.ndarray, d: np.ndarray) -> np.ndarray:
    codes = q4_0_codes(qs)
    scales = np.repeat(fp16_bits_to_f64(d), 32, axis=1)
    return scales * (codes - 8)


def q8_0_values(qx: np.ndarray, dx: np.ndarray) -> np.ndarray:
    return np.repeat(dx.astype(np.float64), 32, axis=1) * qx.astype(np.float64)


def affine_codes(q: np.ndarray) -> np.ndarray:
    N, W = q.shape
    shifts = (4 * np.arange(8, dtype=np.uint32))[None, None, :]
    return ((q[:, :, None] >> shifts) & 0xF).reshape(N, W * 8).astype(np.int64)


def affine_weights(q: np.ndarray, scale: np.ndarray, bias: np.ndarray, group: int) -> np.ndarray:
    codes = affine_codes(q)
    s = np.repeat(bf16_bits_to_f64(scale), group, axis=1)
    b = np.repeat(bf16_bits_to_f64(bias), group, axis=1)
    return s * codes + b


def read_golden(path):
    out = {}
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                out[k.strip()] = v.split()
            else:
                rows.append(line.split())
    if rows:
        out["rows"] = rows
    return out


def affine_codes_bits(q: np.ndarray, bits: int) -> np.ndarray:
    qb = np.ascontiguousarray(q).view(np.uint8)
    N = qb.shape[0]
    stream = np.unpackbits(qb.reshape(N, -1), axis=1, bitorder="little")  # bit i of byte j at 8j + i
    K = stream.shape[1] // bits
    return (stream.reshape(N, K, bits).astype(np.int64) << np.arange(bits)).sum(axis=2)


def affine_weights_bits(q: np.ndarray, scale: np.ndarray, bias: np.ndarray, group: int, bits: int) -> np.ndarray:
    codes = affine_codes_bits(q, bits)
    s = np.repeat(bf16_bits_to_f64(scale), group, axis=1)
    b = np.repeat(bf16_bits_to_f64(bias), group, axis=1)
    return s * codes + b


def q4_k_scales(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """(..., 12) scale bytes -> (..., 8) sub-block scales and mins of 6 bits (llama.cpp
    Q4_K packing: the low 6 bits of bytes 0-3 / 4-7 are sc / m of sub-blocks 0-3; sub-blocks
    4-7 take their low 4 bits from the nibbles of bytes 8-11 and their top 2 bits from the
    top 2 bits of bytes 0-3 (sc) and 4-7 (m))."""
    s = s.astype(np.int64)
    sc = np.concatenate([s[..., 0:4] & 63, (s[..., 8:12] & 15) | ((s[..., 0:4] >> 6) << 4)], axis=-1)
    m = np.concatenate([s[..., 4:8] & 63, (s[..., 8:12] >> 4) | ((s[..., 4:8] >> 6) << 4)], axis=-1)
    return sc, m


def q4_k_weights(W: np.ndarray, N: int, K: int) -> np.ndarray:
    """Q4_K rows (N, K/256*144 bytes) -> f64 weights (N, K)."""
    b = np.ascontiguousarray(W, dtype=np.uint8).reshape(N, K // 256, 144)
    d = b[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    dmin = b[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    sc, m = q4_k_scales(b[..., 4:16])
    qs = b[..., 16:].reshape(N, K // 256, 4, 32).astype(np.int64)
    codes = np.concatenate([qs & 15, qs >> 4], axis=-1).reshape(N, K // 256, 256)  # per 64: low 32, high 32
    sub = np.arange(256) // 32                                                      # sub-block of each element
    w = d[..., None] * sc[..., sub] * codes - dmin[..., None] * m[..., sub]
    return w.reshape(N, K)

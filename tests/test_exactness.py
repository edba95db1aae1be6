"""Host-side check of the arithmetic the tensor-core path relies on (no GPU): the weight
operand of the tcgen05 GEMM holds each Q4_0 weight d*(q-8) as two fp16 values
d_hi*(q-8) + d_lo*(q-8), d_hi = d with its three lowest significand bits cleared, and each
affine weight as s*(q-8) with the bf16 group scale s. Both are formed in the kernel by one
fused multiply-add (8 + q/2)*(2d) - 24d. This test checks, for every finite fp16 scale
within the documented range and every code, that the split is exact, that each product and
the fused form's addend are representable in fp16 (so a single rounding returns the exact
value), and that the range bound is tight. The same for the 6- and 8-bit affine codes of
the CTA-pair kernel ((1024 + q) * s_part - (1024 + c) * s_part with the bf16 scale split
into two parts; every bf16 scale in range, every code) and for the two-part fp16 column
of the bias MMA."""
import numpy as np


def _fp16_exact(v):
    v = np.asarray(v, dtype=np.float64)
    return np.all(v.astype(np.float16).astype(np.float64) == v)


def test_q4_0_scale_split_is_exact_in_fp16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    d = bits.view(np.float16).astype(np.float64)
    hi_bits = bits & np.uint16(0xFFF8)
    ok = np.isfinite(d) & (np.abs(hi_bits.view(np.float16).astype(np.float64)) <= 2720.0)
    d, dh = d[ok], hi_bits[ok].view(np.float16).astype(np.float64)
    dl = d - dh
    assert _fp16_exact(dl)
    for part in (dh, dl):
        assert _fp16_exact(24.0 * part)          # the fused multiply-add's addend
        assert _fp16_exact(2.0 * part)           # its multiplier
        for q in range(16):
            assert _fp16_exact(part * (q - 8))   # the operand value
            # (8 + q/2) * 2d - 24d equals (q - 8) * d exactly (no rounding needed)
            assert np.all((8.0 + q / 2.0) * (2.0 * part) - 24.0 * part == part * (q - 8))


def test_q4_0_range_bound_is_tight():
    # the first d_hi above 2720 makes 24 * d_hi overflow fp16
    above = np.array([0x6958], dtype=np.uint16).view(np.float16).astype(np.float64)[0]
    assert above > 2720.0 and 24.0 * above > 65504.0


def test_affine_scale_times_centred_code_is_exact_in_fp16():
    bits = (np.arange(1 << 16, dtype=np.uint64) << 16).astype(np.uint32)
    with np.errstate(invalid="ignore"):
        s = bits.view(np.float32).astype(np.float64)
    a = np.abs(s)
    ok = np.isfinite(s) & (((a >= 2.0 ** -17) & (a <= 2720.0)) | (a == 0))
    s = s[ok]
    assert _fp16_exact(s) and _fp16_exact(24.0 * s)
    for q in range(16):
        assert _fp16_exact(s * (q - 8))
    # just below the range the products are no longer exact
    tiny = np.array([2.0 ** -18 * (1 + 1 / 128)])
    assert not all(_fp16_exact(tiny * (q - 8)) for q in range(16))


def _bf16_scales(lo, hi):
    """Every finite bf16 value with lo <= |s| <= hi, or 0, as f64."""
    bits = (np.arange(1 << 16, dtype=np.uint64) << 16).astype(np.uint32)
    with np.errstate(invalid="ignore"):
        s = bits.view(np.float32).astype(np.float64)
    a = np.abs(s)
    ok = np.isfinite(s) & (((a >= lo) & (a <= hi)) | (a == 0))
    return s[ok], (bits[ok] >> 16).astype(np.uint16)


def test_wide_affine_codes_expand_exactly():
    """6- and 8-bit affine codes on the CTA-pair kernel: the bf16 scale s splits into s_hi
    (its top 4 significant bits for 8-bit codes, 5 for 6-bit; the bf16 bit pattern with the
    low 4 or 3 significand bits cleared) and s_lo = s - s_hi; each part is exact in fp16,
    the addend -(1024 + c) * s_part of the fused multiply-add is exact in fp16, and the
    result (1024 + q) * s_part - (1024 + c) * s_part = (q - c) * s_part is representable,
    so its single rounding is exact, for every bf16 scale 2^-17 <= |s| <= 32 and every code;
    1024 + q itself is exact (the binade [1024, 2048) has unit spacing)."""
    for bits, mask, c in ((8, 0xFFF0, 128), (6, 0xFFF8, 32)):
        s, sb = _bf16_scales(2.0 ** -17, 32.0)
        hb = (sb & np.uint16(mask)).astype(np.uint32) << 16
        s_hi = hb.view(np.float32).astype(np.float64)
        s_lo = s - s_hi
        assert np.all(s_hi + s_lo == s)
        q = np.arange(1 << bits, dtype=np.float64)
        assert _fp16_exact(1024.0 + q)
        for part in (s_hi, s_lo):
            assert _fp16_exact(part)
            assert _fp16_exact(-(1024.0 + c) * part)
            assert np.all(np.abs((1024.0 + q.max()) * part) <= 65504.0)  # no overflow inside the FMA
            res = (1024.0 + q[None, :]) * part[:, None] - (1024.0 + c) * part[:, None]
            assert np.all(res == (q[None, :] - c) * part[:, None])
            assert _fp16_exact(res)


def test_wide_affine_range_bound_is_needed():
    """The kernel accepts 2^-17 <= |s| <= 32: 32 is a power-of-two bound below the point
    where the FMA's product (1024 + 255) * s_hi leaves fp16 (65504 / 1279 = 51.2; the
    bf16 scale 52 is past it), and just below 2^-17 the low part's products fall below
    fp16's resolution."""
    assert (1024.0 + 255) * 32.0 <= 65504.0 < (1024.0 + 255) * 52.0
    tiny = 2.0 ** -18 * (1 + 1 / 128)  # bf16-exact; its low part is 2^-25
    s_hi = np.array([tiny], np.float32).view(np.uint32) & np.uint32(0xFFF00000)
    s_lo = tiny - s_hi.view(np.float32).astype(np.float64)[0]
    assert s_lo != 0 and not _fp16_exact(np.array([s_lo * 3]))


def test_bias_column_split_carries_22_bits():
    """The bias MMA's weight column holds C = b + c*s as C_hi = fp16(C) and
    C_lo = fp16((C - C_hi) * 2^11); C_hi + C_lo / 2^11 is within 2^-22 |C| of C for
    |C| >= 2^-14 (both parts normal) and within 2^-36 below (checked on a dense sample of
    f32 values over fp16's range), and each product with a token code sum |S| <= 2032 (or
    S / 2^11) is exact in f32 (11 x 11 significant bits)."""
    rng = np.random.default_rng(0)
    mags = np.exp2(rng.uniform(-30, np.log2(65504.0), 200000))
    C = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32).astype(np.float64)
    C_hi = C.astype(np.float16).astype(np.float64)
    rem = C - C_hi
    assert np.all(rem.astype(np.float32).astype(np.float64) == rem)       # C - C_hi exact in f32
    C_lo = (rem * 2048.0).astype(np.float16).astype(np.float64)
    err = np.abs(C_hi + C_lo / 2048.0 - C)
    normal = np.abs(C) >= 2.0 ** -14
    assert np.all(err[normal] <= 2.0 ** -22 * np.abs(C[normal]))
    assert np.all(err[~normal] <= 2.0 ** -36)
    S = np.arange(-2032, 2033, dtype=np.float64)
    for part in (C_hi[:2000], C_lo[:2000]):
        for scale in (1.0, 2.0 ** -11):
            prod = part[:, None] * (S[None, :] * scale)
            assert np.all(prod.astype(np.float32).astype(np.float64) == prod)


def test_q4_k_weight_product_is_exact_in_f32():
    """Q4_K on the GPU forms each weight as fma(d*sc, q, -dmin*m): d*sc (fp16 times a 6-bit
    scale) and d*sc*q (times a 4-bit code) are exact in f32 for every finite fp16 d, so the
    single rounding of the fused form is the page's d1*q - m1 with d1 = d*sc (whose product
    is exact), and dmin*m is exact likewise."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    d = bits.view(np.float16).astype(np.float64)
    d = d[np.isfinite(d)]
    sc = np.arange(64, dtype=np.float64)
    d1 = d[:, None] * sc[None, :]
    assert np.all(d1.astype(np.float32).astype(np.float64) == d1)
    for q in (13.0, 15.0):  # the codes with the most significant bits
        p = d1 * q
        assert np.all(p.astype(np.float32).astype(np.float64) == p)

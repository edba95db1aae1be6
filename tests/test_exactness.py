"""Host-side check of the arithmetic the tensor-core path relies on (no GPU): the weight
operand of the tcgen05 GEMM holds each Q4_0 weight d*(q-8) as two fp16 values
d_hi*(q-8) + d_lo*(q-8), d_hi = d with its three lowest significand bits cleared, and each
affine weight as s*(q-8) with the bf16 group scale s. Both are formed in the kernel by one
fused multiply-add (8 + q/2)*(2d) - 24d. This test checks, for every finite fp16 scale
within the documented range and every code, that the split is exact, that each product and
the fused form's addend are representable in fp16 (so a single rounding returns the exact
value), and that the range bound is tight."""
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

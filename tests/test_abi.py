"""Host-side checks of the C-ABI library (no GPU): it loads, exports every entry point
include/w4a8.h declares, sizes workspaces, and rejects bad arguments with the status
codes the header documents before touching the device."""
import ctypes
import os
import re

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import block_quantized_w4a8_b200 as w4a8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a8.h")


@pytest.fixture(scope="module")
def lib():
    from block_quantized_w4a8_b200 import build
    build.build()
    return w4a8.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a8_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["w4a8_pack_q4_0", "w4a8_quant_act_q8_0", "w4a8_gemm", "w4a8_gemm_affine",
                     "w4a8_pack_affine", "w4a8_workspace_bytes"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(w4a8.EXPORTS) >= set(declared_functions())


def test_status_strings(lib):
    for code, name in w4a8.STATUS_NAMES.items():
        assert w4a8.w4a8_status_string(code) == name


def _align(v):
    return (v + 255) // 256 * 256


@pytest.mark.parametrize("M,N,K,group", [(1, 4096, 4096, 0), (64, 1536, 384, 0), (1024, 4096, 4096, 0),
                                         (1024, 4096, 4096, 64), (1024, 4096, 4096, 128), (300, 333, 800, 0),
                                         (300, 333, 800, 32), (20, 64, 256, 32), (4096, 4096, 14336, 0),
                                         (256, 4096, 14336, 0), (3, 5, 8192, 0), (100, 333, 8192, 64)])
def test_workspace_bytes(lib, M, N, K, group):
    B = K // 32
    gemv = _align(M * K) + _align(M * B * 4) + _align(M * B * 4)
    tt = 16 if M <= 16 else (32 if M <= 32 else (64 if M <= 64 else 128))
    ntok = -(-M // tt)
    if tt == 128:  # 128-token tiles go to CTA pairs: an even count
        ntok += ntok % 2
    rows = ntok * tt
    tc = _align(rows * B * 64) + _align(rows * B * 4) + (_align(rows * (K // group) * 4) if group else 0)
    if group and tt == 128:  # affine on CTA pairs: 16 bytes of code sums per token and block
        tc += _align(rows * B * 16)
    # split of K: at least one split per 128 quant blocks (the accumulation chain bound),
    # more when the output tiles do not fill the SMs (148 without a GPU): partial outputs of
    # M*N f32 per split, at least 16 quant blocks per split
    tiles = -(-N // 128) * ntok
    kmin = -(-B // 128)
    ks = kmin
    if (M * N) % 4 == 0 and tiles < 148:
        ks = max(kmin, min(148 // tiles, B // 16))
    if ks > 1:
        tc += _align(ks * M * N * 4)
    assert w4a8.w4a8_workspace_bytes(M, N, K, group) == max(gemv, tc)


@pytest.mark.parametrize("args", [(0, 16, 32, 0), (16, 16, 33, 0), (16, 16, 64, 16), (16, 16, 96, 64),
                                  (-1, 16, 32, 0), (16, (1 << 20) + 1, 32, 0)])
def test_workspace_bytes_rejects(lib, args):
    assert w4a8.w4a8_workspace_bytes(*args) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below fails its checks first


def _gemm(lib, M, N, K, x=FAKE, dt=0, qs=FAKE, d=FAKE, y=FAKE, ws=FAKE, wsb=1 << 40, path=0):
    P = ctypes.c_void_p
    return lib.w4a8_gemm_ex(M, N, K, P(x), dt, P(qs), P(d), P(y), P(ws), wsb, path, P(0))


def test_gemm_argument_errors(lib):
    assert _gemm(lib, 0, 8, 32) == 1            # INVALID_ARG
    assert _gemm(lib, 8, 8, 48) == 1            # K % 32
    assert _gemm(lib, 8, 8, 32, x=0) == 1       # null
    assert _gemm(lib, 8, 8, 32, dt=7) == 2      # UNSUPPORTED dtype
    assert _gemm(lib, 8, 8, 32, path=9) == 2    # UNSUPPORTED path
    assert _gemm(lib, 8, 8, 32, y=FAKE + 4) == 6   # MISALIGNED
    assert _gemm(lib, 8, 8, 32, ws=0) == 3      # WORKSPACE missing
    assert _gemm(lib, 8, 8, 32, wsb=16) == 3    # WORKSPACE too small


def test_affine_argument_errors(lib):
    P = ctypes.c_void_p
    f = lib.w4a8_gemm_affine_ex
    base = dict(x=P(FAKE), q=P(FAKE), s=P(FAKE), b=P(FAKE), y=P(FAKE), ws=P(FAKE))

    def call(M=8, N=8, K=128, group=64, b=base["b"], dt=0):
        return f(M, N, K, group, base["x"], dt, base["q"], base["s"], b, base["y"], base["ws"], 1 << 40, 0, P(0))

    assert call(group=16) == 2      # only 32, 64 and 128 (the guard of meTile PR #29: bit width / group checked)
    assert call(group=256) == 2
    assert call(K=192, group=128) == 1
    assert call(b=P(0)) == 1
    assert lib.w4a8_pack_affine(P(FAKE), 0, 8, 128, 96, P(FAKE), P(FAKE), P(FAKE), P(0)) == 2


def test_pack_and_quant_argument_errors(lib):
    P = ctypes.c_void_p
    assert lib.w4a8_pack_q4_0(P(FAKE), 0, 8, 40, P(FAKE), P(FAKE), P(0)) == 1
    assert lib.w4a8_pack_q4_0(P(FAKE), 3, 8, 32, P(FAKE), P(FAKE), P(0)) == 2
    assert lib.w4a8_pack_q4_0(P(FAKE + 8), 0, 8, 32, P(FAKE), P(FAKE), P(0)) == 6
    assert lib.w4a8_quant_act_q8_0(P(FAKE), 0, 0, 32, P(FAKE), P(FAKE), P(0), P(0)) == 1
    assert lib.w4a8_quant_act_q8_0(P(FAKE), 0, 4, 32, P(FAKE), P(0), P(0), P(0)) == 1
    assert lib.w4a8_quant_act_q8_0(P(FAKE), 0, 4, 32, P(FAKE), P(FAKE), P(FAKE + 4), P(0)) == 6


def test_affine_nbit_argument_errors(lib):
    P = ctypes.c_void_p

    def gemm(bits=6, group=64, path=0, K=128):
        return lib.w4a8_gemm_affine_nbit(8, 8, K, group, bits, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), None,
                                         P(FAKE), P(FAKE), 1 << 40, path, P(0))

    def pack(bits=6, group=64, K=128, q=FAKE):
        return lib.w4a8_pack_affine_nbit(P(FAKE), 0, 8, K, group, bits, P(q), P(FAKE), P(FAKE), P(0))

    assert gemm(bits=5) == 2 and gemm(bits=16) == 2   # UNSUPPORTED code width
    assert gemm(group=16) == 2                         # UNSUPPORTED group
    assert gemm(K=96, group=64) == 1                   # K not a multiple of the group
    assert gemm(path=2) == 2                           # no tensor-core path for 6/8-bit codes
    assert gemm(bits=8, path=2) == 2
    # M > 64 but K/group = 4 (scale rows not a multiple of 16 bytes): no pair kernel
    assert lib.w4a8_gemm_affine_nbit(200, 8, 256, 64, 8, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), None,
                                     P(FAKE), P(FAKE), 1 << 40, 2, P(0)) == 2
    assert pack(bits=7) == 2 and pack(group=256) == 2
    assert pack(K=96) == 1 and pack(q=0) == 1
    assert pack(q=FAKE + 8) == 6                       # MISALIGNED
    e = w4a8.Epilogue()
    e.bias, e.bias_dtype, e.out_dtype = FAKE, 0, 5     # unknown output type
    assert lib.w4a8_gemm_affine_nbit(8, 8, 128, 64, 8, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), ctypes.byref(e),
                                     P(FAKE), P(FAKE), 1 << 40, 0, P(0)) == 2
    e.out_dtype, e.bias = 0, FAKE + 2                   # f32 bias not 4-byte aligned
    assert lib.w4a8_gemm_affine_nbit(8, 8, 128, 64, 6, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), ctypes.byref(e),
                                     P(FAKE), P(FAKE), 1 << 40, 0, P(0)) == 6
    assert lib.w4a8_gemm_affine_nbit(8, 8, 128, 64, 8, P(FAKE), 0, P(FAKE), P(FAKE), P(FAKE), None,
                                     P(FAKE), P(FAKE), 16, 0, P(0)) == 3   # workspace too small


def test_q4_k_argument_errors(lib):
    P = ctypes.c_void_p
    f, b = lib.w4a8_gemv_q4_k, lib.w4a8_gemv_q4_k_backward
    assert f(1, 8, 300, P(FAKE), P(FAKE), P(FAKE), P(0)) == 1      # K not a multiple of 256
    assert f(0, 8, 256, P(FAKE), P(FAKE), P(FAKE), P(0)) == 1
    assert f(1, 8, 256, P(0), P(FAKE), P(FAKE), P(0)) == 1
    assert f(1, 8, 256, P(FAKE + 4), P(FAKE), P(FAKE), P(0)) == 6  # MISALIGNED
    assert b(1, 8, 256, P(FAKE), P(FAKE), P(FAKE + 8), P(FAKE), 1 << 20, P(0)) == 6
    assert b(1, 4096, 4096, P(FAKE), P(FAKE), P(FAKE), P(0), 0, P(0)) == 3  # WORKSPACE missing
    assert lib.w4a8_q4_k_backward_workspace_bytes(1, 4096, 4000) == 0
    assert lib.w4a8_q4_k_backward_workspace_bytes(1, 8, 256) == 16      # one row range: no partials


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (2, 4096, 4096), (1, 14336, 4096), (1, 4096, 14336),
                                   (5, 100000, 256), (1, 64, 512), (3, 20, 1024)])
def test_q4_k_backward_workspace(lib, M, N, K):
    """Row ranges of the Q4_K backward (148 SMs without a GPU): about one CTA per SM over
    the K/256 super-block columns, at least 16 rows per range, at most 512 rows per range
    (the bound on a lane's chain of sums); partial sums of min(M, 2) tokens per range."""
    nb = K // 256
    R = min(-(-148 // nb), -(-N // 16))
    R = max(R, -(-N // 512), 1)
    want = R * min(M, 2) * K * 4 if R > 1 else 16
    assert lib.w4a8_q4_k_backward_workspace_bytes(M, N, K) == want


def test_checked_build_exports_the_same_boundary():
    """The checked variant (-DW4A8_CHECKED: device-side checks of each copy's alignment,
    reported as W4A8_ERR_CHECK) builds and exports every declared entry point."""
    from block_quantized_w4a8_b200 import build
    path = build.build(checked=True)
    chk = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(chk, name), name
    chk.w4a8_status_string.restype = ctypes.c_char_p
    assert chk.w4a8_status_string(8) == b"W4A8_ERR_CHECK"


@pytest.mark.parametrize("M,N,K,group,path,want", [
    (1, 4096, 4096, 0, 0, "gemv"),            # decode
    (2, 14336, 4096, 0, 0, "gemv"),           # K x N = 4096 x 14336: the GEMV at M = 2
    (2, 4096, 14336, 0, 0, "gemm_i8"),        # K x N = 14336 x 4096: the long rows favour the int8 kernel
    (3, 4096, 14336, 0, 0, "gemm_i8"),        # large weights: the int8 kernel from M = 3
    (3, 4096, 4096, 0, 0, "gemv"),            # small weights: the GEMV up to M = 4
    (4, 2048, 8192, 0, 0, "gemv"),
    (5, 4096, 4096, 0, 0, "gemm_i8"),
    (64, 4096, 4096, 0, 0, "gemm_i8"),
    (65, 4096, 4096, 0, 0, "gemm_pair"),      # 128-token tiles on CTA pairs
    (16, 1536, 384, 0, 0, "gemm_tc"),         # K not a multiple of 256: no int8 kernel
    (8, 1536, 384, 0, 0, "gemv"),
    (200, 333, 800, 0, 0, "gemm_tc"),         # K/32 = 25 scales per row: no TMA pitch for pairs
    (1, 4096, 4096, 0, 2, "gemm_i8"),         # forced tensor path
    (300, 4096, 4096, 0, 1, "gemv"),          # forced GEMV
    (8, 4096, 4096, 64, 0, "gemv"),           # affine: the GEMV up to M = 8
    (9, 4096, 4096, 64, 0, "gemm_tc"),
    (1024, 4096, 4096, 128, 0, "gemm_pair"),
])
def test_gemm_path_rule(lib, M, N, K, group, path, want):
    """The dispatch (host logic) at the measured crossovers and the format limits."""
    assert w4a8.w4a8_gemm_path(M, N, K, group, path) == want


shapes = st.tuples(st.integers(1, 5000), st.integers(1, 20000), st.integers(1, 600).map(lambda b: 32 * b),
                   st.sampled_from([0, 32, 64, 128]))


@settings(max_examples=400, deadline=None)
@given(shape=shapes)
def test_gemm_path_properties(lib, shape):
    """Over random valid shapes: AUTO takes one of the four kernel families; the int8
    kernel only for Q4_0 with K a multiple of 256 and M <= 64, the CTA pairs only above 64
    tokens; a forced GEMV is always the GEMV and a forced tensor path never is; AUTO
    follows the measured crossover; and the workspace size is defined."""
    M, N, K, group = shape
    if group and K % group:
        assert lib.w4a8_gemm_path(M, N, K, group, 0) == 0
        assert lib.w4a8_workspace_bytes(M, N, K, group) == 0
        return
    auto = lib.w4a8_gemm_path(M, N, K, group, 0)
    assert auto in (1, 2, 3, 4)
    assert lib.w4a8_gemm_path(M, N, K, group, 1) == 1
    assert lib.w4a8_gemm_path(M, N, K, group, 2) in (2, 3, 4)
    i8 = group == 0 and K % 256 == 0 and M <= 64
    if auto == 2 or lib.w4a8_gemm_path(M, N, K, group, 2) == 2:
        assert i8
    if auto == 4:
        assert M > 64
    small = N * K <= 1 << 25
    want_gemv = (M == 1 or (M == 2 and (K <= 8192 or small)) or (M <= 4 and small)) if i8 else M <= 8
    assert (auto == 1) == want_gemv, (M, N, K, group, auto)
    assert lib.w4a8_workspace_bytes(M, N, K, group) > 0


@settings(max_examples=200, deadline=None)
@given(shape=shapes)
def test_gemm_path_never_returns_to_the_gemv_as_m_grows(lib, shape):
    """Once AUTO takes a tensor-core kernel at some M, it does so at every larger M."""
    _, N, K, group = shape
    if group and K % group:
        return
    seen_tensor = False
    for M in list(range(1, 70)) + [128, 256, 1024]:
        auto = lib.w4a8_gemm_path(M, N, K, group, 0)
        if seen_tensor:
            assert auto != 1, (M, N, K, group)
        seen_tensor = seen_tensor or auto != 1


def test_gemm_path_rejects(lib):
    for args in [(0, 8, 32, 0, 0), (8, 8, 48, 0, 0), (8, 8, 128, 16, 0), (8, 8, 96, 64, 0), (8, 8, 32, 0, 7)]:
        assert lib.w4a8_gemm_path(*args) == 0


def test_selftest_hook_argument_errors(lib):
    """The failure-path self-test rejects its arguments before touching the device."""
    P = ctypes.c_void_p
    out = ctypes.c_uint(0)
    f = lib.w4a8_selftest_bounded_wait
    assert f(ctypes.c_ulonglong(100000), None, P(0)) == 1          # outcome NULL
    assert f(ctypes.c_ulonglong(0), ctypes.byref(out), P(0)) == 1  # limit below 1 us
    assert f(ctypes.c_ulonglong(2 * 10 ** 9), ctypes.byref(out), P(0)) == 1  # above 1 s


def test_status_string_of_check(lib):
    assert w4a8.w4a8_status_string(8) == "W4A8_ERR_CHECK"

"""Python binding of libw4a8, the block-quantized W4A8 matmul for NVIDIA B200 (sm_100a).

Argument marshalling only: every function here forwards torch CUDA tensors (their
device pointers and sizes) and the current CUDA stream to the C ABI declared in
``include/w4a8.h`` under the same name; all computation runs in the library's CUDA
kernels. PyTorch provides device memory and streams, nothing else. The library is
built in-tree (``block_quantized_w4a8_b200/libw4a8.so``); if it is missing or cannot be
loaded, every call raises -- there is no fallback.

The ``pack_q4_0`` / ``pack_affine`` / ``gemm`` / ``gemm_affine`` helpers at the bottom
allocate the outputs and the workspace with torch and then call the same entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# W4A8_LIB=checked selects the checked variant (device-side checks, W4A8_ERR_CHECK), built
# beside it; the default is the production library.
LIB_PATH = os.path.join(_HERE, "libw4a8_checked.so" if os.environ.get("W4A8_LIB") == "checked" else "libw4a8.so")

W4A8_OK = 0
STATUS_NAMES = {0: "W4A8_OK", 1: "W4A8_ERR_INVALID_ARG", 2: "W4A8_ERR_UNSUPPORTED", 3: "W4A8_ERR_WORKSPACE",
                4: "W4A8_ERR_CUDA", 5: "W4A8_ERR_DEVICE_TIMEOUT", 6: "W4A8_ERR_MISALIGNED", 7: "W4A8_ERR_RANGE",
                8: "W4A8_ERR_CHECK"}
W4A8_F32, W4A8_BF16 = 0, 1
PATH_AUTO, PATH_GEMV, PATH_GEMM = 0, 1, 2

EXPORTS = ["w4a8_pack_q4_0", "w4a8_quant_act_q8_0", "w4a8_workspace_bytes", "w4a8_gemm", "w4a8_gemm_ex",
           "w4a8_pack_affine", "w4a8_gemm_affine", "w4a8_gemm_affine_ex", "w4a8_gemm_epi", "w4a8_gemm_affine_epi",
           "w4a8_pack_affine_nbit", "w4a8_gemm_affine_nbit", "w4a8_gemv_q4_k", "w4a8_gemv_q4_k_backward",
           "w4a8_q4_k_backward_workspace_bytes", "w4a8_prepare_act",
           "w4a8_gemm_prepared", "w4a8_gemm_affine_prepared", "w4a8_gemm_noalloc", "w4a8_last_device_error",
           "w4a8_last_cuda_error_string", "w4a8_status_string", "w4a8_selftest_bounded_wait",
           "w4a8_gemm_path"]
KERNEL_NAMES = {1: "gemv", 2: "gemm_i8", 3: "gemm_tc", 4: "gemm_pair"}


class W4A8Error(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        msg = f"{fn} failed: {STATUS_NAMES.get(status, status)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))
        self.status = status


class Epilogue(ctypes.Structure):
    """w4a8_epilogue: bias (N values or NULL), its element type, the element type of y."""
    _fields_ = [("bias", ctypes.c_void_p), ("bias_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int)]


_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_EPI = ctypes.POINTER(Epilogue)
# (result type, argument types) of every entry point, in the order include/w4a8.h declares
# the arguments.
SIGNATURES = {
    "w4a8_pack_q4_0": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "w4a8_quant_act_q8_0": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
    "w4a8_workspace_bytes": (_Z, [_I, _I, _I, _I]),
    "w4a8_gemm": (_I, [_I, _I, _I, _P, _I, _P, _P, _P, _P, _Z, _P]),
    "w4a8_gemm_ex": (_I, [_I, _I, _I, _P, _I, _P, _P, _P, _P, _Z, _I, _P]),
    "w4a8_pack_affine": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P]),
    "w4a8_gemm_affine": (_I, [_I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "w4a8_gemm_affine_ex": (_I, [_I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _Z, _I, _P]),
    "w4a8_gemm_epi": (_I, [_I, _I, _I, _P, _I, _P, _P, _EPI, _P, _P, _Z, _I, _P]),
    "w4a8_gemm_affine_epi": (_I, [_I, _I, _I, _I, _P, _I, _P, _P, _P, _EPI, _P, _P, _Z, _I, _P]),
    "w4a8_pack_affine_nbit": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "w4a8_gemm_affine_nbit": (_I, [_I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _EPI, _P, _P, _Z, _I, _P]),
    "w4a8_gemv_q4_k": (_I, [_I, _I, _I, _P, _P, _P, _P]),
    "w4a8_gemv_q4_k_backward": (_I, [_I, _I, _I, _P, _P, _P, _P, _Z, _P]),
    "w4a8_q4_k_backward_workspace_bytes": (_Z, [_I, _I, _I]),
    "w4a8_prepare_act": (_I, [_I, _I, _I, _P, _I, _P, _Z, _I, _P]),
    "w4a8_gemm_prepared": (_I, [_I, _I, _I, _P, _P, _P, _P, _Z, _I, _P]),
    "w4a8_gemm_affine_prepared": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _I, _P]),
    "w4a8_gemm_noalloc": (_I, [_I, _I, _I, _P, _I, _P, _P, _P, _P]),
    "w4a8_last_device_error": (_I, []),
    "w4a8_selftest_bounded_wait": (_I, [ctypes.c_ulonglong, _P, _P]),
    "w4a8_gemm_path": (_I, [_I, _I, _I, _I, _I]),
    "w4a8_status_string": (ctypes.c_char_p, [_I]),
    "w4a8_last_cuda_error_string": (ctypes.c_char_p, []),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libw4a8.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libw4a8 is not built ({path} missing); run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


# ------------------------------------------------------------------ argument checks
# The C ABI takes bare pointers, so the kernels would read or write past a tensor that is
# smaller than the layout its call implies, or reach into another GPU's memory. Every
# pointer argument is therefore checked here against the bytes its layout needs and the
# device of the call's first tensor, which must be the thread's current CUDA device (the
# library launches there). A need of 0 defers to the library (a shape or mode it rejects).
def _device(t: torch.Tensor) -> int:
    """Device index of the call: that of `t`, which must be the current CUDA device."""
    if not t.is_cuda:
        raise ValueError("libw4a8 takes device tensors")
    dev = t.get_device()
    cur = torch.cuda.current_device()
    if dev != cur:
        raise ValueError(f"libw4a8: tensors on cuda:{dev} while cuda:{cur} is the current device")
    return dev


def _ptr(t: torch.Tensor | None, dev: int, need: int = 0, name: str = "tensor"):
    if t is None:
        return None
    if t.get_device() != dev:
        raise ValueError(f"libw4a8: {name} is not on the call's device")
    if not t.is_contiguous():
        raise ValueError(f"libw4a8 takes contiguous tensors ({name})")
    if t.nbytes < need:
        raise ValueError(f"libw4a8: {name} holds {t.nbytes} bytes; this call uses {need}")
    return ctypes.c_void_p(t.data_ptr())


def _valid_group(group: int) -> bool:
    return group in (32, 64, 128)


def _q4_0_bytes(N: int, K: int):
    """Q4_0 weights: packed codes N x K/2 bytes, fp16 scales N x K/32."""
    return N * (K // 2), N * (K // 32) * 2


def _affine_bytes(N: int, K: int, group: int, bits: int = 4):
    """Affine weights: codes N x K*bits/8 bytes, bf16 scale and bias N x K/group each."""
    codes = N * (K * bits // 8) if bits in (4, 6, 8) else 0
    return codes, (N * (K // group) * 2 if _valid_group(group) else 0)


def _q4_k_bytes(N: int, K: int) -> int:
    """Q4_K weights: N rows of K/256 super-blocks of 144 bytes."""
    return N * (K // 256) * 144


def _epilogue(bias: torch.Tensor | None, y: torch.Tensor, N: int, dev: int) -> Epilogue:
    e = Epilogue()
    p = _ptr(bias, dev, N * bias.element_size(), "bias") if bias is not None else None
    e.bias = p.value if p is not None else None
    e.bias_dtype = _dtype(bias) if bias is not None else W4A8_F32
    out_dtype = y.dtype
    e.out_dtype = W4A8_BF16 if out_dtype == torch.bfloat16 else (W4A8_F32 if out_dtype == torch.float32 else 99)
    return e


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return W4A8_F32
    if t.dtype == torch.bfloat16:
        return W4A8_BF16
    return 99  # rejected by the library as W4A8_ERR_UNSUPPORTED


def _check(fn: str, status: int) -> None:
    if status != W4A8_OK:
        detail = load_library().w4a8_last_cuda_error_string().decode() if status == 4 else ""
        raise W4A8Error(fn, status, detail)


# ------------------------------------------------------------------ C ABI, one to one
def w4a8_pack_q4_0(w: torch.Tensor, qs: torch.Tensor, d: torch.Tensor, stream=None) -> None:
    N, K = w.shape
    dev = _device(w)
    nq, nd = _q4_0_bytes(N, K)
    _check("w4a8_pack_q4_0", load_library().w4a8_pack_q4_0(_ptr(w, dev), _dtype(w), N, K, _ptr(qs, dev, nq, "qs"),
                                                           _ptr(d, dev, nd, "d"), _stream(stream)))


def w4a8_quant_act_q8_0(x: torch.Tensor, qx: torch.Tensor, dx: torch.Tensor, sx: torch.Tensor | None = None,
                        stream=None) -> None:
    M, K = x.shape
    dev = _device(x)
    nb = M * (K // 32) * 4
    _check("w4a8_quant_act_q8_0",
           load_library().w4a8_quant_act_q8_0(_ptr(x, dev), _dtype(x), M, K, _ptr(qx, dev, M * K, "qx"),
                                              _ptr(dx, dev, nb, "dx"), _ptr(sx, dev, nb, "sx"), _stream(stream)))


def w4a8_workspace_bytes(M: int, N: int, K: int, group: int = 0) -> int:
    return int(load_library().w4a8_workspace_bytes(M, N, K, group))


def w4a8_gemm_ex(x, qs, d, y, ws, path: int = PATH_AUTO, stream=None) -> None:
    M, K = x.shape
    N = qs.shape[0]
    dev = _device(x)
    nq, nd = _q4_0_bytes(N, K)
    _check("w4a8_gemm_ex", load_library().w4a8_gemm_ex(M, N, K, _ptr(x, dev), _dtype(x), _ptr(qs, dev, nq, "qs"),
                                                       _ptr(d, dev, nd, "d"), _ptr(y, dev, M * N * 4, "y"),
                                                       _ptr(ws, dev), ws.nbytes, path, _stream(stream)))


def w4a8_gemm(x, qs, d, y, ws, stream=None) -> None:
    M, K = x.shape
    N = qs.shape[0]
    dev = _device(x)
    nq, nd = _q4_0_bytes(N, K)
    _check("w4a8_gemm", load_library().w4a8_gemm(M, N, K, _ptr(x, dev), _dtype(x), _ptr(qs, dev, nq, "qs"),
                                                 _ptr(d, dev, nd, "d"), _ptr(y, dev, M * N * 4, "y"), _ptr(ws, dev),
                                                 ws.nbytes, _stream(stream)))


def w4a8_gemm_epi(x, qs, d, y, ws, bias=None, path: int = PATH_AUTO, stream=None) -> None:
    """y (f32 or bf16, M x N) = x . W^T + bias (bias: N values, f32 or bf16, or None)."""
    M, K = x.shape
    N = qs.shape[0]
    dev = _device(x)
    nq, nd = _q4_0_bytes(N, K)
    epi = _epilogue(bias, y, N, dev)
    _check("w4a8_gemm_epi", load_library().w4a8_gemm_epi(M, N, K, _ptr(x, dev), _dtype(x), _ptr(qs, dev, nq, "qs"),
                                                         _ptr(d, dev, nd, "d"), ctypes.byref(epi),
                                                         _ptr(y, dev, M * N * y.element_size(), "y"), _ptr(ws, dev),
                                                         ws.nbytes, path, _stream(stream)))


def w4a8_gemm_affine_epi(x, q, scale, bias_w, y, ws, group: int, bias=None, path: int = PATH_AUTO,
                         stream=None) -> None:
    """Affine weights (scale, bias_w from w4a8_pack_affine) with the output epilogue."""
    M, K = x.shape
    N = q.shape[0]
    dev = _device(x)
    nq, ns = _affine_bytes(N, K, group)
    epi = _epilogue(bias, y, N, dev)
    _check("w4a8_gemm_affine_epi",
           load_library().w4a8_gemm_affine_epi(M, N, K, group, _ptr(x, dev), _dtype(x), _ptr(q, dev, nq, "q"),
                                               _ptr(scale, dev, ns, "scale"), _ptr(bias_w, dev, ns, "bias_w"),
                                               ctypes.byref(epi), _ptr(y, dev, M * N * y.element_size(), "y"),
                                               _ptr(ws, dev), ws.nbytes, path, _stream(stream)))


def w4a8_pack_affine_nbit(w, group: int, bits: int, q, scale, bias, stream=None) -> None:
    N, K = w.shape
    dev = _device(w)
    nq, ns = _affine_bytes(N, K, group, bits)
    _check("w4a8_pack_affine_nbit", load_library().w4a8_pack_affine_nbit(_ptr(w, dev), _dtype(w), N, K, group, bits,
                                                                         _ptr(q, dev, nq, "q"),
                                                                         _ptr(scale, dev, ns, "scale"),
                                                                         _ptr(bias, dev, ns, "bias"),
                                                                         _stream(stream)))


def w4a8_gemm_affine_nbit(x, q, scale, bias_w, y, ws, group: int, bits: int, bias=None, path: int = PATH_AUTO,
                          stream=None) -> None:
    """Affine weights with 4-, 6- or 8-bit codes (from w4a8_pack_affine_nbit), with the
    output epilogue (y f32 or bf16; `bias` per column or None)."""
    M, K = x.shape
    N = q.shape[0]
    dev = _device(x)
    nq, ns = _affine_bytes(N, K, group, bits)
    epi = _epilogue(bias, y, N, dev)
    _check("w4a8_gemm_affine_nbit",
           load_library().w4a8_gemm_affine_nbit(M, N, K, group, bits, _ptr(x, dev), _dtype(x), _ptr(q, dev, nq, "q"),
                                                _ptr(scale, dev, ns, "scale"), _ptr(bias_w, dev, ns, "bias_w"),
                                                ctypes.byref(epi), _ptr(y, dev, M * N * y.element_size(), "y"),
                                                _ptr(ws, dev), ws.nbytes, path, _stream(stream)))


def w4a8_gemv_q4_k(x, w_q4k, y, stream=None) -> None:
    """y (M, N) f32 = x (M, K) f32 . W^T, W in Q4_K (uint8 (N, K/256*144))."""
    M, K = x.shape
    N = w_q4k.shape[0]
    dev = _device(x)
    _check("w4a8_gemv_q4_k", load_library().w4a8_gemv_q4_k(M, N, K, _ptr(x, dev), _ptr(w_q4k, dev, _q4_k_bytes(N, K),
                                                                                          "w_q4k"),
                                                           _ptr(y, dev, M * N * 4, "y"), _stream(stream)))


def w4a8_gemv_q4_k_backward(dy, w_q4k, dx, ws, stream=None) -> None:
    """dx (M, K) f32 = dy (M, N) f32 . W (the input gradient), W in Q4_K."""
    M, N = dy.shape
    K = dx.shape[1]
    dev = _device(dy)
    nbytes = ws.nbytes if ws is not None else 0
    _check("w4a8_gemv_q4_k_backward",
           load_library().w4a8_gemv_q4_k_backward(M, N, K, _ptr(dy, dev), _ptr(w_q4k, dev, _q4_k_bytes(N, K), "w_q4k"),
                                                  _ptr(dx, dev, M * K * 4, "dx"), _ptr(ws, dev), nbytes,
                                                  _stream(stream)))


def w4a8_q4_k_backward_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load_library().w4a8_q4_k_backward_workspace_bytes(M, N, K))


def gemv_q4_k(x, w_q4k, stream=None):
    y = torch.empty(x.shape[0], w_q4k.shape[0], dtype=torch.float32, device=x.device)
    w4a8_gemv_q4_k(x, w_q4k, y, stream)
    return y


def gemv_q4_k_backward(dy, w_q4k, K: int, ws=None, stream=None):
    M, N = dy.shape
    dx = torch.empty(M, K, dtype=torch.float32, device=dy.device)
    if ws is None:
        ws = torch.empty(max(16, w4a8_q4_k_backward_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dy.device)
    w4a8_gemv_q4_k_backward(dy, w_q4k, dx, ws, stream)
    return dx


def w4a8_pack_affine(w, group: int, q, scale, bias, stream=None) -> None:
    N, K = w.shape
    dev = _device(w)
    nq, ns = _affine_bytes(N, K, group)
    _check("w4a8_pack_affine", load_library().w4a8_pack_affine(_ptr(w, dev), _dtype(w), N, K, group,
                                                               _ptr(q, dev, nq, "q"), _ptr(scale, dev, ns, "scale"),
                                                               _ptr(bias, dev, ns, "bias"), _stream(stream)))


def w4a8_gemm_affine_ex(x, q, scale, bias, y, ws, group: int, path: int = PATH_AUTO, stream=None) -> None:
    M, K = x.shape
    N = q.shape[0]
    dev = _device(x)
    nq, ns = _affine_bytes(N, K, group)
    _check("w4a8_gemm_affine_ex",
           load_library().w4a8_gemm_affine_ex(M, N, K, group, _ptr(x, dev), _dtype(x), _ptr(q, dev, nq, "q"),
                                              _ptr(scale, dev, ns, "scale"), _ptr(bias, dev, ns, "bias"),
                                              _ptr(y, dev, M * N * 4, "y"), _ptr(ws, dev), ws.nbytes, path,
                                              _stream(stream)))


def w4a8_gemm_affine(x, q, scale, bias, y, ws, group: int, stream=None) -> None:
    M, K = x.shape
    N = q.shape[0]
    dev = _device(x)
    nq, ns = _affine_bytes(N, K, group)
    _check("w4a8_gemm_affine",
           load_library().w4a8_gemm_affine(M, N, K, group, _ptr(x, dev), _dtype(x), _ptr(q, dev, nq, "q"),
                                           _ptr(scale, dev, ns, "scale"), _ptr(bias, dev, ns, "bias"),
                                           _ptr(y, dev, M * N * 4, "y"), _ptr(ws, dev), ws.nbytes, _stream(stream)))


def w4a8_prepare_act(x, ws, group: int = 0, path: int = PATH_AUTO, stream=None) -> None:
    M, K = x.shape
    dev = _device(x)
    _check("w4a8_prepare_act", load_library().w4a8_prepare_act(M, K, group, _ptr(x, dev), _dtype(x), _ptr(ws, dev),
                                                               ws.nbytes, path, _stream(stream)))


def w4a8_gemm_prepared(M: int, K: int, qs, d, y, ws, path: int = PATH_AUTO, stream=None) -> None:
    N = qs.shape[0]
    dev = _device(qs)
    nq, nd = _q4_0_bytes(N, K)
    _check("w4a8_gemm_prepared", load_library().w4a8_gemm_prepared(M, N, K, _ptr(qs, dev, nq, "qs"),
                                                                   _ptr(d, dev, nd, "d"), _ptr(y, dev, M * N * 4, "y"),
                                                                   _ptr(ws, dev), ws.nbytes, path, _stream(stream)))


def w4a8_gemm_affine_prepared(M: int, K: int, group: int, q, scale, bias, y, ws, path: int = PATH_AUTO,
                              stream=None) -> None:
    N = q.shape[0]
    dev = _device(q)
    nq, ns = _affine_bytes(N, K, group)
    _check("w4a8_gemm_affine_prepared",
           load_library().w4a8_gemm_affine_prepared(M, N, K, group, _ptr(q, dev, nq, "q"),
                                                    _ptr(scale, dev, ns, "scale"), _ptr(bias, dev, ns, "bias"),
                                                    _ptr(y, dev, M * N * 4, "y"), _ptr(ws, dev), ws.nbytes, path,
                                                    _stream(stream)))


def w4a8_gemm_noalloc(x, qs, d, y, stream=None) -> None:
    """w4a8_gemm with the library's built-in scratch array instead of a caller workspace
    (for callers that may not allocate device memory). Calls must not overlap on the GPU."""
    M, K = x.shape
    N = qs.shape[0]
    dev = _device(x)
    nq, nd = _q4_0_bytes(N, K)
    _check("w4a8_gemm_noalloc", load_library().w4a8_gemm_noalloc(M, N, K, _ptr(x, dev), _dtype(x),
                                                                 _ptr(qs, dev, nq, "qs"), _ptr(d, dev, nd, "d"),
                                                                 _ptr(y, dev, M * N * 4, "y"), _stream(stream)))


def w4a8_last_device_error() -> int:
    return int(load_library().w4a8_last_device_error())


def w4a8_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """Runs the library's self-test of its bounded device waits (see the header) and
    returns the outcome bits (7 = the wait ran out, and the second warp stopped through the
    abort flag within 100 ms)."""
    out = ctypes.c_uint(0)
    _check("w4a8_selftest_bounded_wait",
           load_library().w4a8_selftest_bounded_wait(int(limit_ns), ctypes.byref(out), _stream(stream)))
    return int(out.value)


def w4a8_gemm_path(M: int, N: int, K: int, group: int = 0, path: int = 0) -> str:
    """The kernel family the matmul of this shape runs ("gemv", "gemm_i8", "gemm_tc",
    "gemm_pair"); raises ValueError for a shape the call would reject."""
    k = int(load_library().w4a8_gemm_path(M, N, K, group, path))
    if k not in KERNEL_NAMES:
        raise ValueError(f"no kernel for M={M} N={N} K={K} group={group} path={path}")
    return KERNEL_NAMES[k]


def w4a8_last_cuda_error_string() -> str:
    return load_library().w4a8_last_cuda_error_string().decode()


def w4a8_status_string(status: int) -> str:
    return load_library().w4a8_status_string(status).decode()


# ------------------------------------------------------------------ allocating helpers
def pack_q4_0(w: torch.Tensor, stream=None):
    N, K = w.shape
    qs = torch.empty(N, K // 2, dtype=torch.uint8, device=w.device)
    d = torch.empty(N, K // 32, dtype=torch.int16, device=w.device)
    w4a8_pack_q4_0(w, qs, d, stream)
    return qs, d


def quant_act_q8_0(x: torch.Tensor, stream=None):
    M, K = x.shape
    qx = torch.empty(M, K, dtype=torch.int8, device=x.device)
    dx = torch.empty(M, K // 32, dtype=torch.float32, device=x.device)
    sx = torch.empty(M, K // 32, dtype=torch.int32, device=x.device)
    w4a8_quant_act_q8_0(x, qx, dx, sx, stream)
    return qx, dx, sx


def pack_affine(w: torch.Tensor, group: int, stream=None):
    N, K = w.shape
    q = torch.empty(N, K // 8, dtype=torch.int32, device=w.device)
    s = torch.empty(N, K // group, dtype=torch.int16, device=w.device)
    b = torch.empty(N, K // group, dtype=torch.int16, device=w.device)
    w4a8_pack_affine(w, group, q, s, b, stream)
    return q, s, b


def pack_affine_nbit(w: torch.Tensor, group: int, bits: int, stream=None):
    """Codes as uint8 (N, K*bits/8) little-endian bit streams, scale and bias bf16 bits."""
    N, K = w.shape
    q = torch.empty(N, K * bits // 8, dtype=torch.uint8, device=w.device)
    s = torch.empty(N, K // group, dtype=torch.int16, device=w.device)
    b = torch.empty(N, K // group, dtype=torch.int16, device=w.device)
    w4a8_pack_affine_nbit(w, group, bits, q, s, b, stream)
    return q, s, b


def gemm_affine_nbit(x, q, s, b, group: int, bits: int, path: int = PATH_AUTO, ws=None, stream=None):
    M, K = x.shape
    N = q.shape[0]
    y = torch.empty(M, N, dtype=torch.float32, device=x.device)
    ws = workspace(M, N, K, group, x.device) if ws is None else ws
    w4a8_gemm_affine_nbit(x, q, s, b, y, ws, group, bits, path=path, stream=stream)
    return y


def workspace(M: int, N: int, K: int, group: int = 0, device="cuda") -> torch.Tensor:
    nbytes = w4a8_workspace_bytes(M, N, K, group)
    if nbytes == 0:
        raise W4A8Error("w4a8_workspace_bytes", 1)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def gemm(x, qs, d, path: int = PATH_AUTO, ws=None, stream=None):
    M, K = x.shape
    N = qs.shape[0]
    y = torch.empty(M, N, dtype=torch.float32, device=x.device)
    ws = workspace(M, N, K, 0, x.device) if ws is None else ws
    w4a8_gemm_ex(x, qs, d, y, ws, path, stream)
    return y


def gemm_affine(x, q, s, b, group: int, path: int = PATH_AUTO, ws=None, stream=None):
    M, K = x.shape
    N = q.shape[0]
    y = torch.empty(M, N, dtype=torch.float32, device=x.device)
    ws = workspace(M, N, K, group, x.device) if ws is None else ws
    w4a8_gemm_affine_ex(x, q, s, b, y, ws, group, path, stream)
    return y

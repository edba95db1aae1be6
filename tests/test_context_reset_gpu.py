"""Calls after a CUDA context reset: the library raises each kernel's shared-memory limit
once per context (the attribute does not survive cudaDeviceReset) and looks the no-alloc
scratch up again in the new context. A child process (so that the reset does not touch
this process's torch context) runs the resident GEMV (M = 1), the int8 kernel (M = 16) and
the CTA-pair kernel (M = 1024) on the same inputs, resets the device, runs them again in
the new context, and requires every call to succeed with bit-identical outputs."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

CHILD = textwrap.dedent(r"""
    import ctypes
    import numpy as np
    import block_quantized_w4a8_b200 as w4a8

    lib = w4a8.load_library()
    # the CUDA runtime the library itself is linked against (same instance, same contexts)
    rt_path = next(l.split()[-1] for l in open("/proc/self/maps") if "libcudart.so" in l)
    rt = ctypes.CDLL(rt_path)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    rt.cudaMalloc.argtypes = [ctypes.POINTER(P), Z]
    rt.cudaMemcpy.argtypes = [P, P, Z, I]
    lib.w4a8_pack_q4_0.argtypes = [P, I, I, I, P, P, P]
    lib.w4a8_gemm.argtypes = [I, I, I, P, I, P, P, P, P, Z, P]
    lib.w4a8_gemm_noalloc.argtypes = [I, I, I, P, I, P, P, P, P]
    lib.w4a8_workspace_bytes.argtypes = [I, I, I, I]
    lib.w4a8_workspace_bytes.restype = Z

    N = K = 4096
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xs = {M: rng.standard_normal((M, K)).astype(np.float32) for M in (1, 16, 1024)}

    def dmalloc(n):
        p = P()
        assert rt.cudaMalloc(ctypes.byref(p), n) == 0
        return p

    def run():
        out = {}
        dw = dmalloc(w.nbytes)
        assert rt.cudaMemcpy(dw, w.ctypes.data, w.nbytes, 1) == 0
        qs, d = dmalloc(N * K // 2), dmalloc(N * K // 32 * 2)
        assert lib.w4a8_pack_q4_0(dw, 0, N, K, qs, d, None) == 0
        for M, x in xs.items():
            dx, dy = dmalloc(x.nbytes), dmalloc(M * N * 4)
            nws = lib.w4a8_workspace_bytes(M, N, K, 0)
            ws = dmalloc(nws)
            assert rt.cudaMemcpy(dx, x.ctypes.data, x.nbytes, 1) == 0
            y = np.empty((M, N), np.float32)
            st = lib.w4a8_gemm(M, N, K, dx, 0, qs, d, dy, ws, nws, None)
            assert st == 0, (M, st)
            assert rt.cudaMemcpy(y.ctypes.data, dy, y.nbytes, 2) == 0
            out[("gemm", M)] = y.copy()
            if M <= 16:
                st = lib.w4a8_gemm_noalloc(M, N, K, dx, 0, qs, d, dy, None)
                assert st == 0, ("noalloc", M, st)
                assert rt.cudaMemcpy(y.ctypes.data, dy, y.nbytes, 2) == 0
                out[("noalloc", M)] = y.copy()
        assert rt.cudaDeviceSynchronize() == 0
        assert lib.w4a8_last_device_error() == 0
        return out

    first = run()
    assert rt.cudaDeviceReset() == 0
    second = run()
    for key, y in first.items():
        assert np.isfinite(y).all(), key
        assert np.array_equal(y.view(np.uint32), second[key].view(np.uint32)), key
    assert np.array_equal(first[("gemm", 1)], first[("noalloc", 1)])
    print("context reset ok")
""")


def test_calls_after_a_context_reset():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "context reset ok" in r.stdout

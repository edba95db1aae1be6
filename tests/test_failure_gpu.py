"""Failure detection on the GPU without a fault: a bounded device wait is made to run out
(a barrier that nothing arrives at, through the library's own wait code), the status word
reports it, the other warp stops through the abort flag, and the context stays usable for
the next call, whose result is checked against the oracle."""
import numpy as np
import pytest

import block_quantized_w4a8_b200 as w4a8
import oracle
from block_quantized_w4a8_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_next_call_succeeds():
    w4a8.load_library()
    assert w4a8.w4a8_last_device_error() == w4a8.W4A8_OK
    outcome = w4a8.w4a8_selftest_bounded_wait(100_000)  # 100 us limit
    assert outcome == 7, f"outcome bits {outcome:#x}"
    assert w4a8.w4a8_last_device_error() == 5          # W4A8_ERR_DEVICE_TIMEOUT
    assert w4a8.w4a8_last_device_error() == w4a8.W4A8_OK  # read and cleared
    # the next real call runs normally
    M, N, K = 5, 300, 2048
    x = inputs.randn((M, K), seed=91)
    w = inputs.randn((N, K), seed=92, std=0.02)
    qs, d = w4a8.pack_q4_0(w.cuda())
    for path in (w4a8.PATH_GEMV, w4a8.PATH_GEMM):
        y = w4a8.gemm(x.cuda(), qs, d, path=path).cpu().numpy().astype(np.float64)
        rqx, rdx, _ = oracle.quant_act_q8_0(x.numpy())
        rqs, rd = oracle.pack_q4_0(w.numpy())
        yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd)
        assert np.all(np.abs(y - yref) <= 1e-5 * T)
    assert w4a8.w4a8_last_device_error() == w4a8.W4A8_OK

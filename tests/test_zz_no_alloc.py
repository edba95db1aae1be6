"""w4a8_gemm_noalloc: the matmul for callers that may not allocate device memory (a host
that reserved all device memory up front, or an interface that passes only inputs and the
output). It takes its scratch from an array built into the library instead of a caller
workspace. Checked through the C ABI against w4a8_gemm on two calls in a row (the second
on other data, so whatever the first call left in the shared array must not leak into
it), within the tolerance of the other parity tests. Collected last on purpose."""
import numpy as np
import pytest
import torch

import block_quantized_w4a8_b200 as w4a8
import oracle
from block_quantized_w4a8_b200 import inputs

pytestmark = pytest.mark.gpu
TOL = 1e-5


# (4, 512, 8192): M*K too large for the GEMV to quantise x itself, so the activation goes
# through the scratch array's row-major Q8_0 region before the GEMV reads it.
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (4, 512, 8192), (200, 333, 800), (1024, 512, 4096)])
def test_noalloc_matches_workspace_entry_point(M, N, K):
    w4a8.load_library()
    for call in range(2):
        wl = inputs.Workload("noalloc", M=M, K=K, N=N, seed=10 * call + 1)
        x, w = inputs.make(wl)
        xd, wd = x.cuda(), w.cuda()
        qs, d = w4a8.pack_q4_0(wd)
        y_ref = w4a8.gemm(xd, qs, d)
        y = torch.full((M, N), float("nan"), device="cuda")
        w4a8.w4a8_gemm_noalloc(xd, qs, d, y)
        torch.cuda.synchronize()
        assert w4a8.w4a8_last_device_error() == 0  # no bounded wait ran out, no scale out of range
        rqx, rdx, _ = oracle.quant_act_q8_0(x.numpy())
        ms, ns = inputs.sample_indices(M, N, 2000, seed=call)
        _, T = oracle.gemm_q4_0_sampled(rqx, rdx, qs.cpu().numpy(), d.cpu().numpy().view(np.uint16), ms, ns)
        a = y.cpu().numpy().astype(np.float64)
        b = y_ref.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(a))
        # The built-in scratch may allow a smaller split of K than a full workspace, so the
        # two calls can round differently: compare both with the oracle's tolerance.
        yref, _ = oracle.gemm_q4_0_sampled(rqx, rdx, qs.cpu().numpy(), d.cpu().numpy().view(np.uint16), ms, ns)
        assert np.all(np.abs(a[ms, ns] - yref) <= TOL * T)
        assert np.all(np.abs(b[ms, ns] - yref) <= TOL * T)
        assert np.all(np.abs(a[ms, ns] - b[ms, ns]) <= 2 * TOL * T)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w4a8.load_library()
    M, N, K = 4096, 64, 8192   # workspace well above 16 MiB
    assert w4a8.w4a8_workspace_bytes(M, N, K, 0) > 16 << 20
    x = torch.zeros(M, K, device="cuda")
    qs = torch.zeros(N, K // 2, dtype=torch.uint8, device="cuda")
    d = torch.zeros(N, K // 32, dtype=torch.int16, device="cuda")
    y = torch.zeros(M, N, device="cuda")
    with pytest.raises(w4a8.W4A8Error) as e:
        w4a8.w4a8_gemm_noalloc(x, qs, d, y)
    assert e.value.status == 3  # W4A8_ERR_WORKSPACE

"""Failure detection without a GPU fault: a kernel's bounded wait on an
mbarrier that nothing arrives on runs out, the device status word records
it, vlaq_check reports VLAQ_ERR_TIMEOUT once and then clears, and the
context stays usable (a quantize + GEMM afterwards still matches the
oracle)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from gpu_helpers import REL_FRO_TOL, bits, gemm_error, gpu_linear_nvfp4, vq

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives():
    m = vq()
    m.vlaq_check()  # start from a clear status
    m.vlaq_selftest_wait_timeout()
    torch.cuda.synchronize()
    with pytest.raises(m.VlaqError) as ei:
        m.vlaq_check()
    assert ei.value.status == 6 and "bounded wait" in ei.value.message
    m.vlaq_check()  # read and cleared: OK now

    X, W = si.tiny_inputs(0)
    M, K = X.shape
    N = W.shape[0]
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    m.vlaq_quantize_weight_nvfp4(W.cuda(), N, K, 0, wq, ws, wg)
    m.vlaq_quantize_act_nvfp4(X.cuda(), M, K, None, 1e-6, 0, xq, xs, xg)
    Y = gpu_linear_nvfp4(xq, xs, xg, wq, ws, wg, M, N, K)
    cx, sx, gx = oracle.quantize_nvfp4(bits(X))
    cw, sw, gw = oracle.quantize_nvfp4(bits(W), per_tensor=True)
    Y64 = oracle.linear_f64(oracle.decode_nvfp4(cx, sx, gx, K), oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True))
    rel, mx = gemm_error(Y, Y64)
    assert rel < REL_FRO_TOL, (rel, mx)

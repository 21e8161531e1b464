"""vlaq_linear_nvfp4_noalloc: the NVFP4 linear for callers that cannot
allocate device memory (host callbacks, real-time control loops that must not
touch the allocator, embeddings whose own arena owns all device memory).

The entry point takes no workspace; its split-K scratch is a fixed array
inside the library.  These tests call it through the C ABI and compare it
with vlaq_linear_nvfp4 given a caller-allocated workspace, on two calls in a
row with different inputs (the second call must not see the first call's
scratch contents): both run the same kernel with the same split plan, so the
outputs must be identical bit for bit, and both are checked against the
oracle.  This file is named to be collected last, so a run that stops at the
first failure has run every other test before it."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from gpu_helpers import bits, check_gemm, residual_f64, vq

pytestmark = pytest.mark.gpu


def _case(m, M, N, K, seed, residual):
    X = si.projection_activations(K, M, seed)
    W = si.projection_weight(K, N, seed)
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    m.vlaq_quantize_weight_nvfp4(W.cuda(), N, K, 0, wq, ws, wg)
    m.vlaq_quantize_act_nvfp4(X.cuda(), M, K, None, 1e-6, 0, xq, xs, xg)
    R = si.residual(M, N, seed) if residual else None
    return (xq, xs, xg, wq, ws, wg, None if R is None else R.cuda()), (X, W, R)


def _oracle(host, K):
    X, W, R = host
    cx, sx, gx = oracle.quantize_nvfp4(bits(X))
    cw, sw, gw = oracle.quantize_nvfp4(bits(W), per_tensor=True)
    dx = oracle.decode_nvfp4(cx, sx, gx, K)
    dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    return oracle.linear_f64(dx, dw, None if R is None else bits(R)), dx, dw


def _both(m, dev, M, N, K):
    """(workspace path output, allocation-free output), bf16 bits."""
    xq, xs, xg, wq, ws, wg, R = dev
    Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, R, Y_ref, M, N, K, wsp, nb)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.vlaq_linear_nvfp4_noalloc(xq, xs, xg, wq, ws, wg, R, Y, M, N, K)
    torch.cuda.synchronize()
    m.vlaq_check()
    return Y_ref.cpu(), Y.cpu()


def _assert_same_bits(Y, Y_ref, what):
    a = Y.view(torch.int16).numpy()
    b = Y_ref.view(torch.int16).numpy()
    bad = np.argwhere(a != b)
    assert bad.size == 0, f"{what}: {len(bad)} outputs differ from the workspace path, first {bad[:4].tolist()}"


# M <= 2 with weights of at most 2^25 elements runs the few-row kernel (no
# scratch); M = 3..8 on these shapes runs split-K through the scratch array.
@pytest.mark.parametrize("M,N,K,residual", [(5, 512, 4096, False), (6, 4608, 3584, True), (8, 3584, 18944, True),
                                            (3, 3584, 3584, False), (1, 4608, 3584, True)])
def test_noalloc_matches_workspace_path_twice(M, N, K, residual):
    m = vq()
    if M > 2:
        assert m.vlaq_linear_workspace_bytes(M, N, K) > 0, "shape must take the split-K path"
    for call, seed in enumerate((101, 202)):
        dev, host = _case(m, M, N, K, seed, residual)
        Y_ref, Y = _both(m, dev, M, N, K)
        _assert_same_bits(Y, Y_ref, f"call {call}")
        Y64, dx, dw = _oracle(host, K)
        check_gemm(Y.float().numpy(), Y64, dx, dw, K, residual_f64(host[2]), f"noalloc call {call} {M}x{N}x{K}")


def test_noalloc_direct_path_without_split():
    """A prefill-sized shape needs no scratch and must still work."""
    m = vq()
    M, N, K = 1024, 2560, 512
    assert m.vlaq_linear_workspace_bytes(M, N, K) == 0
    dev, host = _case(m, M, N, K, 303, False)
    Y_ref, Y = _both(m, dev, M, N, K)
    _assert_same_bits(Y, Y_ref, "direct path")
    Y64, dx, dw = _oracle(host, K)
    check_gemm(Y.float().numpy(), Y64, dx, dw, K, None, "noalloc direct")


def test_noalloc_refuses_shapes_beyond_the_static_scratch():
    m = vq()
    M, N, K = 128, 2048, 8192
    need = m.vlaq_linear_workspace_bytes(M, N, K)
    assert need > 4 * 1024 * 1024, f"this split-K plan needs {need} bytes"
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.VlaqError) as ei:
        m.vlaq_linear_nvfp4_noalloc(xq, xs, xg, wq, ws, wg, None, Y, M, N, K)
    assert ei.value.status == 7 and "static scratch" in ei.value.message


def test_noalloc_after_reported_timeout():
    """vlaq_check clears the static scratch when it reports a timeout (a GEMM
    that gave up could have left split-K tile counters set).  The timeout is
    made on the host's terms: a self-test kernel's bounded wait on an
    mbarrier that nothing arrives on runs out (no fault, no hang).  The
    split-K call before and after must both match the workspace path."""
    m = vq()
    M, N, K = 4, 4608, 3584
    assert m.vlaq_linear_workspace_bytes(M, N, K) > 0
    dev, host = _case(m, M, N, K, 404, True)
    Y_ref, Y = _both(m, dev, M, N, K)
    _assert_same_bits(Y, Y_ref, "before the timeout")
    m.vlaq_selftest_wait_timeout()
    torch.cuda.synchronize()
    with pytest.raises(m.VlaqError) as ei:
        m.vlaq_check()
    assert ei.value.status == 6
    m.vlaq_check()  # read and cleared
    Y_ref2, Y2 = _both(m, dev, M, N, K)
    _assert_same_bits(Y2, Y_ref2, "after the timeout")
    _assert_same_bits(Y2, Y, "after vs before the timeout")
    Y64, dx, dw = _oracle(host, K)
    check_gemm(Y2.float().numpy(), Y64, dx, dw, K, residual_f64(host[2]), "noalloc after timeout")

"""vlaq_linear_nvfp4_noalloc: the NVFP4 linear for callers that cannot
allocate device memory (host callbacks, real-time control loops that must not
touch the allocator, embeddings whose own arena owns all device memory).

The entry point takes no workspace; its split-K scratch is a fixed array
inside the library.  These tests call it through the C ABI and compare it
with vlaq_linear_nvfp4 given a caller-allocated workspace, on two calls in a
row with different inputs (the second call must not see the first call's
scratch contents).  This file is named to be collected last, so a run that
stops at the first failure has run every other test before it."""
import numpy as np
import pytest
import torch

import synthetic_inputs as si
from gpu_helpers import REL_FRO_TOL, gemm_error, vq

pytestmark = pytest.mark.gpu


def _case(m, M, N, K, seed, residual):
    X = si.projection_activations(K, M, seed).cuda()
    W = si.projection_weight(K, N, seed).cuda()
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    m.vlaq_quantize_weight_nvfp4(W, N, K, 0, wq, ws, wg)
    m.vlaq_quantize_act_nvfp4(X, M, K, None, 1e-6, 0, xq, xs, xg)
    R = si.residual(M, N, seed).cuda() if residual else None
    return xq, xs, xg, wq, ws, wg, R


@pytest.mark.parametrize("M,N,K,residual", [(5, 512, 4096, False), (6, 4608, 3584, True), (8, 3584, 18944, True),
                                            (1, 4608, 3584, True)])
def test_noalloc_matches_workspace_path_twice(M, N, K, residual):
    m = vq()
    if M > 4:  # M <= 4 runs the few-row kernel, which needs no scratch
        assert m.vlaq_linear_workspace_bytes(M, N, K) > 0, "shape must take the split-K path"
    for call, seed in enumerate((101, 202)):
        xq, xs, xg, wq, ws, wg, R = _case(m, M, N, K, seed, residual)
        Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        wsp, nb = m.alloc_workspace(M, N, K)
        m.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, R, Y_ref, M, N, K, wsp, nb)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        m.vlaq_linear_nvfp4_noalloc(xq, xs, xg, wq, ws, wg, R, Y, M, N, K)
        torch.cuda.synchronize()
        m.vlaq_check()
        a = Y.float().cpu().numpy()
        b = Y_ref.float().cpu().numpy()
        assert np.isfinite(a).all(), f"call {call}: non-finite output"
        rel, mx = gemm_error(a, b.astype(np.float64))
        assert rel < REL_FRO_TOL, (call, rel, mx)


def test_noalloc_direct_path_without_split():
    """A prefill-sized shape needs no scratch and must still work."""
    m = vq()
    M, N, K = 1024, 2560, 512
    assert m.vlaq_linear_workspace_bytes(M, N, K) == 0
    xq, xs, xg, wq, ws, wg, _ = _case(m, M, N, K, 303, False)
    Y_ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    m.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, None, Y_ref, M, N, K)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    m.vlaq_linear_nvfp4_noalloc(xq, xs, xg, wq, ws, wg, None, Y, M, N, K)
    torch.cuda.synchronize()
    rel, _ = gemm_error(Y.float().cpu().numpy(), Y_ref.float().cpu().numpy().astype(np.float64))
    assert rel < REL_FRO_TOL


def test_noalloc_refuses_shapes_beyond_the_static_scratch():
    m = vq()
    M, N, K = 128, 2048, 8192  # split-K plan needs ~9.4 MB > 4 MiB
    need = m.vlaq_linear_workspace_bytes(M, N, K)
    assert need > 4 * 1024 * 1024
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.VlaqError) as ei:
        m.vlaq_linear_nvfp4_noalloc(xq, xs, xg, wq, ws, wg, None, Y, M, N, K)
    assert ei.value.status == 7 and "static scratch" in ei.value.message

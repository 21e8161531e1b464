"""Shared helpers of the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same bytes, compare."""
import numpy as np
import torch

import layouts
import oracle
import synthetic_inputs as si

REL_FRO_TOL = 2e-3  # GEMM gate: relative Frobenius error vs the fp64 oracle


def vq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device (no fallback exists)"
    from conftest import build_library
    build_library()
    import vlaq_quantize_act_b200 as m
    return m


def bits(t):
    return si.to_bits(t)


def gpu_quant_act_nvfp4(X, gamma=None, eps=1e-6, flags=0):
    m = vq()
    M, K = X.shape
    Xd = X.cuda()
    gd = None if gamma is None else gamma.cuda()
    codes, scales, g = m.alloc_nvfp4(M, K)
    m.vlaq_quantize_act_nvfp4(Xd, M, K, gd, eps, flags, codes, scales, g)
    torch.cuda.synchronize()
    m.vlaq_check()
    return codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()


def gpu_quant_weight_nvfp4(W, flags=0):
    m = vq()
    N, K = W.shape
    codes, scales, g = m.alloc_nvfp4(N, K, per_tensor=True)
    m.vlaq_quantize_weight_nvfp4(W.cuda(), N, K, flags, codes, scales, g)
    torch.cuda.synchronize()
    m.vlaq_check()
    return codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()


def gpu_quant_fp8(X, gamma=None, eps=1e-6, flags=0, weight=False):
    m = vq()
    R, K = X.shape
    codes, s = m.alloc_fp8(R, K)
    if weight:
        m.vlaq_quantize_weight_fp8(X.cuda(), R, K, flags, codes, s)
    else:
        m.vlaq_quantize_act_fp8(X.cuda(), R, K, None if gamma is None else gamma.cuda(), eps, flags, codes, s)
    torch.cuda.synchronize()
    m.vlaq_check()
    return codes.cpu().numpy(), s.cpu().numpy()


def assert_nvfp4_equal(gpu, ref, rows, K, what=""):
    gc, gs, gg = gpu
    rc, rs, rg = ref
    assert gc.shape[1] == layouts.code_pitch(K)
    bad = np.argwhere(gc[:rows, : K // 2] != rc)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first {bad[:4].tolist()}"
    assert not gc[:rows, K // 2:].any(), f"{what}: code padding not zero"
    us = layouts.untile_scales(gs, rows, K)
    bad = np.argwhere(us != rs)
    assert bad.size == 0, f"{what}: {len(bad)} scale bytes differ, first {bad[:4].tolist()}"
    pad = layouts.padded_scale_offsets(rows, K)
    assert not gs.reshape(-1)[pad].any(), f"{what}: scale padding not zero"
    assert np.array_equal(gg.view(np.uint32)[: rg.size], rg.view(np.uint32)), f"{what}: global scales differ"


def gemm_error(Y_gpu, Y64):
    d = Y_gpu.astype(np.float64) - Y64
    rel = np.linalg.norm(d) / max(np.linalg.norm(Y64), 1e-300)
    return rel, float(np.abs(d).max())


def gpu_linear_nvfp4(xq, xs, gx, wq, ws, gw, M, N, K, residual=None):
    """Device tensors in the library layouts -> Y (bf16, host numpy fp32)."""
    m = vq()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_nvfp4(xq, xs, gx, wq, ws, gw, residual, Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    return Y.float().cpu().numpy()


def gpu_linear_fp8(xq, sx, wq, sw, M, N, K, residual=None):
    m = vq()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_fp8(xq, sx, wq, sw, residual, Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    return Y.float().cpu().numpy()


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()

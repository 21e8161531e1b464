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


U32 = 2.0 ** -24  # fp32 unit roundoff


def half_ulp_bf16(v):
    """Half the bf16 spacing at |v| (8 significant bits; subnormal floor)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(np.int64) - 8)


def elementwise_bound(Y64, Y_gpu, absdot, K, residual=None):
    """Per-element bound on |Y - Y64| for a GEMM that accumulates in fp32
    and rounds its output to bf16 once:
      1/2 ulp_bf16 of the larger of |Y|, |Y64|        (output rounding)
      + K u sum_k |x_k w_k|                           (at most K fp32 additions
                                                       in the accumulation
                                                       chain, split-K partials
                                                       included: gamma_K <= K u
                                                       to first order)
      + 4 u (sum_k |x_k w_k| + |residual|)            (global-scale product,
                                                       scaling, residual add)
    with u = 2^-24 and x, w the decoded operands (absdot = |X| |W|^T)."""
    bound = half_ulp_bf16(np.maximum(np.abs(Y64), np.abs(Y_gpu.astype(np.float64))))
    bound = bound + (K + 4) * U32 * absdot
    if residual is not None:
        bound = bound + 4 * U32 * np.abs(residual)
    return bound


def check_gemm(Y_gpu, Y64, dx, dw, K, residual=None, what=""):
    """Relative Frobenius gate (< REL_FRO_TOL) and the element-wise bound on
    every compared element.  dx [rows, K], dw [N, K] are the decoded
    operands of exactly the compared rows; residual (fp64 [rows, N]) or
    None.  Returns (rel_fro, max_abs, worst error / bound)."""
    Yg = Y_gpu.astype(np.float64)
    rel, mx = gemm_error(Yg, Y64)
    absdot = np.abs(np.asarray(dx, np.float64)) @ np.abs(np.asarray(dw, np.float64)).T
    bound = elementwise_bound(Y64, Yg, absdot, K, residual)
    ratio = np.abs(Yg - Y64) / bound
    worst = float(ratio.max()) if ratio.size else 0.0
    print(f"{what}: rel_fro={rel:.3e} max_abs={mx:.3e} worst err/bound={worst:.3f}")
    assert np.isfinite(Yg).all(), f"{what}: non-finite output"
    assert rel < REL_FRO_TOL, (what, rel, mx)
    if worst > 1.0:
        i = np.unravel_index(int(ratio.argmax()), ratio.shape)
        raise AssertionError(f"{what}: element {tuple(int(t) for t in i)} off by {abs(Yg[i] - Y64[i]):.4e} "
                             f"> bound {bound[i]:.4e} (Y={Yg[i]:.6e}, Y64={Y64[i]:.6e})")
    return rel, mx, worst


def residual_f64(R_bf16, rows=None):
    """bf16 residual tensor -> fp64 numpy (optionally a row subset)."""
    if R_bf16 is None:
        return None
    r = R_bf16.float().cpu().numpy().astype(np.float64)
    return r if rows is None else r[rows]


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

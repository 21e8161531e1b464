"""Parity at the full workload sizes (Qwen2.5-VL-7B-shaped projections).

Every code, block scale and global scale is compared bit-exactly in full;
GEMM outputs are compared on sampled token rows (the oracle computes those
rows one by one in fp64): at least one row of every 128-row tile, all
columns (so every output tile of the launch is visited), in the same launch
configuration the benchmark times, against the relative Frobenius gate and
the element-wise bound of gpu_helpers.check_gemm.  Covers prefill M = 1024,
decode M in {1, 4, 8}, the fused RMSNorm + Hadamard + residual path with its
FP8 variant, and M = 4580, the largest token count of the native-FP4
numeric gate in "Alpamayo 2 Super NVFP4: full test reflection" (36 m-tiles,
several tiles per CTA on the qkv shape)."""
import numpy as np
import pytest
import torch

import layouts
import oracle
import synthetic_inputs as si
from gpu_helpers import assert_nvfp4_equal, bits, check_gemm, residual_f64, vq

pytestmark = pytest.mark.gpu

_W_CACHE = {}


def _weights(name, flags):
    """Oracle quantization + decode of a projection weight (cached)."""
    key = (name, flags)
    if key not in _W_CACHE:
        K, N, seed = si.PROJECTIONS[name]
        W = si.projection_weight(K, N, seed)
        cw, sw, gw = oracle.quantize_nvfp4(bits(W), flags=flags, per_tensor=True)
        dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
        _W_CACHE.clear()
        _W_CACHE[key] = (W, (cw, sw, gw), dw)
    return _W_CACHE[key]


def _sample_rows(M, n=16):
    """n random rows, the first and last row, and one random row of every
    128-row tile (every m-tile of the GEMM launch is compared)."""
    rng = np.random.default_rng(M)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows.update({0, M - 1})
    for t0 in range(0, M, 128):
        rows.add(int(t0 + rng.integers(0, min(128, M - t0))))
    return np.array(sorted(rows))


def _run_projection(name, M, flags=0, residual=False, full_codes=True):
    m = vq()
    K, N, seed = si.PROJECTIONS[name]
    W, wref, dw = _weights(name, flags & 2)
    X = si.projection_activations(K, M, seed)
    gam = si.norm_gain(K, seed)
    R = si.residual(M, N, seed) if residual else None
    # GPU path
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    m.vlaq_quantize_weight_nvfp4(W.cuda(), N, K, flags & 2, wq, ws, wg)
    xq, xs, xg = m.alloc_nvfp4(M, K)
    m.vlaq_quantize_act_nvfp4(X.cuda(), M, K, gam.cuda(), 1e-6, flags, xq, xs, xg)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, None if R is None else R.cuda(), Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    # oracle
    assert_nvfp4_equal((wq.cpu().numpy(), ws.cpu().numpy(), wg.cpu().numpy()), wref, N, K, f"{name} W")
    rows = _sample_rows(M)
    if full_codes:
        xref = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, flags)
        assert_nvfp4_equal((xq.cpu().numpy(), xs.cpu().numpy(), xg.cpu().numpy()), xref, M, K, f"{name} X")
        xr = (xref[0][rows], xref[1][rows], xref[2][rows])
    else:
        # rows are independent: the oracle quantizes the sampled rows only,
        # compared with the same rows of the GPU output (codes, scales, g)
        xr = oracle.quantize_nvfp4(bits(X[rows]), bits(gam), 1e-6, flags)
        gc, gs, gg = xq.cpu().numpy(), xs.cpu().numpy(), xg.cpu().numpy()
        assert np.array_equal(gc[rows, : K // 2], xr[0]), f"{name} X codes (sampled rows)"
        us = layouts.untile_scales(gs, M, K)
        assert np.array_equal(us[rows], xr[1]), f"{name} X scales (sampled rows)"
        assert np.array_equal(gg[rows].view(np.uint32), xr[2].view(np.uint32)), f"{name} X g (sampled rows)"
    dx = oracle.decode_nvfp4(xr[0], xr[1], xr[2], K)
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R)[rows])
    check_gemm(Y.float().cpu().numpy()[rows], Y64, dx, dw, K, residual_f64(R, rows),
               f"{name} M={M} flags={flags} res={residual}")


@pytest.mark.parametrize("name", ["qkv", "o", "gate_up", "down"])
def test_prefill_m1024(name):
    _run_projection(name, 1024)


@pytest.mark.parametrize("name", ["qkv", "o", "gate_up", "down"])
@pytest.mark.parametrize("M", [1, 4, 8])
def test_decode(name, M):
    _run_projection(name, M)


@pytest.mark.parametrize("name", ["qkv", "down"])
def test_prefill_m4580(name):
    """The largest token count of the pages' native-FP4 gate (M = 4580):
    36 m-tiles with a ragged last tile (4580 = 35 * 128 + 100)."""
    _run_projection(name, 4580, full_codes=False)


# the fused workload: RMSNorm + WHT on the qkv / gate_up inputs, WHT and a
# residual add on o / down (flags 1 = RMSNorm, 2 = WHT)
FUSED = [(c.name, 3 if c.rmsnorm else 2, c.residual) for c in si.FUSED_CASES]


@pytest.mark.parametrize("name,flags,residual", FUSED)
def test_fused_prologue_m1024(name, flags, residual):
    _run_projection(name, 1024, flags, residual)


@pytest.mark.parametrize("name,flags,residual", [("qkv", 3, False), ("down", 2, True)])
def test_fused_fp8_m1024(name, flags, residual):
    _run_fp8(name, 1024, flags, residual)


def test_fp8_m4580():
    """The FP8 GEMM over CTA pairs at M = 4580 on the o shape: 18 x 14 tiles
    of 256 x 256 on 74 clusters (several tiles per cluster through both
    accumulator buffers, a ragged last row tile), with the residual."""
    _run_fp8("o", 4580, 0, True)


def _run_fp8(name, M, flags, residual):
    m = vq()
    K, N, seed = si.PROJECTIONS[name]
    W = si.projection_weight(K, N, seed)
    X = si.projection_activations(K, M, seed)
    gam = si.norm_gain(K, seed)
    R = si.residual(M, N, seed) if residual else None
    wq, sw = m.alloc_fp8(N, K)
    m.vlaq_quantize_weight_fp8(W.cuda(), N, K, flags & 2, wq, sw)
    xq, sx = m.alloc_fp8(M, K)
    m.vlaq_quantize_act_fp8(X.cuda(), M, K, gam.cuda(), 1e-6, flags, xq, sx)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_fp8(xq, sx, wq, sw, None if R is None else R.cuda(), Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    rw = oracle.quantize_fp8(bits(W), flags=flags & 2)
    rx = oracle.quantize_fp8(bits(X), bits(gam), 1e-6, flags)
    assert np.array_equal(wq.cpu().numpy(), rw[0]) and np.array_equal(xq.cpu().numpy(), rx[0])
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), rw[1].view(np.uint32))
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rx[1].view(np.uint32))
    rows = _sample_rows(M)
    dx, dw = oracle.decode_fp8(rx[0][rows], rx[1][rows]), oracle.decode_fp8(rw[0], rw[1])
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R)[rows])
    check_gemm(Y.float().cpu().numpy()[rows], Y64, dx, dw, K, residual_f64(R, rows),
               f"fp8 {name} M={M} flags={flags} res={residual}")


def test_k3420_refused_on_device():
    m = vq()
    X = torch.zeros(4, 3420, dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros(4, 2048, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.VlaqError) as ei:
        m.vlaq_quantize_act_nvfp4(X, 4, 3420, None, 1e-6, 0, codes, codes, codes)
    assert "3420 / 16 = 213.75" in ei.value.message
    assert not codes.any()

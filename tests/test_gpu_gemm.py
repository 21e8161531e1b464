"""GPU parity of the tcgen05 GEMMs against the fp64 oracle.

The GEMM is fed the oracle's own codes and scales (re-laid out into the
library's padded / tiled buffers), so the comparison isolates the GEMM; the
end-to-end cases run the GPU quantizers too (their bytes are bit-exact, see
test_gpu_quant.py).  Gates, on every output element: relative Frobenius
error < 2e-3 against the fp64 result on the same decoded operands, and the
element-wise bound of an fp32-accumulated GEMM with one bf16 output rounding
(gpu_helpers.elementwise_bound); max-abs and the worst error / bound ratio
are printed."""
import numpy as np
import pytest
import torch

import layouts
import oracle
import synthetic_inputs as si
from gpu_helpers import (REL_FRO_TOL, bits, check_gemm, gemm_error, gpu_linear_fp8, gpu_linear_nvfp4,
                         gpu_quant_act_nvfp4, gpu_quant_weight_nvfp4, residual_f64, to_dev, vq)

pytestmark = pytest.mark.gpu


def _oracle_case(M, N, K, seed, residual=False, flags=0):
    X = si.projection_activations(K, M, seed)
    W = si.projection_weight(K, N, seed)
    cx, sx, gx = oracle.quantize_nvfp4(bits(X), flags=flags)
    cw, sw, gw = oracle.quantize_nvfp4(bits(W), flags=flags, per_tensor=True)
    R = si.residual(M, N, seed) if residual else None
    dx = oracle.decode_nvfp4(cx, sx, gx, K)
    dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R))
    return (cx, sx, gx, cw, sw, gw, R, Y64, dx, dw)


def _check(Y, case, K, what):
    """Frobenius gate and the element-wise bound against the oracle case."""
    return check_gemm(Y, case[7], case[8], case[9], K, residual_f64(case[6]), what)


def _run_nvfp4_from_oracle(M, N, K, case):
    cx, sx, gx, cw, sw, gw, R = case[:7]
    return gpu_linear_nvfp4(to_dev(layouts.pad_codes(cx, K)), to_dev(layouts.tile_scales(sx, M, K)), to_dev(gx),
                            to_dev(layouts.pad_codes(cw, K)), to_dev(layouts.tile_scales(sw, N, K)), to_dev(gw),
                            M, N, K, None if R is None else R.cuda())


# (M, N, K): one tile; ragged M / N / K tails; several K stages; split-K
# decode shapes (M <= 8 with few N tiles); residual add; the last row count
# of the few-row kernel (32) and the first of the wide one (33).
NVFP4_CASES = [
    (16, 128, 256, False),
    (128, 128, 256, False),
    (300, 392, 1024, False),
    (130, 264, 336, True),
    (257, 136, 3584, True),
    (1, 512, 4096, False),
    (4, 256, 2048, True),
    (8, 1024, 3584, False),
    (1, 8, 64, False),
    (64, 4608, 256, False),
    (32, 264, 512, True),
    (33, 256, 1024, False),
]


@pytest.mark.parametrize("M,N,K,res", NVFP4_CASES)
def test_linear_nvfp4_vs_oracle(M, N, K, res):
    case = _oracle_case(M, N, K, 21, residual=res)
    Y = _run_nvfp4_from_oracle(M, N, K, case)
    _check(Y, case, K, f"nvfp4 M={M} N={N} K={K} res={res}")


def test_linear_nvfp4_single_element_parity_positions():
    """1x16x1-style probe: one non-zero element at every position of a
    16-block (both nibbles, every k-step) must land on the right product."""
    M, N, K = 1, 8, 256
    for pos in range(0, K, 7):
        x = np.zeros((M, K), np.float32)
        w = np.zeros((N, K), np.float32)
        x[0, pos] = 3.0
        w[:, pos] = np.arange(1, N + 1, dtype=np.float32)
        Xb = torch.from_numpy(x).to(torch.bfloat16)
        Wb = torch.from_numpy(w).to(torch.bfloat16)
        cx, sx, gx = oracle.quantize_nvfp4(bits(Xb))
        cw, sw, gw = oracle.quantize_nvfp4(bits(Wb), per_tensor=True)
        dx = oracle.decode_nvfp4(cx, sx, gx, K)
        dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
        case = (cx, sx, gx, cw, sw, gw, None, oracle.linear_f64(dx, dw), dx, dw)
        Y = _run_nvfp4_from_oracle(M, N, K, case)
        _check(Y, case, K, f"single element at {pos}")


@pytest.mark.parametrize("M,N,K,res", [(16, 128, 256, False), (300, 392, 1024, True), (129, 136, 208, False),
                                       (1, 512, 4096, True), (8, 256, 2048, False), (257, 264, 3584, False)])
def test_linear_fp8_vs_oracle(M, N, K, res):
    X = si.projection_activations(K, M, 31)
    W = si.projection_weight(K, N, 31)
    cx, sx = oracle.quantize_fp8(bits(X))
    cw, sw = oracle.quantize_fp8(bits(W))
    R = si.residual(M, N, 31) if res else None
    dx, dw = oracle.decode_fp8(cx, sx), oracle.decode_fp8(cw, sw)
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R))
    Y = gpu_linear_fp8(to_dev(cx), to_dev(sx), to_dev(cw), to_dev(sw), M, N, K, None if R is None else R.cuda())
    check_gemm(Y, Y64, dx, dw, K, residual_f64(R), f"fp8 M={M} N={N} K={K} res={res}")


@pytest.mark.parametrize("M,N,K,flags,res", [(200, 256, 1024, 0, False), (70, 384, 512, 3, True),
                                             (3, 640, 2048, 2, True)])
def test_end_to_end_nvfp4(M, N, K, flags, res):
    """GPU quantizers + GPU GEMM vs oracle quantizers + fp64 GEMM."""
    m = vq()
    X = si.projection_activations(K, M, 41)
    W = si.projection_weight(K, N, 41)
    gam = si.norm_gain(K, 41)
    R = si.residual(M, N, 41) if res else None
    cx, sx, gx = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, flags)
    cw, sw, gw = oracle.quantize_nvfp4(bits(W), flags=flags & 2, per_tensor=True)
    dx = oracle.decode_nvfp4(cx, sx, gx, K)
    dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R))
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    m.vlaq_quantize_weight_nvfp4(W.cuda(), N, K, flags & 2, wq, ws, wg)
    m.vlaq_quantize_act_nvfp4(X.cuda(), M, K, gam.cuda(), 1e-6, flags, xq, xs, xg)
    Y = gpu_linear_nvfp4(xq, xs, xg, wq, ws, wg, M, N, K, None if R is None else R.cuda())
    check_gemm(Y, Y64, dx, dw, K, residual_f64(R), f"end to end M={M} N={N} K={K} flags={flags}")


@pytest.mark.parametrize("M,N,K", [(1024, 2560, 1024), (8, 1024, 3584), (1, 512, 4096)])
def test_weights_quantized_right_before_linear(M, N, K):
    """The stream-order contract of vlaq_linear_nvfp4: the GEMM may read wq /
    ws before its dependency wait, and weights quantized by
    vlaq_quantize_weight_nvfp4 immediately before it are complete (their
    codes and scales come from its second-to-last kernel).  Everything is
    allocated first; then the activation quantizer, the weight quantizer and
    the GEMM are launched back to back on the stream, nothing in between
    (CTA pairs, split-K tensor-core path, few-row kernel)."""
    m = vq()
    X = si.projection_activations(K, M, 51)
    W = si.projection_weight(K, N, 51)
    cx, sx, gx = oracle.quantize_nvfp4(bits(X))
    cw, sw, gw = oracle.quantize_nvfp4(bits(W), per_tensor=True)
    dx = oracle.decode_nvfp4(cx, sx, gx, K)
    dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    Y64 = oracle.linear_f64(dx, dw, None)
    Xd, Wd = X.cuda(), W.cuda()
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    torch.cuda.synchronize()
    for _ in range(2):
        m.vlaq_quantize_act_nvfp4(Xd, M, K, None, 1e-6, 0, xq, xs, xg)
        m.vlaq_quantize_weight_nvfp4(Wd, N, K, 0, wq, ws, wg)
        m.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, None, Y, M, N, K, wsp, nb)
        torch.cuda.synchronize()
        m.vlaq_check()
        check_gemm(Y.float().cpu().numpy(), Y64, dx, dw, K, None, f"weights right before M={M} N={N} K={K}")


def test_workspace_is_checked():
    m = vq()
    M, N, K = 8, 512, 4096
    need = m.vlaq_linear_workspace_bytes(M, N, K)
    assert need > 0  # this decode shape runs split-K
    xq, xs, xg = m.alloc_nvfp4(M, K)
    wq, ws, wg = m.alloc_nvfp4(N, K, per_tensor=True)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.VlaqError) as ei:
        m.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, None, Y, M, N, K, None, 0)
    assert ei.value.status == 7


# Shapes with more than 74 output tiles of 128 x 256 run without split-K.
# With more than 128 rows they take the paired kernel (256 x 256 tiles over
# the two CTAs of a cluster): ragged M (a tile whose odd CTA has no rows,
# 777; rows 129-256, 200), ragged N (a tile whose odd CTA has no B rows,
# 2568), several tiles per CTA pair (9728, 19200).  K % 256 == 0 runs two
# K-chunks per stage (an odd chunk count, 1024 + 256 ... 256, leaves the
# last stage half outside K); other K one chunk per stage with TMA stores
# (336, 320).  With at most 128 rows, the single-CTA kernel with its direct
# epilogue (100 rows).
WIDE_CASES = [
    (1024, 2560, 1024, False),
    (1000, 2568, 336, True),
    (777, 4096, 512, True),
    (1024, 9728, 512, False),
    (200, 19200, 256, True),
    (512, 19200, 320, False),
    (384, 9728, 1280, True),
    (100, 19456, 256, True),
]


@pytest.mark.parametrize("M,N,K,res", WIDE_CASES)
def test_linear_nvfp4_wide_tiles_vs_oracle(M, N, K, res):
    m = vq()
    assert m.vlaq_linear_workspace_bytes(M, N, K) == 0
    case = _oracle_case(M, N, K, 23, residual=res)
    Y = _run_nvfp4_from_oracle(M, N, K, case)
    _check(Y, case, K, f"nvfp4 wide M={M} N={N} K={K} res={res}")


# the first two wide cases, then 256 x 256 tiles over CTA pairs (more than
# 128 rows, enough tiles, K % 256 == 0): ragged M with two tiles per
# cluster, ragged N with K = 3 stages, K = 1 stage, 200 rows in one tile
@pytest.mark.parametrize("M,N,K,res", WIDE_CASES[:2] + [(300, 9728, 512, True), (1000, 4104, 768, False),
                                                        (512, 19200, 256, True), (200, 19200, 256, False)])
def test_linear_fp8_wide_tiles_vs_oracle(M, N, K, res):
    X = si.projection_activations(K, M, 33)
    W = si.projection_weight(K, N, 33)
    cx, sx = oracle.quantize_fp8(bits(X))
    cw, sw = oracle.quantize_fp8(bits(W))
    R = si.residual(M, N, 33) if res else None
    dx, dw = oracle.decode_fp8(cx, sx), oracle.decode_fp8(cw, sw)
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R))
    Y = gpu_linear_fp8(to_dev(cx), to_dev(sx), to_dev(cw), to_dev(sw), M, N, K, None if R is None else R.cuda())
    check_gemm(Y, Y64, dx, dw, K, residual_f64(R), f"fp8 wide M={M} N={N} K={K} res={res}")


def test_split_workspace_reused_across_calls_and_shapes():
    """The NVFP4 split-K tile counters return to zero after every call: one
    zeroed workspace serves repeated calls and shapes with different split
    counts.  A counter left non-zero would keep the next call's last split
    from recognising itself, and its tile would stay NaN."""
    m = vq()
    shapes = [(5, 512, 4096), (8, 1024, 3584), (6, 256, 2048)]
    need = max(m.vlaq_linear_workspace_bytes(*s) for s in shapes)
    assert all(m.vlaq_linear_workspace_bytes(*s) > 0 for s in shapes)  # all three split K
    wsp = torch.zeros(need, dtype=torch.uint8, device="cuda")
    cases = {s: _oracle_case(*s, 51) for s in shapes}
    dev = {}
    for (M, N, K), (cx, sx, gx, cw, sw, gw, *_) in cases.items():
        dev[(M, N, K)] = (to_dev(layouts.pad_codes(cx, K)), to_dev(layouts.tile_scales(sx, M, K)), to_dev(gx),
                          to_dev(layouts.pad_codes(cw, K)), to_dev(layouts.tile_scales(sw, N, K)), to_dev(gw))
    first = {}
    for rep in range(3):
        for (M, N, K) in shapes:
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            m.vlaq_linear_nvfp4(*dev[(M, N, K)], None, Y, M, N, K, wsp, need)
            torch.cuda.synchronize()
            m.vlaq_check()
            y = Y.float().cpu().numpy()
            _check(y, cases[(M, N, K)], K, f"rep {rep} {M}x{N}x{K}")
            if rep == 0:
                first[(M, N, K)] = y
            else:
                assert np.array_equal(y, first[(M, N, K)]), (rep, M, N, K)


# one or two token rows against weights of at most 2^25 elements take the
# weight-streaming CUDA-core kernel (larger M or weights the tensor-core
# one, split K): ragged K (K % 64 in {16, 32, 48}, K = 16), N = 8, a partial
# last group of rows per CTA, the decode projection shapes, up to 32 token
# rows, residual on and off
FEW_ROW_CASES = [(1, 8, 16, False), (2, 24, 48, True), (3, 136, 208, False), (4, 512, 4096, True),
                 (1, 4608, 3584, True), (4, 4608, 3584, False), (1, 3584, 18944, True), (2, 3584, 18944, False),
                 (3, 40, 336, True), (1, 37888, 3584, False), (8, 37888, 3584, True), (32, 1000, 1024, True),
                 (17, 3584, 18944, False), (2, 1024, 18944, True)]


@pytest.mark.parametrize("M,N,K,res", FEW_ROW_CASES + [(2, 4608, 3584, True), (2, 3584, 3584, False)])
def test_linear_nvfp4_few_rows(M, N, K, res):
    m = vq()
    X = si.projection_activations(K, M, 61)
    W = si.projection_weight(K, N, 61)
    cx, sx, gx = oracle.quantize_nvfp4(bits(X))
    cw, sw, gw = oracle.quantize_nvfp4(bits(W), per_tensor=True)
    R = si.residual(M, N, 61) if res else None
    dx = oracle.decode_nvfp4(cx, sx, gx, K)
    dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    Y64 = oracle.linear_f64(dx, dw, None if R is None else bits(R))
    dev = (to_dev(layouts.pad_codes(cx, K)), to_dev(layouts.tile_scales(sx, M, K)), to_dev(gx),
           to_dev(layouts.pad_codes(cw, K)), to_dev(layouts.tile_scales(sw, N, K)), to_dev(gw))
    Y = gpu_linear_nvfp4(*dev, M, N, K, None if R is None else R.cuda())
    check_gemm(Y, Y64, dx, dw, K, residual_f64(R), f"few rows M={M} N={N} K={K} res={res}")
    # a second call gives the same bits (a shape without a split plan runs
    # without a workspace)
    Y2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = (None, 0) if m.vlaq_linear_workspace_bytes(M, N, K) == 0 else m.alloc_workspace(M, N, K)
    m.vlaq_linear_nvfp4(*dev, None if R is None else R.cuda(), Y2, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    assert np.array_equal(Y2.float().cpu().numpy(), Y)

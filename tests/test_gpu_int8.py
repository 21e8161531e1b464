"""GPU parity of the INT8 W8A8 path (FoldQuant's 8-bit integer path:
symmetric per-row weight / per-token activation scales, round half to even,
clamp): codes and scales bit-exact against the oracle, and -- because the
integer sums are exact and every fp32 epilogue step is rounded once -- GEMM
outputs bit-exact too, at every tile shape, split-K plan and ragged edge."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from gpu_helpers import bits, to_dev, vq

pytestmark = pytest.mark.gpu


def gpu_quant_int8(X, gamma=None, eps=1e-6, flags=0, weight=False):
    m = vq()
    R, K = X.shape
    codes, s = m.alloc_int8(R, K)
    if weight:
        m.vlaq_quantize_weight_int8(X.cuda(), R, K, flags, codes, s)
    else:
        m.vlaq_quantize_act_int8(X.cuda(), R, K, None if gamma is None else gamma.cuda(), eps, flags, codes, s)
    torch.cuda.synchronize()
    m.vlaq_check()
    return codes.cpu().numpy()[:R], s.cpu().numpy()[:R]


def gpu_linear_int8(cx, sx, cw, sw, M, N, K, residual=None):
    """Device tensors -> Y as bf16 bit patterns (uint16 numpy)."""
    m = vq()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_int8(cx, sx, cw, sw, residual, Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    return Y.cpu().view(torch.int16).numpy().view(np.uint16)


def assert_bits_equal(got, want, what):
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{what}: {len(bad)} of {got.size} outputs differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("M,K", [(16, 256), (1, 16), (130, 336), (257, 1024), (5, 18944), (2, 32768)])
@pytest.mark.parametrize("flags", [0, 1, 3])
def test_act_int8_vs_oracle(M, K, flags):
    if flags & 2 and K % 64:
        pytest.skip("Hadamard needs K % 64 == 0")
    X = si.projection_activations(K, M, 51)
    gam = si.norm_gain(K, 51)
    rc, rs = oracle.quantize_int8(bits(X), bits(gam), 1e-6, flags)
    gc, gs = gpu_quant_int8(X, gam, 1e-6, flags)
    assert_bits_equal(gc, rc, f"int8 codes {M}x{K} f{flags}")
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("N,K,flags", [(128, 256, 0), (77, 1024, 2), (40, 208, 0), (3584, 3584, 2)])
def test_weight_int8_vs_oracle(N, K, flags):
    W = si.projection_weight(K, N, 52)
    rc, rs = oracle.quantize_int8(bits(W), flags=flags)
    gc, gs = gpu_quant_int8(W, flags=flags, weight=True)
    assert_bits_equal(gc, rc, f"int8 weight {N}x{K}")
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))


def test_int8_ties_and_edge_rows():
    """Rows with exact ties (amax 127: s = 1), an all-zero row, extreme
    magnitudes and a lone outlier."""
    K = 64
    rows = []
    r = np.zeros(K, np.float32); r[0] = 127.0; r[1:14] = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 63.5, 64.5, 125.5,
                                                          126.5, -126.5, 0.25]; rows.append(r)
    rows.append(np.zeros(K, np.float32))
    r = np.full(K, 3e38, np.float32); r[5] = -3.3e38; rows.append(r)
    r = np.full(K, 1e-38, np.float32); r[3] = 3e-38; rows.append(r)
    r = np.zeros(K, np.float32); r[9] = -1e4; r[10] = 1e-3; rows.append(r)
    X = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    rc, rs = oracle.quantize_int8(bits(X))
    gc, gs = gpu_quant_int8(X)
    assert_bits_equal(gc, rc, "int8 edge rows")
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))


# (M, N, K, residual): tile-aligned, ragged M / N / K (K % 128 in {16, 48}),
# decode rows (split-K over the SMs), both tile widths, the projection
# shapes; then 256 x 256 tiles over CTA pairs (more than 128 rows, enough
# tiles, K % 256 == 0): one tile per cluster, ragged M with two tiles per
# cluster (both accumulator buffers), ragged N with K = 3 stages, K = 1 stage,
# and 200 rows (one 256-row tile, the second CTA's 128 rows partly past M)
INT8_GEMMS = [(16, 128, 256, False), (300, 392, 1024, True), (129, 136, 208, False), (1, 512, 4096, True),
              (8, 256, 2048, False), (257, 264, 3584, False), (1, 3584, 18944, True), (4, 4608, 3584, False),
              (1024, 512, 3584, True), (33, 8, 48, True),
              (1024, 2560, 1024, True), (300, 9728, 512, False), (1000, 4104, 768, True), (512, 19200, 256, False),
              (200, 19200, 256, True)]


@pytest.mark.parametrize("M,N,K,res", INT8_GEMMS)
def test_linear_int8_bit_exact(M, N, K, res):
    X = si.projection_activations(K, M, 53)
    W = si.projection_weight(K, N, 53)
    cx, sx = oracle.quantize_int8(bits(X))
    cw, sw = oracle.quantize_int8(bits(W))
    R = si.residual(M, N, 53) if res else None
    want, _ = oracle.linear_int8(cx, sx, cw, sw, None if R is None else bits(R))
    got = gpu_linear_int8(to_dev(cx), to_dev(sx), to_dev(cw), to_dev(sw), M, N, K, None if R is None else R.cuda())
    assert_bits_equal(got, want, f"int8 GEMM {M}x{N}x{K}")


def test_int8_split_workspace_reused_across_calls_and_shapes():
    """The 8-bit split-K tile counters return to zero after every call: one
    zeroed workspace serves repeated INT8 calls of shapes with different
    split counts, every output bit-exact (a counter left non-zero would keep
    a tile's last split from recognising itself)."""
    m = vq()
    shapes = [(5, 512, 4096), (8, 1024, 3584), (6, 256, 2048)]
    need = max(m.vlaq_linear_workspace_bytes(*s) for s in shapes)
    assert all(m.vlaq_linear_workspace_bytes(*s) > 0 for s in shapes)  # all three split K
    wsp = torch.zeros(need, dtype=torch.uint8, device="cuda")
    cases = {}
    for (M, N, K) in shapes:
        X = si.projection_activations(K, M, 59)
        W = si.projection_weight(K, N, 59)
        cx, sx = oracle.quantize_int8(bits(X))
        cw, sw = oracle.quantize_int8(bits(W))
        want, _ = oracle.linear_int8(cx, sx, cw, sw)
        cases[(M, N, K)] = ((to_dev(cx), to_dev(sx), to_dev(cw), to_dev(sw)), want)
    for rep in range(3):
        for (M, N, K), (dev, want) in cases.items():
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            m.vlaq_linear_int8(*dev, None, Y, M, N, K, wsp, need)
            torch.cuda.synchronize()
            m.vlaq_check()
            assert_bits_equal(Y.cpu().view(torch.int16).numpy().view(np.uint16), want, f"rep {rep} {M}x{N}x{K}")


def test_linear_int8_extreme_sums():
    """Every product +-127^2 at the largest K: |acc| = K 127^2 < 2^31, where
    fp32(acc) rounds (acc > 2^24)."""
    M, N, K = 3, 24, 32768
    cx = np.full((M, K), 127, np.int8); cx[1] = -127; cx[2, ::2] = -127
    cw = np.full((N, K), 127, np.int8); cw[::3] = -127
    sx = np.array([1e-3, 0.5, 3.0], np.float32)
    sw = np.linspace(1e-4, 2e-3, N).astype(np.float32)
    want, acc = oracle.linear_int8(cx, sx, cw, sw)
    assert np.abs(acc).max() == K * 127 * 127
    got = gpu_linear_int8(to_dev(cx), to_dev(sx), to_dev(cw), to_dev(sw), M, N, K)
    assert_bits_equal(got, want, "int8 extreme sums")


@pytest.mark.parametrize("M,N,K,flags,res", [(200, 256, 1024, 0, False), (70, 384, 512, 3, True),
                                             (3, 640, 2048, 2, True)])
def test_end_to_end_int8(M, N, K, flags, res):
    """GPU quantizers + GPU GEMM vs oracle quantizers + oracle GEMM: bit-exact."""
    m = vq()
    X = si.projection_activations(K, M, 54)
    W = si.projection_weight(K, N, 54)
    gam = si.norm_gain(K, 54)
    R = si.residual(M, N, 54) if res else None
    xq, sx = m.alloc_int8(M, K)
    wq, sw = m.alloc_int8(N, K)
    m.vlaq_quantize_weight_int8(W.cuda(), N, K, flags & 2, wq, sw)
    m.vlaq_quantize_act_int8(X.cuda(), M, K, gam.cuda(), 1e-6, flags, xq, sx)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_int8(xq, sx, wq, sw, None if R is None else R.cuda(), Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    cx, rsx = oracle.quantize_int8(bits(X), bits(gam), 1e-6, flags)
    cw, rsw = oracle.quantize_int8(bits(W), flags=flags & 2)
    want, _ = oracle.linear_int8(cx, rsx, cw, rsw, None if R is None else bits(R))
    assert_bits_equal(Y.cpu().view(torch.int16).numpy().view(np.uint16), want, f"int8 e2e {M}x{N}x{K}")


def test_linear_int8_m4580_sampled_rows():
    """The INT8 GEMM over CTA pairs at M = 4580, o shape (3584 x 3584) with
    the residual: 18 x 14 tiles of 256 x 256 on 74 clusters, so clusters run
    several tiles through both accumulator buffers and the last row tile is
    ragged (4580 = 17 * 256 + 228); outputs bit-exact on sampled rows, one
    in every 128-row block."""
    m = vq()
    M, N, K = 4580, 3584, 3584
    X = si.projection_activations(K, M, 57)
    W = si.projection_weight(K, N, 57)
    R = si.residual(M, N, 57)
    xq, sx = m.alloc_int8(M, K)
    wq, sw = m.alloc_int8(N, K)
    m.vlaq_quantize_weight_int8(W.cuda(), N, K, 0, wq, sw)
    m.vlaq_quantize_act_int8(X.cuda(), M, K, None, 1e-6, 0, xq, sx)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_int8(xq, sx, wq, sw, R.cuda(), Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    rng = np.random.default_rng(58)
    rows = {0, M - 1} | {int(t + rng.integers(0, min(128, M - t))) for t in range(0, M, 128)}
    rows = np.array(sorted(rows))
    cx, rsx = oracle.quantize_int8(bits(X)[rows])
    assert np.array_equal(xq.cpu().numpy()[rows], cx)
    cw, rsw = oracle.quantize_int8(bits(W))
    assert np.array_equal(wq.cpu().numpy(), cw)
    want, _ = oracle.linear_int8(cx, rsx, cw, rsw, bits(R)[rows])
    got = Y.cpu().view(torch.int16).numpy().view(np.uint16)[rows]
    assert_bits_equal(got, want, "int8 o M=4580 sampled rows")


@pytest.mark.parametrize("N,K", [(37888, 3584), (3584, 18944)])
def test_linear_int8_full_size_sampled_rows(N, K):
    """gate_up (1024 x 37888 x 3584) and down (1024 x 3584 x 18944, 37 stages
    per tile) at the full prefill size: GPU quantizers and GEMM over CTA
    pairs, outputs bit-exact on sampled rows."""
    m = vq()
    M = 1024
    X = si.projection_activations(K, M, 55)
    W = si.projection_weight(K, N, 55)
    xq, sx = m.alloc_int8(M, K)
    wq, sw = m.alloc_int8(N, K)
    m.vlaq_quantize_weight_int8(W.cuda(), N, K, 0, wq, sw)
    m.vlaq_quantize_act_int8(X.cuda(), M, K, None, 1e-6, 0, xq, sx)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    wsp, nb = m.alloc_workspace(M, N, K)
    m.vlaq_linear_int8(xq, sx, wq, sw, None, Y, M, N, K, wsp, nb)
    torch.cuda.synchronize()
    m.vlaq_check()
    rows = np.array(sorted(set(np.random.default_rng(56).choice(M, 12, replace=False).tolist()) | {0, M - 1}))
    cx, rsx = oracle.quantize_int8(bits(X)[rows])
    assert np.array_equal(xq.cpu().numpy()[rows], cx)
    cw, rsw = oracle.quantize_int8(bits(W))
    assert np.array_equal(wq.cpu().numpy(), cw) and np.array_equal(sw.cpu().numpy().view(np.uint32),
                                                                   rsw.view(np.uint32))
    want, _ = oracle.linear_int8(cx, rsx, cw, rsw)
    got = Y.cpu().view(torch.int16).numpy().view(np.uint16)[rows]
    assert_bits_equal(got, want, f"int8 {M}x{N}x{K} sampled rows")

"""GPU parity of the quantizers: bit-exact codes, block scales and global
scales against the CPU oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
import layouts
from gpu_helpers import (assert_nvfp4_equal, bits, gpu_quant_act_nvfp4, gpu_quant_fp8,
                         gpu_quant_weight_nvfp4, to_dev, vq)

pytestmark = pytest.mark.gpu

# (M, K): several 64-blocks per row, ragged K % 64 in {16, 32, 48}, multiple
# 128-row tiles with a ragged tail, the minimum K and the maximum supported K.
SHAPES = [(16, 256), (1, 16), (3, 48), (130, 336), (257, 1024), (64, 3584), (5, 18944), (2, 32768),
          (129, 96)]


def _inputs(M, K, seed):
    X = si.projection_activations(K, M, seed)
    return X


@pytest.mark.parametrize("M,K", SHAPES)
def test_act_nvfp4_plain(M, K):
    X = _inputs(M, K, 7)
    ref = oracle.quantize_nvfp4(bits(X))
    assert_nvfp4_equal(gpu_quant_act_nvfp4(X), ref, M, K, f"act {M}x{K}")


@pytest.mark.parametrize("M,K", [(s[0], s[1]) for s in SHAPES if s[1] % 64 == 0])
@pytest.mark.parametrize("flags", [1, 2, 3])
def test_act_nvfp4_norm_hadamard(M, K, flags):
    X = _inputs(M, K, 8)
    gam = si.norm_gain(K, 8)
    ref = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, flags)
    assert_nvfp4_equal(gpu_quant_act_nvfp4(X, gam, 1e-6, flags), ref, M, K, f"act {M}x{K} f{flags}")


def test_act_nvfp4_rmsnorm_ragged_k():
    X = _inputs(33, 336, 9)
    gam = si.norm_gain(336, 9)
    ref = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-5, 1)
    assert_nvfp4_equal(gpu_quant_act_nvfp4(X, gam, 1e-5, 1), ref, 33, 336, "rmsnorm K=336")


@pytest.mark.parametrize("M", [1, 300])
def test_act_nvfp4_rmsnorm_tree_golden_row(M):
    """The hand-worked row of tests/golden/sumsq_tree.txt through the fused
    RMSNorm prologue: its global scale separates the page's reduction tree
    (FoldQuant SYCL commit) from every other summation order, so the kernel's
    tree is pinned by a value worked by hand, not only by the oracle.  M = 300
    takes the many-rows CTA shape, M = 1 the few-rows one."""
    from test_oracle_pins import sumsq_golden
    x, _, rec = sumsq_golden()
    K = x.size
    X = torch.from_numpy(np.tile(x, (M, 1))).to(torch.bfloat16)
    gam = torch.ones(K, dtype=torch.bfloat16)
    gam[0] = torch.from_numpy(np.array([int(rec["gain0"], 16)], np.uint16).view(np.int16)).view(torch.bfloat16)[0]
    got = gpu_quant_act_nvfp4(X, gam, 1e-6, 1)
    assert (got[2].view(np.uint32)[:M] == int(rec["g_bits"], 16)).all(), [hex(v) for v in got[2].view(np.uint32)[:4]]
    ref = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, 1)
    assert_nvfp4_equal(got, ref, M, K, "golden tree row")


def test_act_nvfp4_tiny_config_outliers():
    X, _ = si.tiny_inputs(0)
    ref = oracle.quantize_nvfp4(bits(X))
    assert_nvfp4_equal(gpu_quant_act_nvfp4(X), ref, 16, 256, "tiny")


def test_act_nvfp4_edge_values():
    """Zero rows, negative zeros, rounding ties, tiny and huge magnitudes."""
    K = 256
    rows = []
    rows.append(np.zeros(K, np.float32))                                   # all-zero row: g = 0
    r = np.zeros(K, np.float32); r[::2] = -0.0; r[7] = 6.0; rows.append(r)  # -0 next to a max
    # grid midpoints relative to amax 6 -> ties in x / S
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    r = np.tile(np.concatenate([mids, -mids]), K // 16).astype(np.float32); rows.append(r)
    r = np.full(K, 1e-38, np.float32); r[3] = 3e-38; rows.append(r)         # subnormal-ish scales
    r = np.full(K, 3e38, np.float32); r[5] = -3.3e38; rows.append(r)        # near bf16 max
    r = np.zeros(K, np.float32); r[100] = 1e-3; r[200] = 1e3; rows.append(r)  # mixed block scales
    rng = np.random.default_rng(3)
    r = (rng.standard_normal(K) * np.exp2(rng.integers(-30, 30, K))).astype(np.float32); rows.append(r)
    X = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    ref = oracle.quantize_nvfp4(bits(X))
    assert_nvfp4_equal(gpu_quant_act_nvfp4(X), ref, X.shape[0], K, "edge values")


@pytest.mark.parametrize("N,K,flags", [(128, 256, 0), (300, 1024, 2), (37, 336, 0), (1, 64, 2),
                                       (513, 3584, 0)])
def test_weight_nvfp4(N, K, flags):
    W = si.projection_weight(K, N, 11)
    ref = oracle.quantize_nvfp4(bits(W), flags=flags, per_tensor=True)
    assert_nvfp4_equal(gpu_quant_weight_nvfp4(W, flags), ref, N, K, f"weight {N}x{K} f{flags}")


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("flags", [0, 3])
def test_act_fp8(M, K, flags):
    if flags and K % 64:
        pytest.skip("Hadamard needs K % 64 == 0")
    X = _inputs(M, K, 12)
    gam = si.norm_gain(K, 12)
    rc, rs = oracle.quantize_fp8(bits(X), bits(gam), 1e-6, flags)
    gc, gs = gpu_quant_fp8(X, gam, 1e-6, flags)
    bad = np.argwhere(gc != rc)
    assert bad.size == 0, f"{len(bad)} fp8 codes differ, first {bad[:4].tolist()}"
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("N,K,flags", [(128, 256, 0), (77, 1024, 2), (40, 208, 0)])
def test_weight_fp8(N, K, flags):
    W = si.projection_weight(K, N, 13)
    rc, rs = oracle.quantize_fp8(bits(W), flags=flags)
    gc, gs = gpu_quant_fp8(W, flags=flags, weight=True)
    assert np.array_equal(gc, rc)
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("flags", [0, 2, 3])
def test_act_nvfp4_stress_many_quotients(flags):
    """8M quotients (fp32-valued after the rotation): every code and scale
    bit-exact; exercises the reciprocal shortcut and its exact fallback."""
    M, K = 2048, 4096
    X = _inputs(M, K, 77 + flags)
    gam = si.norm_gain(K, 77)
    ref = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, flags)
    assert_nvfp4_equal(gpu_quant_act_nvfp4(X, gam, 1e-6, flags), ref, M, K, f"stress f{flags}")


@pytest.mark.parametrize("flags", [0, 2])
def test_act_fp8_stress_many_quotients(flags):
    M, K = 1024, 4096
    X = _inputs(M, K, 88 + flags)
    rc, rs = oracle.quantize_fp8(bits(X), flags=flags)
    gc, gs = gpu_quant_fp8(X, flags=flags)
    assert np.array_equal(gc, rc), f"{int((gc != rc).sum())} fp8 codes differ"
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32))


def test_act_nvfp4_values_near_decision_points():
    """Rows whose quotients sit on and next to every E2M1 decision point:
    amax 6 makes the block scale ~1, elements are midpoints scaled by
    1 + k/256 (bf16-representable neighbours)."""
    rows = []
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for j in range(-8, 9):
        r = np.zeros(64, np.float32)
        r[0] = 6.0
        for i, m in enumerate(mids):
            r[1 + i] = m * (1 + j / 256.0)
            r[9 + i] = -m * (1 - j / 256.0)
        rows.append(r)
    X = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    for scale in (1.0, 2.0 ** -20, 2.0 ** 20, 3.0, 0.1):
        Xs = (X.float() * scale).to(torch.bfloat16)
        ref = oracle.quantize_nvfp4(bits(Xs))
        assert_nvfp4_equal(gpu_quant_act_nvfp4(Xs), ref, Xs.shape[0], 64, f"near points x{scale}")


@pytest.mark.parametrize("M,K", [(300, 1008), (1, 3584), (129, 16), (1024, 18944)])
def test_scales_to_rowmajor_matches_oracle(M, K):
    """GPU quantizer's tiled scales, converted back to the logical row-major
    layout by vlaq_scales_to_rowmajor, equal the oracle's scales byte for
    byte (K / 16 = 63 and 1 exercise the partial last word of a row)."""
    m = vq()
    X = si.projection_activations(K, M, 61)
    xq, xs, xg = m.alloc_nvfp4(M, K)
    m.vlaq_quantize_act_nvfp4(X.cuda(), M, K, None, 1e-6, 0, xq, xs, xg)
    out = torch.full((M, K // 16), 0xAB, dtype=torch.uint8, device="cuda")
    m.vlaq_scales_to_rowmajor(xs, out, M, K)
    torch.cuda.synchronize()
    m.vlaq_check()
    _, sref, _ = oracle.quantize_nvfp4(bits(X))
    assert np.array_equal(out.cpu().numpy(), sref)


def test_scales_to_rowmajor_random_buffer():
    """Any tiled buffer: the conversion equals the layout's definition
    (test-side index math), padding dropped."""
    m = vq()
    rows, K = 257, 336
    n = layouts.scale_bytes(rows, K)
    buf = np.random.default_rng(3).integers(0, 256, n, dtype=np.uint8)
    out = torch.empty(rows, K // 16, dtype=torch.uint8, device="cuda")
    m.vlaq_scales_to_rowmajor(to_dev(buf), out, rows, K)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), layouts.untile_scales(buf, rows, K))


def _awq_like_smoothing(K, seed):
    """Per-channel factors spread like the AWQ scales the pages report for
    Qwen2.5-VL-7B (0.1553 .. 6.4375, log-uniform here)."""
    rng = np.random.default_rng(seed)
    return np.exp(rng.uniform(np.log(0.1553), np.log(6.4375), K)).astype(np.float32)


# (M, K, transform flags): ragged K (no rotation), several 64-blocks, the
# 16-warp row kernel, and full-size rows of the qkv and down inputs
SMOOTH_CASES = [(5, 336, 0), (37, 1024, 0), (37, 1024, 3), (9, 18944, 2), (1024, 3584, 3), (256, 18944, 0)]


@pytest.mark.parametrize("M,K,tf", SMOOTH_CASES)
@pytest.mark.parametrize("mode", [0, 4, 8, 12])
def test_act_nvfp4_smooth_vs_oracle(M, K, tf, mode):
    m = vq()
    X = si.projection_activations(K, M, 71)
    gam = si.norm_gain(K, 71)
    a = _awq_like_smoothing(K, 72)
    flags = tf | mode
    xq, xs, xg = m.alloc_nvfp4(M, K)
    m.vlaq_quantize_act_nvfp4_smooth(X.cuda(), M, K, gam.cuda(), to_dev(a), 1e-6, flags, xq, xs, xg)
    torch.cuda.synchronize()
    m.vlaq_check()
    ref = oracle.quantize_nvfp4_smooth(bits(X), a, bits(gam), 1e-6, flags)
    assert_nvfp4_equal((xq.cpu().numpy(), xs.cpu().numpy(), xg.cpu().numpy()), ref, M, K,
                       f"smooth M={M} K={K} flags={flags}")


# Static (calibrated) global scale: g relative to the tensor's largest
# per-token g -- equal (no saturation), far below (scales and codes
# saturate), far above (tiny and zero block scales), and absolute extremes
# that take the exact-division path for 6 g and S.
STATIC_RATIOS = [1.0, 1e-3, 0.25, 4.0, 1e6]
STATIC_ABS = [1e-30, 1e-20, 3e19, 1e36]


def _static_run(X, M, K, g, gam=None, a=None, flags=0):
    m = vq()
    xq, xs, xg = m.alloc_nvfp4(M, K)
    m.vlaq_quantize_act_nvfp4_static(X.cuda(), M, K, None if gam is None else gam.cuda(),
                                     None if a is None else to_dev(a), 1e-6, flags, g, xq, xs, xg)
    torch.cuda.synchronize()
    m.vlaq_check()
    return xq.cpu().numpy(), xs.cpu().numpy(), xg.cpu().numpy()


@pytest.mark.parametrize("M,K", [(16, 256), (130, 336), (257, 1024), (5, 18944), (3, 48), (1024, 1024)])
@pytest.mark.parametrize("ratio", STATIC_RATIOS)
def test_act_nvfp4_static_vs_oracle(M, K, ratio):
    X = _inputs(M, K, 91)
    _, _, gd = oracle.quantize_nvfp4(bits(X))
    g = float(np.float32(gd.max() * ratio))
    ref = oracle.quantize_nvfp4_static(bits(X), g)
    assert_nvfp4_equal(_static_run(X, M, K, g), ref, M, K, f"static {M}x{K} r{ratio}")


@pytest.mark.parametrize("g", STATIC_ABS)
def test_act_nvfp4_static_extreme_scales(g):
    X = _inputs(37, 1024, 92)
    ref = oracle.quantize_nvfp4_static(bits(X), g)
    assert_nvfp4_equal(_static_run(X, 37, 1024, g), ref, 37, 1024, f"static g={g}")


@pytest.mark.parametrize("M,K,tf", [(37, 1024, 3), (1024, 3584, 3), (9, 18944, 2), (64, 3584, 1)])
@pytest.mark.parametrize("mode", [None, 0, 12])
@pytest.mark.parametrize("ratio", [1.0, 0.05])
def test_act_nvfp4_static_fused_vs_oracle(M, K, tf, mode, ratio):
    X = _inputs(M, K, 93)
    gam = si.norm_gain(K, 93)
    a = None if mode is None else _awq_like_smoothing(K, 94)
    flags = tf | (mode or 0)
    if a is None:
        _, _, gd = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, tf)
    else:
        _, _, gd = oracle.quantize_nvfp4_smooth(bits(X), a, bits(gam), 1e-6, flags)
    g = float(np.float32(np.median(gd) * ratio))
    ref = oracle.quantize_nvfp4_static(bits(X), g, a, bits(gam), 1e-6, flags)
    assert_nvfp4_equal(_static_run(X, M, K, g, gam, a, flags), ref, M, K, f"static fused {M}x{K} f{flags}")


def test_act_nvfp4_static_edge_values():
    K = 256
    rows = [np.zeros(K, np.float32)]
    r = np.zeros(K, np.float32); r[::2] = -0.0; r[7] = 6.0; rows.append(r)
    r = np.full(K, 3e38, np.float32); r[5] = -3.3e38; rows.append(r)
    r = np.full(K, 1e-38, np.float32); r[3] = 3e-38; rows.append(r)
    rng = np.random.default_rng(95)
    r = (rng.standard_normal(K) * np.exp2(rng.integers(-30, 30, K))).astype(np.float32); rows.append(r)
    X = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    for g in (1.0, 1e-3, 2.0 ** -100, 1e30):
        ref = oracle.quantize_nvfp4_static(bits(X), g)
        assert_nvfp4_equal(_static_run(X, X.shape[0], K, g), ref, X.shape[0], K, f"static edge g={g}")

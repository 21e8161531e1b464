"""The 28-layer stack: 196 projections (7 unfused per layer, seed
1000 + 7 l + p for weights and activations) captured as one CUDA graph of
prologue + GEMM pairs, at prefill M = 1024 and decode M = 1, the way the
stack is timed.  On a seeded sample of entries, one per projection kind,
weight and activation codes, block scales and global scales are compared
with the oracle bit for bit in full, and GEMM outputs on sampled token rows
(one in every 128-row tile) against the relative Frobenius gate and the
element-wise bound of gpu_helpers.check_gemm; every output of every entry
must be finite.
All NVFP4, and mixed (o / down FP8 W8A8, the rest NVFP4)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from gpu_helpers import assert_nvfp4_equal, bits, check_gemm, vq

pytestmark = pytest.mark.gpu

# one entry per projection kind, at seeded layers
_rng = np.random.default_rng(5)
SAMPLE = [(int(_rng.integers(si.STACK_LAYERS)), p) for p in range(len(si.STACK_PROJECTIONS))]


@pytest.fixture(scope="module")
def weights():
    m = vq()
    import bench
    w = bench.stack_weights(m, "cuda")
    yield w
    del w
    torch.cuda.empty_cache()


def _sample_rows(M, n=16):
    rng = np.random.default_rng(M + 7)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows.update({0, M - 1})
    for t0 in range(0, M, 128):
        rows.add(int(t0 + rng.integers(0, min(128, M - t0))))
    return np.array(sorted(rows))


@pytest.mark.parametrize("M", [1024, 1])
def test_stack_in_one_graph(weights, M):
    m = vq()
    import bench
    st = bench.Stack(m, M, "cuda", weights=weights)
    assert len(st.entries) == 196
    g = bench.capture(st)
    g.replay()
    torch.cuda.synchronize()
    m.vlaq_check()
    for e in st.entries:
        assert torch.isfinite(e["Y"].float()).all(), (e["layer"], e["name"])
    for l, p in SAMPLE:
        e = st.entries[7 * l + p]
        K, N = e["K"], e["N"]
        seed = si.stack_seed(l, p)
        wref = oracle.quantize_nvfp4(bits(si.projection_weight(K, N, seed)), per_tensor=True)
        wq, ws, wg = e["W"]
        assert_nvfp4_equal((wq.cpu().numpy(), ws.cpu().numpy(), wg.cpu().numpy()), wref, N, K,
                           f"layer {l} {e['name']} W")
        xref = oracle.quantize_nvfp4(bits(si.projection_activations(K, M, seed)))
        xq, xs, xg = e["act"]
        assert_nvfp4_equal((xq.cpu().numpy(), xs.cpu().numpy(), xg.cpu().numpy()), xref, M, K,
                           f"layer {l} {e['name']} X")
        rows = _sample_rows(M)
        dx = oracle.decode_nvfp4(xref[0][rows], xref[1][rows], xref[2][rows], K)
        dw = oracle.decode_nvfp4(*wref, K, per_tensor=True)
        Y64 = oracle.linear_f64(dx, dw)
        check_gemm(e["Y"].float().cpu().numpy()[rows], Y64, dx, dw, K, None, f"stack M={M} layer {l} {e['name']}")
    del g, st
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def mixed_weights():
    m = vq()
    import bench
    w = bench.stack_weights(m, "cuda", fp8=bench.MIXED_FP8)
    yield w
    del w
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M", [1024, 1])
def test_mixed_stack_in_one_graph(mixed_weights, M):
    """The mixed-precision stack (o and down FP8 W8A8 with per-row scales,
    q/k/v/gate/up NVFP4) in one graph: FP8 codes and scales bit-exact,
    NVFP4 as above, GEMM outputs on sampled rows within the tolerance."""
    m = vq()
    import bench
    st = bench.Stack(m, M, "cuda", weights=mixed_weights, fp8=bench.MIXED_FP8)
    assert sum(e["fp8"] for e in st.entries) == 2 * si.STACK_LAYERS
    g = bench.capture(st)
    g.replay()
    torch.cuda.synchronize()
    m.vlaq_check()
    for e in st.entries:
        assert torch.isfinite(e["Y"].float()).all(), (e["layer"], e["name"])
    rows = _sample_rows(M)
    for l, p in SAMPLE:
        e = st.entries[7 * l + p]
        K, N = e["K"], e["N"]
        seed = si.stack_seed(l, p)
        Wb = bits(si.projection_weight(K, N, seed))
        Xb = bits(si.projection_activations(K, M, seed))
        if e["fp8"]:
            cw, sw = oracle.quantize_fp8(Wb)
            cx, sx = oracle.quantize_fp8(Xb)
            wq, swd = e["W"]
            xq, sxd = e["act"]
            assert np.array_equal(wq.cpu().numpy(), cw) and np.array_equal(swd.cpu().numpy().view(np.uint32),
                                                                           sw.view(np.uint32))
            assert np.array_equal(xq.cpu().numpy()[:M], cx) and np.array_equal(
                sxd.cpu().numpy()[:M].view(np.uint32), sx.view(np.uint32))
            dx, dw = oracle.decode_fp8(cx[rows], sx[rows]), oracle.decode_fp8(cw, sw)
        else:
            wref = oracle.quantize_nvfp4(Wb, per_tensor=True)
            xref = oracle.quantize_nvfp4(Xb)
            assert_nvfp4_equal(tuple(t.cpu().numpy() for t in e["W"]), wref, N, K, f"layer {l} {e['name']} W")
            assert_nvfp4_equal(tuple(t.cpu().numpy() for t in e["act"]), xref, M, K, f"layer {l} {e['name']} X")
            dx = oracle.decode_nvfp4(xref[0][rows], xref[1][rows], xref[2][rows], K)
            dw = oracle.decode_nvfp4(*wref, K, per_tensor=True)
        Y64 = oracle.linear_f64(dx, dw)
        check_gemm(e["Y"].float().cpu().numpy()[rows], Y64, dx, dw, K, None,
                   f"mixed stack M={M} layer {l} {e['name']} ({'fp8' if e['fp8'] else 'nvfp4'})")
    del g, st
    torch.cuda.empty_cache()

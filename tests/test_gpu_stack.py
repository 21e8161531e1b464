"""The 28-layer stack: 196 NVFP4 projections (7 unfused per layer, seed
1000 + 7 l + p for weights and activations) captured as one CUDA graph of
prologue + GEMM pairs, at prefill M = 1024 and decode M = 1, the way the
stack is timed.  On a seeded sample of entries, one per projection kind,
weight and activation codes, block scales and global scales are compared
with the oracle bit for bit in full, and GEMM outputs on sampled token rows
within the GEMM tolerance; every output of every entry must be finite."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from gpu_helpers import REL_FRO_TOL, assert_nvfp4_equal, bits, gemm_error, vq

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
        rel, mx = gemm_error(e["Y"].float().cpu().numpy()[rows], Y64)
        print(f"stack M={M} layer {l} {e['name']}: rel_fro={rel:.3e} max_abs={mx:.3e}")
        assert rel < REL_FRO_TOL, (l, e["name"], rel, mx)
    del g, st
    torch.cuda.empty_cache()

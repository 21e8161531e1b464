"""Pins the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something independent: values the pages
state (golden fixtures with citations), the format definitions worked by
hand, brute-force enumeration, a library routine (torch's float8_e4m3fn
cast, numpy's matmul), closed forms and exact invariants.  A plausible slip
anywhere in the oracle (a dropped factor, a wrong tie rule, a flipped
nibble, a transposed operand, a wrong Hadamard index) fails at least one.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si

def bits(t):
    return si.to_bits(t)


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def _bits_bf16(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ E2M1
E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_grid_roundtrip_golden():
    rows = list(_golden_lines("e2m1_grid.txt"))
    assert len(rows) == 16
    for code_s, val_s in rows:
        code, val = int(code_s), float(val_s)
        assert oracle.e2m1_decode(code) == val
        assert math.copysign(1.0, oracle.e2m1_decode(code)) == math.copysign(1.0, val)
        assert oracle.e2m1_encode(val) == code


def test_e2m1_ties_golden():
    for inp, exp in _golden_lines("e2m1_ties.txt"):
        assert oracle.e2m1_encode(float(inp)) == int(exp), inp


def _e2m1_brute(v: np.float32) -> int:
    """Nearest grid magnitude by enumeration; ties to the even code."""
    a = abs(float(v))
    best, best_d = None, None
    for m, mag in enumerate(E2M1_MAGS):
        d = abs(a - mag)
        if best is None or d < best_d or (d == best_d and m % 2 == 0):
            best, best_d = m, d
    if a > 6.0:
        best = 7
    sign = 8 if math.copysign(1.0, float(v)) < 0 else 0
    return sign | best


def test_e2m1_brute_force_enumeration():
    rng = np.random.default_rng(1)
    vals = list(rng.uniform(-8, 8, 4000).astype(np.float32))
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]
    for m in mids:
        for s in (1, -1):
            x = np.float32(s * m)
            vals += [x, np.nextafter(x, np.float32(0)), np.nextafter(x, np.float32(100 * s))]
    for v in vals:
        assert oracle.e2m1_encode(float(v)) == _e2m1_brute(np.float32(v)), v


def test_e2m1_monotone():
    xs = np.sort(np.random.default_rng(2).uniform(0, 10, 3000).astype(np.float32))
    dec = [oracle.e2m1_decode(oracle.e2m1_encode(float(x))) for x in xs]
    assert all(b >= a for a, b in zip(dec, dec[1:]))


# ------------------------------------------------------------------ E4M3
def _e4m3_pos_values():
    vals = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        vals.append((c, m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)))
    return vals


def test_e4m3_all_codes_roundtrip():
    for code in range(256):
        if code in (0x7F, 0xFF):
            assert math.isnan(oracle.e4m3_decode(code))
            continue
        v = oracle.e4m3_decode(code)
        assert oracle.e4m3_encode(v) == code, hex(code)


def test_e4m3_decode_matches_format_definition():
    for c, v in _e4m3_pos_values():
        assert oracle.e4m3_decode(c) == v
        assert oracle.e4m3_decode(c | 0x80) == -v
    assert oracle.e4m3_decode(0x7E) == 448.0


def test_e4m3_against_torch_float8_cast():
    rng = np.random.default_rng(3)
    mags = np.exp2(rng.uniform(-13, 10, 20000)).astype(np.float32)
    signs = np.where(rng.random(20000) < 0.5, -1, 1).astype(np.float32)
    x = mags * signs
    # every midpoint between adjacent E4M3 values, and its fp32 neighbours
    pos = [v for _, v in _e4m3_pos_values()]
    mids = [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    extra = []
    for m in mids:
        m32 = np.float32(m)
        extra += [m32, np.nextafter(m32, np.float32(0)), np.nextafter(m32, np.float32(1e9))]
    x = np.concatenate([x, np.array(extra, np.float32), -np.array(extra, np.float32)])
    clamped = np.clip(x, -448.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(clamped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode_array(x)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(float(x[i]), int(ref[i]), int(got[i])) for i in bad[:5]]


def test_e4m3_saturates():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(464.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE


def test_e4m3_brute_force_nearest_even():
    pos = _e4m3_pos_values()
    rng = np.random.default_rng(4)
    xs = np.exp2(rng.uniform(-12, 9, 3000)).astype(np.float32)
    for x in xs:
        x = float(x)
        best = min(pos, key=lambda cv: (abs(cv[1] - x), cv[0] & 1))
        assert oracle.e4m3_encode(x) == best[0], x


# ------------------------------------------------------------- NVFP4 block
def test_nvfp4_worked_block_golden():
    rec = {r[0]: r[1:] for r in _golden_lines("nvfp4_worked_block.txt")}
    x = [float(v) for v in rec["x"]]
    X = _bits_bf16(x).reshape(1, 16)
    codes, scales, g = oracle.quantize_nvfp4(X)
    exp_bytes = np.array([int(b, 16) for b in rec["bytes"]], np.uint8)
    assert np.array_equal(codes[0], exp_bytes)
    assert scales[0, 0] == int(rec["scale"][0], 16)
    num, den = float(rec["g_numerator"][0]), float(rec["g_numerator"][2])
    assert g[0] == np.float32(np.float32(num) / np.float32(den))
    # element order = golden code order, low nibble first
    exp_codes = [int(c) for c in rec["codes"]]
    unpacked = [(codes[0, j // 2] >> (4 * (j % 2))) & 0xF for j in range(16)]
    assert unpacked == exp_codes


def test_nvfp4_nibble_order_low_first():
    # Page "Feat/internvla n1 dualvln": low nibble holds the first element.
    X = _bits_bf16([6.0, 0.0] + [0.0] * 14).reshape(1, 16)
    codes, _, _ = oracle.quantize_nvfp4(X)
    assert codes[0, 0] == 0x07
    X = _bits_bf16([0.0, -6.0] + [0.0] * 14).reshape(1, 16)
    codes, _, _ = oracle.quantize_nvfp4(X)
    assert codes[0, 0] == 0xF0


def _grid_half_step(q):
    """Half the gap between the grid points that bracket |q| (|q| <= 6)."""
    a = abs(q)
    for lo, hi in zip(E2M1_MAGS, E2M1_MAGS[1:]):
        if a <= hi:
            return (hi - lo) / 2
    return 1.0


def test_nvfp4_error_bound_and_max_element():
    rng = np.random.default_rng(5)
    rows, K = 24, 512
    X = (rng.standard_normal((rows, K)) * np.exp(rng.standard_normal(K))).astype(np.float32)
    X[3, :] = 0.0                      # an all-zero row
    X[4, 17] = 1e4                     # an outlier
    Xb = _bits_bf16(X.ravel()).reshape(rows, K)
    codes, scales, g = oracle.quantize_nvfp4(Xb)
    xf = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    deq = oracle.decode_nvfp4(codes, scales, g, K)
    for r in range(rows):
        A = np.abs(xf[r]).max()
        assert g[r] == np.float32(np.float32(A) / np.float32(2688.0))
        if A == 0:
            assert not scales[r].any() and not codes[r].any()
            continue
        for b in range(K // 16):
            blk = xf[r, 16 * b:16 * b + 16]
            S = oracle.e4m3_decode(scales[r, b]) * float(g[r])
            if S == 0:
                assert not deq[r, 16 * b:16 * b + 16].any()
                continue
            for i in range(16):
                q = blk[i] / S
                err = abs(blk[i] - deq[r, 16 * b + i])
                if abs(q) <= 6.0:
                    # half a grid step times the block scale (+ fp32 rounding of q)
                    assert err <= (_grid_half_step(q) + 1e-6 * abs(q)) * S * (1 + 1e-6), (r, b, i)
                else:
                    assert abs(deq[r, 16 * b + i]) == 6.0 * S
            # the block's largest element lands on magnitude 6 when the scale is normal
            if scales[r, b] >= 0x08:
                j = int(np.argmax(np.abs(blk)))
                c = (codes[r, 8 * b + j // 2] >> (4 * (j % 2))) & 0x7
                assert c == 7, (r, b)
        # the block holding the row amax gets the top scale 448
        bmax = int(np.argmax(np.abs(xf[r]))) // 16
        assert scales[r, bmax] == 0x7E


def test_nvfp4_power_of_two_scale_invariance():
    rng = np.random.default_rng(6)
    X = rng.standard_normal((4, 256)).astype(np.float32)
    Xb = _bits_bf16(X.ravel()).reshape(4, 256)
    c0, s0, g0 = oracle.quantize_nvfp4(Xb)
    for k in (-20, -3, 5, 30):
        Xk = _bits_bf16((X.astype(np.float64) * 2.0 ** k).astype(np.float32).ravel()).reshape(4, 256)
        # bf16 rounding commutes with power-of-two scaling in the normal range
        ck, sk, gk = oracle.quantize_nvfp4(Xk)
        assert np.array_equal(c0, ck) and np.array_equal(s0, sk)
        assert np.array_equal(gk, (g0.astype(np.float64) * 2.0 ** k).astype(np.float32))


def test_nvfp4_per_tensor_global_is_max_of_rows():
    rng = np.random.default_rng(7)
    Xb = _bits_bf16(rng.standard_normal(64 * 128).astype(np.float32)).reshape(64, 128)
    _, _, g_rows = oracle.quantize_nvfp4(Xb)
    _, _, g_t = oracle.quantize_nvfp4(Xb, per_tensor=True)
    assert g_t[0] == g_rows.max()


def test_nvfp4_rejects_k_not_multiple_of_16():
    rec = dict((r[0], r[1:]) for r in _golden_lines("k3420_rejection.txt"))
    K = int(rec["K"][0])
    assert K % 16 != 0 and K / 16 == 213.75
    with pytest.raises(ValueError):
        oracle.quantize_nvfp4(np.zeros((1, K), np.uint16))
    with pytest.raises(ValueError):
        oracle.quantize_nvfp4(np.zeros((1, 96), np.uint16), flags=oracle.F_HADAMARD64)


# ------------------------------------------------------------- Hadamard
def _sylvester64():
    i = np.arange(64)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0) / 8.0


def test_wht64_equals_explicit_sylvester_matrix():
    rng = np.random.default_rng(8)
    x = rng.integers(-1000, 1000, 256).astype(np.float32)
    H = _sylvester64()
    exp = (x.reshape(4, 64).astype(np.float64) @ H.T).ravel()
    assert np.array_equal(oracle.wht64(x).astype(np.float64), exp)
    # symmetric, orthonormal
    assert np.array_equal(H, H.T)
    assert np.array_equal(H @ H, np.eye(64))


def test_wht64_involution_exact_on_integers():
    rng = np.random.default_rng(9)
    x = rng.integers(-4096, 4096, 640).astype(np.float32)
    assert np.array_equal(oracle.wht64(oracle.wht64(x)), x)


def test_rotation_leaves_product_unchanged():
    rng = np.random.default_rng(10)
    K = 512
    x = rng.standard_normal((8, K)).astype(np.float32)
    w = rng.standard_normal((16, K)).astype(np.float32)
    xr = np.stack([oracle.wht64(r) for r in x]).astype(np.float64)
    wr = np.stack([oracle.wht64(r) for r in w]).astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    rot = xr @ wr.T
    assert np.linalg.norm(rot - ref) / np.linalg.norm(ref) < 1e-5


# ------------------------------------------------------------- RMSNorm
def test_rmsnorm_against_fp64_definition():
    rng = np.random.default_rng(11)
    for K in (256, 3584, 18944):
        x = _bits_bf16((rng.standard_normal(K) * 3).astype(np.float32))
        gam = _bits_bf16(rng.uniform(0.5, 1.5, K).astype(np.float32))
        xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).double().numpy()
        gf = torch.from_numpy(gam.view(np.int16)).view(torch.bfloat16).double().numpy()
        ref = xf / np.sqrt(np.mean(xf * xf) + 1e-6) * gf
        got = oracle.transform_row(x, gam, 1e-6, oracle.F_RMSNORM).astype(np.float64)
        assert np.max(np.abs(got - ref) / np.abs(ref).max()) < 1e-6
        ss = oracle.sumsq_tree(xf.astype(np.float32))
        exact = math.fsum(xf * xf)
        # recursive-summation bound: K/32 sequential terms per lane, 5 levels
        assert abs(float(ss) - exact) <= (K / 32 + 5) * 2.0 ** -23 * exact


def test_sumsq_tree_order_exact_on_small_integers():
    # every partial sum is an integer below 2^24, so any order is exact
    x = np.arange(1, 257, dtype=np.float32) % 17
    assert float(oracle.sumsq_tree(x)) == float(np.sum(x.astype(np.float64) ** 2))


def sumsq_golden():
    """The hand-worked rows of tests/golden/sumsq_tree.txt."""
    rec = {"x": {}, "fma_x": {}}
    for r in _golden_lines("sumsq_tree.txt"):
        if r[0] in rec:
            rec[r[0]][int(r[1])] = float(r[2])
        else:
            rec[r[0]] = r[1]
    x = np.zeros(512, np.float32)
    for k, v in rec["x"].items():
        x[k] = v
    xf = np.zeros(8, np.float32)
    for k, v in rec["fma_x"].items():
        xf[k] = v
    return x, xf, rec


# Other summation orders of the same squares (fp32, one rounding per step;
# a square plus a sum is exact in fp64 for these inputs, so fp64 then one
# fp32 rounding is the fused multiply-add).
def _fma(x, acc):
    return np.float32(np.float64(x) * np.float64(x) + np.float64(acc))


def _add(a, b):
    return np.float32(np.float64(a) + np.float64(b))


def _lanes(x, chunk, owner):
    p = [np.float32(0)] * 32
    for c in range(len(x) // chunk):
        lane = owner(c)
        for e in range(chunk):
            p[lane] = _fma(x[chunk * c + e], p[lane])
    return p


def _butterfly(p, offsets=(16, 8, 4, 2, 1)):
    for o in offsets:
        p = [_add(p[l], p[l ^ o]) for l in range(32)]
    return p[0]


def _pairwise(x):
    if len(x) == 1:
        return np.float32(np.float64(x[0]) ** 2)
    h = len(x) // 2
    return _add(_pairwise(x[:h]), _pairwise(x[h:]))


def _sequential(x):
    acc = np.float32(0)
    for v in x:
        acc = _fma(v, acc)
    return acc


def _lane_order(p):
    s = np.float32(0)
    for v in p:
        s = _add(s, v)
    return s


def test_sumsq_tree_golden_row():
    """The page's tree (lane l owns 8-element chunks l, l+32, ...; fused
    multiply-add in element order; butterfly 16...1) on the hand-worked row
    gives 2^24 + 8; every other plausible order gives 2^24 + 4 or 2^24 + 12,
    so the oracle fails this test under any of them."""
    x, _, rec = sumsq_golden()
    want = np.float32(int(rec["sumsq"]))
    assert float(oracle.sumsq_tree(x)) == float(want)
    rule = _butterfly(_lanes(x, 8, lambda c: c % 32))
    assert rule == want  # the golden's own derivation
    others = {
        "sequential": _sequential(x),
        "pairwise": _pairwise(list(x)),
        "contiguous chunks per lane": _butterfly(_lanes(x, 8, lambda c: c // 2)),
        "1-element chunks": _butterfly(_lanes(x, 1, lambda c: c % 32)),
        "4-element chunks": _butterfly(_lanes(x, 4, lambda c: c % 32)),
        "16-element chunks": _butterfly(_lanes(x, 16, lambda c: c % 32)),
        "butterfly 1..16": _butterfly(_lanes(x, 8, lambda c: c % 32), (1, 2, 4, 8, 16)),
        "lane sums in lane order": _lane_order(_lanes(x, 8, lambda c: c % 32)),
        "exact, rounded once": np.float32(math.fsum(float(v) ** 2 for v in x)),
    }
    same = [k for k, v in others.items() if v == want]
    assert not same, f"the golden row does not separate the tree from {same}"


def test_sumsq_tree_golden_fused_multiply_add():
    """Inside a lane the squares accumulate with a fused multiply-add: the
    hand-worked pair gives 0x1.01f1d2p+1, a multiply then an add gives
    0x1.01f1d0p+1."""
    _, xf, rec = sumsq_golden()
    assert float(oracle.sumsq_tree(xf)) == float.fromhex(rec["fma_sum"])
    sq = np.float32(np.float64(xf[1]) ** 2)
    unfused = _add(np.float32(np.float64(xf[0]) ** 2), sq)
    assert float(unfused) != float.fromhex(rec["fma_sum"])


def test_rmsnorm_global_scale_golden_row():
    """RMSNorm (gain 1 except gain[0]) then the NVFP4 global scale of the
    golden row: the fp32 bits worked by hand in the golden file."""
    x, _, rec = sumsq_golden()
    xb = _bits_bf16(x)
    gam = np.full(512, 0x3F80, np.uint16)
    gam[0] = int(rec["gain0"], 16)
    _, _, g = oracle.quantize_nvfp4(xb[None, :], gam, 1e-6, oracle.F_RMSNORM)
    assert int(g.view(np.uint32)[0]) == int(rec["g_bits"], 16)


# ------------------------------------------------------------- FP8
def test_fp8_row_scale_and_bounds():
    rng = np.random.default_rng(12)
    X = (rng.standard_normal((6, 256)) * 5).astype(np.float32)
    X[2] = 0
    Xb = _bits_bf16(X.ravel()).reshape(6, 256)
    codes, s = oracle.quantize_fp8(Xb)
    xf = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).double().numpy()
    deq = oracle.decode_fp8(codes, s)
    for r in range(6):
        A = np.abs(xf[r]).max()
        assert s[r] == np.float32(np.float32(A) / np.float32(448.0))
        if A == 0:
            assert not codes[r].any()
            continue
        j = int(np.argmax(np.abs(xf[r])))
        assert codes[r, j] & 0x7F == 0x7E
        # relative error of E4M3 is at most 2^-4 for normal values
        big = np.abs(xf[r]) / s[r] >= 2.0 ** -6
        assert np.all(np.abs(deq[r][big] - xf[r][big]) <= 2.0 ** -4 * np.abs(xf[r][big]) + 1e-12)


# ------------------------------------------------------------- GEMM
def test_brute_force_1x16x1():
    rng = np.random.default_rng(13)
    for trial in range(20):
        x = (rng.standard_normal(16) * rng.uniform(0.01, 100)).astype(np.float32)
        w = (rng.standard_normal(16) * rng.uniform(0.01, 100)).astype(np.float32)
        xb, wb = _bits_bf16(x).reshape(1, 16), _bits_bf16(w).reshape(1, 16)
        cx, sx, gx = oracle.quantize_nvfp4(xb)
        cw, sw, gw = oracle.quantize_nvfp4(wb, per_tensor=True)
        total = Fraction(0)
        for (c, s, g, vb) in ((cx, sx, gx, xb), (cw, sw, gw, wb)):
            S = np.float32(np.float32(oracle.e4m3_decode(s[0, 0])) * g[0])
            vf = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).float().numpy()[0]
            for i in range(16):
                code = (c[0, i // 2] >> (4 * (i % 2))) & 0xF
                q = np.float32(vf[i] / S)
                assert code == _e2m1_brute(q), (trial, i)
        dx = oracle.decode_nvfp4(cx, sx, gx, 16)[0]
        dw = oracle.decode_nvfp4(cw, sw, gw, 16, per_tensor=True)[0]
        for i in range(16):
            total += Fraction(dx[i]) * Fraction(dw[i])
        y = oracle.linear_f64(dx.reshape(1, 16), dw.reshape(1, 16))[0, 0]
        assert abs(Fraction(y) - total) <= abs(total) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)


def test_linear_f64_equals_numpy_matmul_and_residual():
    rng = np.random.default_rng(14)
    M, N, K = 7, 9, 64
    Xd = rng.standard_normal((M, K))
    Wd = rng.standard_normal((N, K))
    R = _bits_bf16(rng.standard_normal(M * N).astype(np.float32)).reshape(M, N)
    Rf = torch.from_numpy(R.view(np.int16)).view(torch.bfloat16).double().numpy()
    Y = oracle.linear_f64(Xd, Wd, R)
    ref = Xd @ Wd.T + Rf
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    # transposed operand would break this for a non-square case
    rows = np.array([6, 0, 3])
    Ys = oracle.linear_f64(Xd, Wd, R, rows=rows)
    assert np.allclose(Ys, ref[rows], rtol=1e-12, atol=1e-12)


def test_decode_identity_dense_product():
    """The GEMM on codes equals the dense product of the decoded operands
    (the identity the FoldQuant dequant test checks), here with rotation."""
    rng = np.random.default_rng(15)
    M, N, K = 5, 6, 128
    X = _bits_bf16(rng.standard_normal(M * K).astype(np.float32)).reshape(M, K)
    W = _bits_bf16((rng.standard_normal(N * K) * 0.05).astype(np.float32)).reshape(N, K)
    cx, sx, gx = oracle.quantize_nvfp4(X, flags=oracle.F_HADAMARD64)
    cw, sw, gw = oracle.quantize_nvfp4(W, flags=oracle.F_HADAMARD64, per_tensor=True)
    dx = oracle.decode_nvfp4(cx, sx, gx, K)
    dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    Y = oracle.linear_f64(dx, dw)
    assert np.allclose(Y, dx @ dw.T, rtol=1e-12, atol=1e-14)
    # and it approximates the unquantized product (rotation cancels)
    xf = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).double().numpy()
    wf = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).double().numpy()
    ref = xf @ wf.T
    assert np.linalg.norm(Y - ref) / np.linalg.norm(ref) < 0.2


# ---------------------------------------------------------------- smoothing
# Per-input-channel smoothing ("FoldQuant W8A8/W4A4 inference ...", dequant
# commit: x' = R(x / a) folded before the rotation, R(x) / a after; the AWQ
# pre_quant_scale multiplies instead: "NVIDIA/TensorRT-Edge-LLM PR #193").
# Pinned against numpy's IEEE fp32 divide / multiply applied to the
# separately pinned transform steps.

def _smooth_case(K=192, seed=9):
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.standard_normal(K).astype(np.float32) * 3).to(torch.bfloat16)
    gam = torch.from_numpy((0.5 + rng.random(K)).astype(np.float32)).to(torch.bfloat16)
    a = np.exp(rng.normal(0, 1, K)).astype(np.float32)   # spread like AWQ scales
    return si.to_bits(x), si.to_bits(gam), a


@pytest.mark.parametrize("mul", [False, True])
def test_smoothing_before_rotation_is_fp32_elementwise_then_wht(mul):
    xb, gb, a = _smooth_case()
    fl = oracle.F_RMSNORM | oracle.F_HADAMARD64 | (oracle.F_SMOOTH_MUL if mul else 0)
    normed = oracle.transform_row(xb, gb, 1e-6, oracle.F_RMSNORM)
    z = (normed * a if mul else normed / a).astype(np.float32)
    want = oracle.wht64(z)
    got = oracle.transform_row_smooth(xb, a, gb, 1e-6, fl)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("mul", [False, True])
def test_smoothing_after_rotation_is_wht_then_fp32_elementwise(mul):
    xb, gb, a = _smooth_case()
    fl = oracle.F_RMSNORM | oracle.F_HADAMARD64 | oracle.F_SMOOTH_AFTER | (oracle.F_SMOOTH_MUL if mul else 0)
    rot = oracle.transform_row(xb, gb, 1e-6, oracle.F_RMSNORM | oracle.F_HADAMARD64)
    want = (rot * a if mul else rot / a).astype(np.float32)
    got = oracle.transform_row_smooth(xb, a, gb, 1e-6, fl)
    assert np.array_equal(got, want)


def test_smoothing_without_norm_or_rotation_is_one_fp32_divide():
    xb, _, a = _smooth_case(K=64)
    want = (xb.astype(np.uint32) << 16).view(np.float32) / a
    assert np.array_equal(oracle.transform_row_smooth(xb, a), want.astype(np.float32))


@pytest.mark.parametrize("flags", [0, 2, 2 | 4, 8, 2 | 8])
def test_uniform_power_of_two_smoothing_only_rescales_g(flags):
    """a = 4 everywhere: the transform scales exactly, so codes and block
    scales are unchanged and g is scaled by exactly 1/4 (x4 for multiply);
    before and after the rotation agree."""
    X = si.projection_activations(256, 6, 3)
    a = np.full(256, 4.0, np.float32)
    c0, s0, g0 = oracle.quantize_nvfp4(bits(X), flags=flags & 2)
    c1, s1, g1 = oracle.quantize_nvfp4_smooth(bits(X), a, flags=flags)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    assert np.array_equal(g1, g0 * (4.0 if flags & 8 else 0.25))


def test_unit_smoothing_is_identity():
    X = si.projection_activations(320, 5, 4)
    for fl in (0, 4, 8, 12):
        got = oracle.quantize_nvfp4_smooth(bits(X), np.ones(320, np.float32), flags=fl)
        want = oracle.quantize_nvfp4(bits(X))
        assert all(np.array_equal(u, v) for u, v in zip(got, want))


# ------------------------------------------------------------ static scale
# A calibrated activation global scale (ModelOpt / TensorRT input_scale,
# "NVIDIA/TensorRT-Edge-LLM PR #193") replaces the per-token amax; the block
# and code definitions are unchanged.  The dynamic path is pinned above, so
# equality with it at g = the row's own g transfers those pins; saturation
# and underflow are checked against the E4M3 / E2M1 definitions in fp64.

@pytest.mark.parametrize("flags,smoothed", [(0, False), (3, False), (2 | 8, True), (1 | 2 | 4, True)])
def test_static_g_equal_to_row_g_reproduces_dynamic(flags, smoothed):
    X = si.projection_activations(320, 7, 21)
    gam = si.norm_gain(320, 21)
    a = np.exp(np.random.default_rng(22).normal(0, 0.7, 320)).astype(np.float32) if smoothed else None
    if smoothed:
        c, s, g = oracle.quantize_nvfp4_smooth(bits(X), a, bits(gam), 1e-6, flags)
    else:
        c, s, g = oracle.quantize_nvfp4(bits(X), bits(gam), 1e-6, flags)
    for r in range(7):
        cs, ss, gs = oracle.quantize_nvfp4_static(bits(X)[r:r + 1], float(g[r]), a, bits(gam), 1e-6, flags)
        assert np.array_equal(cs[0], c[r]) and np.array_equal(ss[0], s[r]) and gs[0] == g[r]


def _static_check(y, codes, scales, g):
    """Block scale = E4M3(max|y| / 6 g) (saturating at 448), code =
    E2M1(y / S) with S = scale x g, checked in fp64 away from ties."""
    K = y.size
    for b in range(K // 16):
        blk = y[16 * b:16 * b + 16].astype(np.float64)
        q = np.abs(blk).max() / (6.0 * g)
        sb = scales[b]
        if q >= 464.0:
            assert sb == 0x7E
        elif q < 2.0 ** -10:
            assert sb == 0
        else:
            assert abs(oracle.e4m3_decode(sb) - q) <= q * 2.0 ** -4 + 2.0 ** -10
        S = oracle.e4m3_decode(sb) * g
        for i in range(16):
            c = (codes[8 * b + i // 2] >> (4 * (i % 2))) & 0xF
            if S == 0:
                assert c == 0
                continue
            v = blk[i] / S
            if abs(v) > 5.0 * (1 + 1e-6):
                assert c & 7 == 7 and (c >> 3) == (blk[i] < 0)
            elif abs(v) <= 5.0 * (1 - 1e-6):
                assert abs(abs(oracle.e2m1_decode(c)) - abs(v)) <= _grid_half_step(v) * (1 + 1e-6) + 1e-9


@pytest.mark.parametrize("ratio", [1e-3, 0.3, 2.0, 1e3, 1e6])
def test_static_saturation_and_rounding_definitions(ratio):
    """g well below the row's own g (values beyond the calibrated range:
    scales saturate at 448, codes at 6) and well above it (small block
    scales, down to E4M3 zero and all-zero codes)."""
    X = si.projection_activations(256, 5, 23)
    xf = (bits(X).astype(np.uint32) << 16).view(np.float32)
    _, _, gd = oracle.quantize_nvfp4(bits(X))
    g = float(np.float32(gd.max() * ratio))
    c, s, gs = oracle.quantize_nvfp4_static(bits(X), g)
    assert np.all(gs == np.float32(g))
    for r in range(5):
        _static_check(xf[r], c[r], s[r], np.float32(g))
    if ratio <= 1e-3:
        assert (s == 0x7E).mean() > 0.5
    if ratio >= 1e6:
        assert (s == 0).any() and not c[s.repeat(8, axis=1) == 0].any()


def test_static_extreme_scales_saturate_or_vanish():
    X = si.projection_activations(64, 3, 24)
    c, s, _ = oracle.quantize_nvfp4_static(bits(X), 1e-30)
    nz = np.abs((bits(X).astype(np.uint32) << 16).view(np.float32)).reshape(3, 4, 16).max(axis=2) > 0
    assert np.all(s[nz] == 0x7E)
    c, s, _ = oracle.quantize_nvfp4_static(bits(X), 1e38)   # 6 g overflows: every block scale 0
    assert not s.any() and not c.any()


# ------------------------------------------------------------------- INT8
# Symmetric per-row INT8 ("FoldQuant W8A8/W4A4 inference ...": per-row
# weight scales, per-token activations, round-half-even, clamp) and the
# exact integer GEMM with its fp32 epilogue.

def test_int8_ties_golden():
    rows = list(_golden_lines("int8_ties.txt"))
    x = [float(r[0]) for r in rows]
    want = np.array([int(r[1]) for r in rows], np.int8)
    K = 32
    X = _bits_bf16(x + [0.0] * (K - len(x))).reshape(1, K)
    codes, s = oracle.quantize_int8(X)
    assert s[0] == np.float32(1.0)
    assert np.array_equal(codes[0, :len(x)], want)


def test_int8_error_bound_max_element_and_zero_row():
    rng = np.random.default_rng(31)
    rows, K = 12, 320
    X = (rng.standard_normal((rows, K)) * np.exp(rng.standard_normal(K))).astype(np.float32)
    X[2] = 0.0
    X[5, 9] = -3e3
    Xb = _bits_bf16(X.ravel()).reshape(rows, K)
    xf = (Xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    codes, s = oracle.quantize_int8(Xb)
    deq = oracle.decode_int8(codes, s)
    for r in range(rows):
        A = np.abs(xf[r]).max()
        if A == 0:
            assert s[r] == 0 and not codes[r].any()
            continue
        assert abs(float(s[r]) - A / 127) <= A / 127 * 2.0 ** -24
        # half a step, plus the rounding of s and of the quotient
        assert np.all(np.abs(xf[r] - deq[r]) <= float(s[r]) * (0.5 + 1e-5))
        j = int(np.argmax(np.abs(xf[r])))
        assert abs(int(codes[r, j])) == 127 and np.sign(codes[r, j]) == np.sign(xf[r, j])
        assert codes[r].min() >= -127


def test_int8_power_of_two_scale_invariance():
    X = si.projection_activations(256, 4, 32)
    xf = (bits(X).astype(np.uint32) << 16).view(np.float32)
    c0, s0 = oracle.quantize_int8(bits(X))
    for k in (-40, -1, 7, 60):
        c1, s1 = oracle.quantize_int8(_bits_bf16((xf.astype(np.float64) * 2.0 ** k).ravel()).reshape(xf.shape))
        assert np.array_equal(c0, c1)
        assert np.array_equal(s1, (s0.astype(np.float64) * 2.0 ** k).astype(np.float32))


def test_int8_gemm_integer_sums_equal_numpy():
    rng = np.random.default_rng(33)
    cx = rng.integers(-127, 128, (9, 200), dtype=np.int8)
    cw = rng.integers(-127, 128, (24, 200), dtype=np.int8)
    _, acc = oracle.linear_int8(cx, np.ones(9, np.float32), cw, np.ones(24, np.float32))
    assert np.array_equal(acc, cx.astype(np.int64) @ cw.astype(np.int64).T)
    # every product at the extreme: K * 127^2 (the int32 bound the kernel relies on)
    K = 32768
    _, acc = oracle.linear_int8(np.full((1, K), -127, np.int8), np.ones(1, np.float32),
                                np.full((8, K), 127, np.int8), np.ones(8, np.float32))
    assert np.all(acc == -K * 127 * 127) and K * 127 * 127 < 2 ** 31


def test_int8_gemm_power_of_two_scales_are_exact_bf16_rounding():
    """s_x, s_w powers of two and |acc| < 2^24: t, c and t c are exact, so
    the output is torch's bf16 rounding of acc * s_x * s_w."""
    rng = np.random.default_rng(34)
    K = 512
    cx = rng.integers(-127, 128, (6, K), dtype=np.int8)
    cw = rng.integers(-127, 128, (16, K), dtype=np.int8)
    sx = np.exp2(rng.integers(-20, 5, 6)).astype(np.float32)
    sw = np.exp2(rng.integers(-20, 5, 16)).astype(np.float32)
    Y, acc = oracle.linear_int8(cx, sx, cw, sw)
    exact = acc.astype(np.float64) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.all(np.abs(acc) < 2 ** 24) and np.array_equal(Y, want)


def test_int8_gemm_residual_and_decode_identity():
    """Against the fp64 product of the decoded operands (+ residual): within
    the bf16 rounding of the output and the fp32 epilogue steps."""
    X = si.projection_activations(448, 7, 35)
    W = si.projection_weight(448, 40, 35)
    R = torch.randn(7, 40, generator=torch.Generator().manual_seed(35)).to(torch.bfloat16)
    cx, sx = oracle.quantize_int8(bits(X))
    cw, sw = oracle.quantize_int8(bits(W))
    Y, _ = oracle.linear_int8(cx, sx, cw, sw, bits(R))
    ref = oracle.linear_f64(oracle.decode_int8(cx, sx), oracle.decode_int8(cw, sw), bits(R))
    y = (Y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(y - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6 * np.abs(ref).max())


def test_int8_brute_force_1x16x1():
    """bf16 inputs -> codes -> product, against exact rationals: the code is
    the nearest integer to y / s (ties even) and the output is within one
    bf16 half-ulp (plus fp32 epilogue rounding) of the exact product."""
    rng = np.random.default_rng(36)
    for trial in range(20):
        x = _bits_bf16((rng.standard_normal(16) * 3).astype(np.float32)).reshape(1, 16)
        w = _bits_bf16((rng.standard_normal(16) * 0.1).astype(np.float32)).reshape(1, 16)
        cx, sx = oracle.quantize_int8(x)
        cw, sw = oracle.quantize_int8(w)
        for v, c, s in ((x, cx, sx), (w, cw, sw)):
            vf = (v.astype(np.uint32) << 16).view(np.float32)[0]
            for i in range(16):
                q = Fraction(float(vf[i])) / Fraction(float(s[0]))
                lo = math.floor(q)
                best = lo if (q - lo < Fraction(1, 2) or (q - lo == Fraction(1, 2) and lo % 2 == 0)) else lo + 1
                # fp32 rounding of the quotient can only move an exact tie candidate by < 2^-17 relative
                assert abs(int(c[0, i]) - best) <= (1 if abs(q - lo - Fraction(1, 2)) < abs(q) * 2 ** -22 else 0)
        Y, acc = oracle.linear_int8(cx, sx, cw, sw)
        exact = Fraction(int(acc[0, 0])) * Fraction(float(sx[0])) * Fraction(float(sw[0]))
        y = float((Y.astype(np.uint32) << 16).view(np.float32)[0, 0])
        assert abs(Fraction(y) - exact) <= abs(exact) * Fraction(1, 2 ** 8) * Fraction(1001, 1000)

"""CPU oracle for the NVFP4 / FP8 / INT8 quantize + linear path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's cpu_baseline / reference leg, never by the product package.  It
wraps the plain C file ``vlaq_oracle.c`` (built by ``oracle/build.py``) and
exchanges numpy arrays in the *logical* layouts:

* bf16 inputs as ``uint16`` arrays holding the bf16 bit patterns,
* NVFP4 codes ``uint8 [rows, K/2]`` (element k in byte k/2, low nibble first),
* NVFP4 block scales ``uint8 [rows, K/16]`` (E4M3 bytes, row-major),
* FP8 codes ``uint8 [rows, K]``, INT8 codes ``int8 [rows, K]``.

Every function cites the passage it follows in the C source's header.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

F_RMSNORM = 1
F_HADAMARD64 = 2
F_SMOOTH_AFTER = 4   # smoothing after the rotation (default: before)
F_SMOOTH_MUL = 8     # multiply by the smoothing vector (default: divide)

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from . import build as _build
        _build.build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.vo_e2m1_encode.restype = ctypes.c_uint8
    lib.vo_e2m1_encode.argtypes = [ctypes.c_float]
    lib.vo_e2m1_decode.restype = ctypes.c_double
    lib.vo_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.vo_e4m3_encode.restype = ctypes.c_uint8
    lib.vo_e4m3_encode.argtypes = [ctypes.c_float]
    lib.vo_e4m3_decode.restype = ctypes.c_double
    lib.vo_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.vo_sumsq_tree.restype = ctypes.c_float
    lib.vo_sumsq_tree.argtypes = [P, i64]
    lib.vo_wht64_inplace.restype = None
    lib.vo_wht64_inplace.argtypes = [P, i64]
    lib.vo_transform_row.restype = None
    lib.vo_transform_row.argtypes = [P, i64, P, ctypes.c_float, ctypes.c_uint, P]
    lib.vo_transform_row_smooth.restype = None
    lib.vo_transform_row_smooth.argtypes = [P, i64, P, ctypes.c_float, ctypes.c_uint, P, P]
    lib.vo_quantize_nvfp4_smooth.restype = ctypes.c_int
    lib.vo_quantize_nvfp4_smooth.argtypes = [P, i64, i64, P, ctypes.c_float, ctypes.c_uint, P, P, P, P]
    lib.vo_quantize_nvfp4_static.restype = ctypes.c_int
    lib.vo_quantize_nvfp4_static.argtypes = [P, i64, i64, P, ctypes.c_float, ctypes.c_uint, P, ctypes.c_float,
                                             P, P, P]
    lib.vo_quantize_nvfp4.restype = ctypes.c_int
    lib.vo_quantize_nvfp4.argtypes = [P, i64, i64, P, ctypes.c_float, ctypes.c_uint,
                                      ctypes.c_int, P, P, P]
    lib.vo_decode_nvfp4.restype = None
    lib.vo_decode_nvfp4.argtypes = [P, P, P, i64, i64, ctypes.c_int, P]
    lib.vo_quantize_fp8.restype = ctypes.c_int
    lib.vo_quantize_fp8.argtypes = [P, i64, i64, P, ctypes.c_float, ctypes.c_uint, P, P]
    lib.vo_decode_fp8.restype = None
    lib.vo_decode_fp8.argtypes = [P, P, i64, i64, P]
    lib.vo_quantize_int8.restype = ctypes.c_int
    lib.vo_quantize_int8.argtypes = [P, i64, i64, P, ctypes.c_float, ctypes.c_uint, P, P]
    lib.vo_decode_int8.restype = None
    lib.vo_decode_int8.argtypes = [P, P, i64, i64, P]
    lib.vo_linear_int8.restype = None
    lib.vo_linear_int8.argtypes = [P, P, P, P, P, i64, i64, i64, P, i64, P, P]
    lib.vo_linear_f64.restype = None
    lib.vo_linear_f64.argtypes = [P, P, P, i64, i64, i64, P, i64, P]
    lib.vo_num_threads.restype = ctypes.c_int
    lib.vo_num_threads.argtypes = []
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------ element codecs
def e2m1_encode(v: float) -> int:
    return int(_load().vo_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(_load().vo_e2m1_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(_load().vo_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(_load().vo_e4m3_decode(int(code)))


def e2m1_encode_array(v) -> np.ndarray:
    lib = _load()
    v = np.asarray(v, dtype=np.float32).ravel()
    return np.array([lib.vo_e2m1_encode(float(x)) for x in v], dtype=np.uint8)


def e4m3_encode_array(v) -> np.ndarray:
    lib = _load()
    v = np.asarray(v, dtype=np.float32).ravel()
    return np.array([lib.vo_e4m3_encode(float(x)) for x in v], dtype=np.uint8)


# ------------------------------------------------------------ row transforms
def sumsq_tree(x) -> np.float32:
    x = _c(x, np.float32)
    return np.float32(_load().vo_sumsq_tree(_ptr(x), x.size))


def wht64(y) -> np.ndarray:
    y = _c(y, np.float32).copy()
    _load().vo_wht64_inplace(_ptr(y), y.size)
    return y


def transform_row(x_bf16, gamma_bf16=None, eps=1e-6, flags=0) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    g = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    y = np.empty(x.size, dtype=np.float32)
    _load().vo_transform_row(_ptr(x), x.size, _ptr(g), ctypes.c_float(eps), flags, _ptr(y))
    return y


def transform_row_smooth(x_bf16, smooth_f32, gamma_bf16=None, eps=1e-6, flags=0) -> np.ndarray:
    """transform_row with per-input-channel smoothing (fp32 [K])."""
    x = _c(x_bf16, np.uint16)
    a = _c(smooth_f32, np.float32)
    g = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    y = np.empty(x.size, dtype=np.float32)
    _load().vo_transform_row_smooth(_ptr(x), x.size, _ptr(g), ctypes.c_float(eps), flags, _ptr(a), _ptr(y))
    return y


# ------------------------------------------------------------------- NVFP4
def quantize_nvfp4(X_bf16, gamma_bf16=None, eps=1e-6, flags=0, per_tensor=False):
    """Returns (codes u8 [rows, K/2], scales u8 [rows, K/16], g f32 [rows] or [1])."""
    X = _c(X_bf16, np.uint16)
    rows, K = X.shape
    g_in = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros((rows, max(K // 16, 1)), dtype=np.uint8)
    g = np.zeros(1 if per_tensor else rows, dtype=np.float32)
    rc = _load().vo_quantize_nvfp4(_ptr(X), rows, K, _ptr(g_in), ctypes.c_float(eps), flags,
                                   1 if per_tensor else 0, _ptr(codes), _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError(f"oracle refused NVFP4 quantization of K={K} flags={flags}")
    return codes, scales, g


def quantize_nvfp4_smooth(X_bf16, smooth_f32, gamma_bf16=None, eps=1e-6, flags=0):
    """Per-token NVFP4 of activations smoothed per input channel: (codes,
    scales, g) as quantize_nvfp4."""
    X = _c(X_bf16, np.uint16)
    rows, K = X.shape
    a = _c(smooth_f32, np.float32)
    assert a.size == K
    g_in = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros((rows, max(K // 16, 1)), dtype=np.uint8)
    g = np.zeros(rows, dtype=np.float32)
    rc = _load().vo_quantize_nvfp4_smooth(_ptr(X), rows, K, _ptr(g_in), ctypes.c_float(eps), flags, _ptr(a),
                                          _ptr(codes), _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError(f"oracle refused smoothed NVFP4 quantization of K={K} flags={flags}")
    return codes, scales, g


def quantize_nvfp4_static(X_bf16, g_static, smooth_f32=None, gamma_bf16=None, eps=1e-6, flags=0):
    """Activations with a static global scale g_static (fp32) for every row;
    optional per-channel smoothing.  Returns (codes, scales, g) as
    quantize_nvfp4 (g = g_static per row)."""
    X = _c(X_bf16, np.uint16)
    rows, K = X.shape
    a = None if smooth_f32 is None else _c(smooth_f32, np.float32)
    g_in = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros((rows, max(K // 16, 1)), dtype=np.uint8)
    g = np.zeros(rows, dtype=np.float32)
    rc = _load().vo_quantize_nvfp4_static(_ptr(X), rows, K, _ptr(g_in), ctypes.c_float(eps), flags, _ptr(a),
                                          ctypes.c_float(g_static), _ptr(codes), _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError(f"oracle refused static NVFP4 quantization of K={K} flags={flags}")
    return codes, scales, g


def decode_nvfp4(codes, scales, g, K, per_tensor=False) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    g = _c(g, np.float32)
    rows = codes.shape[0]
    out = np.empty((rows, K), dtype=np.float64)
    _load().vo_decode_nvfp4(_ptr(codes), _ptr(scales), _ptr(g), rows, K,
                            1 if per_tensor else 0, _ptr(out))
    return out


# --------------------------------------------------------------------- FP8
def quantize_fp8(X_bf16, gamma_bf16=None, eps=1e-6, flags=0):
    """Returns (codes u8 [rows, K], s f32 [rows])."""
    X = _c(X_bf16, np.uint16)
    rows, K = X.shape
    g_in = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    codes = np.zeros((rows, K), dtype=np.uint8)
    s = np.zeros(rows, dtype=np.float32)
    rc = _load().vo_quantize_fp8(_ptr(X), rows, K, _ptr(g_in), ctypes.c_float(eps), flags,
                                 _ptr(codes), _ptr(s))
    if rc != 0:
        raise ValueError(f"oracle refused FP8 quantization of K={K} flags={flags}")
    return codes, s


def decode_fp8(codes, s) -> np.ndarray:
    codes = _c(codes, np.uint8)
    s = _c(s, np.float32)
    rows, K = codes.shape
    out = np.empty((rows, K), dtype=np.float64)
    _load().vo_decode_fp8(_ptr(codes), _ptr(s), rows, K, _ptr(out))
    return out


# -------------------------------------------------------------------- INT8
def quantize_int8(X_bf16, gamma_bf16=None, eps=1e-6, flags=0):
    """Symmetric per-row INT8: returns (codes i8 [rows, K], s f32 [rows])."""
    X = _c(X_bf16, np.uint16)
    rows, K = X.shape
    g_in = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    codes = np.zeros((rows, K), dtype=np.int8)
    s = np.zeros(rows, dtype=np.float32)
    rc = _load().vo_quantize_int8(_ptr(X), rows, K, _ptr(g_in), ctypes.c_float(eps), flags, _ptr(codes), _ptr(s))
    if rc != 0:
        raise ValueError(f"oracle refused INT8 quantization of K={K} flags={flags}")
    return codes, s


def decode_int8(codes, s) -> np.ndarray:
    codes = _c(codes, np.int8)
    s = _c(s, np.float32)
    rows, K = codes.shape
    out = np.empty((rows, K), dtype=np.float64)
    _load().vo_decode_int8(_ptr(codes), _ptr(s), rows, K, _ptr(out))
    return out


def linear_int8(cx, sx, cw, sw, residual_bf16=None, rows=None):
    """INT8 GEMM + epilogue for the selected rows: returns (Y bf16 bits
    uint16 [nrows, N], exact integer sums int64 [nrows, N])."""
    cx = _c(cx, np.int8)
    cw = _c(cw, np.int8)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    M, K = cx.shape
    N = cw.shape[0]
    res = None if residual_bf16 is None else _c(residual_bf16, np.uint16)
    idx = None if rows is None else _c(rows, np.int64)
    nrows = M if rows is None else len(idx)
    Y = np.zeros((nrows, N), dtype=np.uint16)
    acc = np.zeros((nrows, N), dtype=np.int64)
    _load().vo_linear_int8(_ptr(cx), _ptr(sx), _ptr(cw), _ptr(sw), _ptr(res), M, N, K, _ptr(idx), nrows, _ptr(Y),
                           _ptr(acc))
    return Y, acc


# -------------------------------------------------------------------- GEMM
def linear_f64(Xd, Wd, residual_bf16=None, rows=None) -> np.ndarray:
    """fp64 Y = Xd[rows] @ Wd.T (+ residual[rows]) with sums in k order."""
    Xd = _c(Xd, np.float64)
    Wd = _c(Wd, np.float64)
    M, K = Xd.shape
    N = Wd.shape[0]
    res = None if residual_bf16 is None else _c(residual_bf16, np.uint16)
    if rows is None:
        idx = None
        nrows = M
    else:
        idx = _c(rows, np.int64)
        nrows = idx.size
    Y = np.empty((nrows, N), dtype=np.float64)
    _load().vo_linear_f64(_ptr(Xd), _ptr(Wd), _ptr(res), M, N, K, _ptr(idx), nrows, _ptr(Y))
    return Y


def num_threads() -> int:
    return int(_load().vo_num_threads())

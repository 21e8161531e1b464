"""Python binding of libvlaq (include/vlaq.h): argument marshalling only.

Every function named ``vlaq_*`` forwards to the C entry point of the same
name; tensors are passed as raw device pointers (``data_ptr()``) and the
stream is the current torch CUDA stream unless one is given.  All work runs
in the CUDA library: there is no CPU fallback, and importing this package
fails loudly if ``libvlaq.so`` has not been built.

The ``alloc_*`` helpers allocate output buffers with torch (the library
itself never allocates) in the sizes the header prescribes.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "VlaqError", "F_RMSNORM", "F_HADAMARD64", "F_SMOOTH_AFTER", "F_SMOOTH_MUL", "LIB_PATH",
    "vlaq_last_error", "vlaq_version", "vlaq_check",
    "vlaq_nvfp4_code_pitch", "vlaq_nvfp4_scale_bytes", "vlaq_linear_workspace_bytes",
    "vlaq_quantize_weight_nvfp4", "vlaq_quantize_act_nvfp4", "vlaq_linear_nvfp4",
    "vlaq_quantize_act_nvfp4_smooth", "vlaq_quantize_act_nvfp4_static", "vlaq_scales_to_rowmajor",
    "vlaq_selftest_wait_timeout",
    "vlaq_quantize_weight_fp8", "vlaq_quantize_act_fp8", "vlaq_linear_fp8", "vlaq_linear_nvfp4_noalloc",
    "vlaq_quantize_weight_int8", "vlaq_quantize_act_int8", "vlaq_linear_int8",
    "alloc_nvfp4", "alloc_fp8", "alloc_int8", "alloc_workspace",
]

F_RMSNORM = 1
F_HADAMARD64 = 2
F_SMOOTH_AFTER = 4
F_SMOOTH_MUL = 8

STATUS_NAMES = {
    0: "VLAQ_OK", 1: "VLAQ_ERR_INVALID_ARG", 2: "VLAQ_ERR_SHAPE", 3: "VLAQ_ERR_ALIGN",
    4: "VLAQ_ERR_ARCH", 5: "VLAQ_ERR_CUDA", 6: "VLAQ_ERR_TIMEOUT", 7: "VLAQ_ERR_WORKSPACE",
}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvlaq.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libvlaq.so is not built ({LIB_PATH}); run `python -m vlaq_quantize_act_b200.build`. "
        "There is no fallback path.")
_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_U32 = ctypes.c_uint32
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGS = {
    "vlaq_last_error": (ctypes.c_char_p, []),
    "vlaq_version": (ctypes.c_int, []),
    "vlaq_check": (ctypes.c_int, [_P]),
    "vlaq_nvfp4_code_pitch": (_I64, [_I64]),
    "vlaq_nvfp4_scale_bytes": (_I64, [_I64, _I64]),
    "vlaq_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "vlaq_quantize_weight_nvfp4": (ctypes.c_int, [_P, _I64, _I64, _U32, _P, _P, _P, _P]),
    "vlaq_quantize_act_nvfp4": (ctypes.c_int, [_P, _I64, _I64, _P, _F, _U32, _P, _P, _P, _P]),
    "vlaq_linear_nvfp4": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "vlaq_quantize_weight_fp8": (ctypes.c_int, [_P, _I64, _I64, _U32, _P, _P, _P]),
    "vlaq_quantize_act_fp8": (ctypes.c_int, [_P, _I64, _I64, _P, _F, _U32, _P, _P, _P]),
    "vlaq_linear_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "vlaq_quantize_weight_int8": (ctypes.c_int, [_P, _I64, _I64, _U32, _P, _P, _P]),
    "vlaq_quantize_act_int8": (ctypes.c_int, [_P, _I64, _I64, _P, _F, _U32, _P, _P, _P]),
    "vlaq_linear_int8": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "vlaq_linear_nvfp4_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "vlaq_scales_to_rowmajor": (ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    "vlaq_selftest_wait_timeout": (ctypes.c_int, [_P]),
    "vlaq_quantize_act_nvfp4_smooth": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _F, _U32, _P, _P, _P, _P]),
    "vlaq_quantize_act_nvfp4_static": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _F, _U32, _F, _P, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class VlaqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status
        self.message = message


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return stream


def _check(status: int):
    if status != 0:
        raise VlaqError(status, _lib.vlaq_last_error().decode())


# ----------------------------------------------------------- plain queries
def vlaq_last_error() -> str:
    return _lib.vlaq_last_error().decode()


def vlaq_version() -> int:
    return _lib.vlaq_version()


def vlaq_check(stream=None) -> None:
    _check(_lib.vlaq_check(_stream(stream)))


def vlaq_nvfp4_code_pitch(K: int) -> int:
    return _lib.vlaq_nvfp4_code_pitch(K)


def vlaq_nvfp4_scale_bytes(rows: int, K: int) -> int:
    return _lib.vlaq_nvfp4_scale_bytes(rows, K)


def vlaq_linear_workspace_bytes(M: int, N: int, K: int) -> int:
    return _lib.vlaq_linear_workspace_bytes(M, N, K)


# ----------------------------------------------------------------- NVFP4
def vlaq_quantize_weight_nvfp4(W, N, K, flags, codes, scales, g_w, stream=None):
    _check(_lib.vlaq_quantize_weight_nvfp4(_ptr(W), N, K, flags, _ptr(codes), _ptr(scales), _ptr(g_w),
                                           _stream(stream)))


def vlaq_quantize_act_nvfp4(X, M, K, gamma, eps, flags, codes, scales, g_x, stream=None):
    _check(_lib.vlaq_quantize_act_nvfp4(_ptr(X), M, K, _ptr(gamma), eps, flags, _ptr(codes), _ptr(scales),
                                        _ptr(g_x), _stream(stream)))


def vlaq_quantize_act_nvfp4_smooth(X, M, K, gamma, smooth, eps, flags, codes, scales, g_x, stream=None):
    _check(_lib.vlaq_quantize_act_nvfp4_smooth(_ptr(X), M, K, _ptr(gamma), _ptr(smooth), eps, flags, _ptr(codes),
                                               _ptr(scales), _ptr(g_x), _stream(stream)))


def vlaq_quantize_act_nvfp4_static(X, M, K, gamma, smooth, eps, flags, g_static, codes, scales, g_x, stream=None):
    _check(_lib.vlaq_quantize_act_nvfp4_static(_ptr(X), M, K, _ptr(gamma), _ptr(smooth), eps, flags, g_static,
                                               _ptr(codes), _ptr(scales), _ptr(g_x), _stream(stream)))


def vlaq_selftest_wait_timeout(stream=None):
    _check(_lib.vlaq_selftest_wait_timeout(_stream(stream)))


def vlaq_scales_to_rowmajor(scales, out, rows, K, stream=None):
    _check(_lib.vlaq_scales_to_rowmajor(_ptr(scales), _ptr(out), rows, K, _stream(stream)))


def vlaq_linear_nvfp4(xq, xs, g_x, wq, ws, g_w, residual, Y, M, N, K, workspace=None, ws_bytes=0,
                      stream=None):
    _check(_lib.vlaq_linear_nvfp4(_ptr(xq), _ptr(xs), _ptr(g_x), _ptr(wq), _ptr(ws), _ptr(g_w), _ptr(residual),
                                  _ptr(Y), M, N, K, _ptr(workspace), ws_bytes, _stream(stream)))


def vlaq_linear_nvfp4_noalloc(xq, xs, g_x, wq, ws, g_w, residual, Y, M, N, K, stream=None):
    """vlaq_linear_nvfp4 for callers that cannot allocate: no workspace; the
    split-K scratch is a fixed 4 MiB array inside the library (see vlaq.h)."""
    _check(_lib.vlaq_linear_nvfp4_noalloc(_ptr(xq), _ptr(xs), _ptr(g_x), _ptr(wq), _ptr(ws), _ptr(g_w),
                                          _ptr(residual), _ptr(Y), M, N, K, _stream(stream)))


# ------------------------------------------------------------------- FP8
def vlaq_quantize_weight_fp8(W, N, K, flags, codes, s_w, stream=None):
    _check(_lib.vlaq_quantize_weight_fp8(_ptr(W), N, K, flags, _ptr(codes), _ptr(s_w), _stream(stream)))


def vlaq_quantize_act_fp8(X, M, K, gamma, eps, flags, codes, s_x, stream=None):
    _check(_lib.vlaq_quantize_act_fp8(_ptr(X), M, K, _ptr(gamma), eps, flags, _ptr(codes), _ptr(s_x),
                                      _stream(stream)))


def vlaq_linear_fp8(xq, s_x, wq, s_w, residual, Y, M, N, K, workspace=None, ws_bytes=0, stream=None):
    _check(_lib.vlaq_linear_fp8(_ptr(xq), _ptr(s_x), _ptr(wq), _ptr(s_w), _ptr(residual), _ptr(Y), M, N, K,
                                _ptr(workspace), ws_bytes, _stream(stream)))


# ------------------------------------------------------------------ INT8
def vlaq_quantize_weight_int8(W, N, K, flags, codes, s_w, stream=None):
    _check(_lib.vlaq_quantize_weight_int8(_ptr(W), N, K, flags, _ptr(codes), _ptr(s_w), _stream(stream)))


def vlaq_quantize_act_int8(X, M, K, gamma, eps, flags, codes, s_x, stream=None):
    _check(_lib.vlaq_quantize_act_int8(_ptr(X), M, K, _ptr(gamma), eps, flags, _ptr(codes), _ptr(s_x),
                                       _stream(stream)))


def vlaq_linear_int8(xq, s_x, wq, s_w, residual, Y, M, N, K, workspace=None, ws_bytes=0, stream=None):
    _check(_lib.vlaq_linear_int8(_ptr(xq), _ptr(s_x), _ptr(wq), _ptr(s_w), _ptr(residual), _ptr(Y), M, N, K,
                                 _ptr(workspace), ws_bytes, _stream(stream)))


# ------------------------------------------------------ buffer allocation
def alloc_nvfp4(rows: int, K: int, device="cuda", per_tensor: bool = False):
    """(codes u8 [rows, pitch], tiled scales u8 [scale_bytes], g f32 [rows or 1])."""
    pitch = vlaq_nvfp4_code_pitch(K)
    codes = torch.empty(max(rows, 1), pitch, dtype=torch.uint8, device=device)
    scales = torch.empty(max(vlaq_nvfp4_scale_bytes(max(rows, 1), K), 16), dtype=torch.uint8, device=device)
    g = torch.empty(1 if per_tensor else max(rows, 1), dtype=torch.float32, device=device)
    return codes, scales, g


def alloc_fp8(rows: int, K: int, device="cuda"):
    """(codes u8 [rows, K], scale f32 [rows])."""
    return (torch.empty(max(rows, 1), K, dtype=torch.uint8, device=device),
            torch.empty(max(rows, 1), dtype=torch.float32, device=device))


def alloc_int8(rows: int, K: int, device="cuda"):
    """(codes int8 [rows, K], scale f32 [rows])."""
    return (torch.empty(max(rows, 1), K, dtype=torch.int8, device=device),
            torch.empty(max(rows, 1), dtype=torch.float32, device=device))


def alloc_workspace(M: int, N: int, K: int, device="cuda"):
    """(workspace tensor or None, bytes) for vlaq_linear_*, allocated zeroed:
    the NVFP4 split-K tile counters must start at zero (every call leaves
    them zero again)."""
    n = vlaq_linear_workspace_bytes(M, N, K)
    if n == 0:
        return None, 0
    return torch.zeros((n + 15) // 16 * 16, dtype=torch.uint8, device=device), n

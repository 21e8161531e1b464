"""Test-side statement of the library's public buffer layouts (from the
format description in include/vlaq.h), used to compare the CUDA path's
tiled scales and padded codes with the oracle's logical layouts.
Pure index arithmetic; no quantization."""
import numpy as np


def code_pitch(K: int) -> int:
    return (K + 63) // 64 * 32


def scale_offsets(rows: int, K: int) -> np.ndarray:
    """Byte offset of scale (r, j) in the 128x4 tiled layout, [rows, K/16]."""
    cp = (K + 63) // 64 * 4
    r = np.arange(rows, dtype=np.int64)[:, None]
    j = np.arange(K // 16, dtype=np.int64)[None, :]
    return ((r // 128) * (cp // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)


def scale_bytes(rows: int, K: int) -> int:
    return (rows + 127) // 128 * 128 * ((K + 63) // 64 * 4)


def untile_scales(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return np.asarray(buf).reshape(-1)[scale_offsets(rows, K)]


def padded_scale_offsets(rows: int, K: int) -> np.ndarray:
    """Offsets of the padding columns j in [K/16, Cp) of real rows."""
    cp = (K + 63) // 64 * 4
    if cp == K // 16:
        return np.zeros(0, np.int64)
    r = np.arange(rows, dtype=np.int64)[:, None]
    j = np.arange(K // 16, cp, dtype=np.int64)[None, :]
    return (((r // 128) * (cp // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)).ravel()


def tile_scales(rowmajor: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.zeros(scale_bytes(rows, K), np.uint8)
    out[scale_offsets(rows, K)] = rowmajor
    return out


def pad_codes(codes: np.ndarray, K: int) -> np.ndarray:
    rows = codes.shape[0]
    out = np.zeros((rows, code_pitch(K)), np.uint8)
    out[:, : K // 2] = codes
    return out

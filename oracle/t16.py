"""ctypes front end of the scalar C oracle (``t16_oracle.c``) -- test infrastructure.

Source of the arithmetic: "DeepSeek-V4.1-Flash-1017 · dsx T16" model card, section
"How T16 works", item 1 (T16 codebook: multiply the 16-bit window by 0x3A2F and add
the product's two bytes) and item 2 (column-major positions in a 16x16 tile).  The
bit order, window origin, tail-biting, centring and tile order are the readings
written at the top of ``t16_oracle.c``.
"""
import ctypes
import numpy as np

from . import build_oracle

_lib = None


def lib():
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.oracle_window.argtypes = [u32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64]
        L.oracle_window.restype = ctypes.c_uint32
        L.oracle_t16.argtypes = [ctypes.c_uint32]
        L.oracle_t16.restype = ctypes.c_int
        L.oracle_code.argtypes = [ctypes.c_uint32]
        L.oracle_code.restype = ctypes.c_int
        L.oracle_decode_stream.argtypes = [u32p, ctypes.c_int64, ctypes.c_int, i32p]
        L.oracle_decode_stream.restype = None
        L.oracle_decode_tile.argtypes = [u32p, ctypes.c_int, i32p]
        L.oracle_decode_tile.restype = None
        L.oracle_decode_rows.argtypes = [u32p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                         i64p, ctypes.c_int64, i32p]
        L.oracle_decode_rows.restype = ctypes.c_int
        L.oracle_decode_matrix.argtypes = [u32p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                           i32p]
        L.oracle_decode_matrix.restype = ctypes.c_int
        _lib = L
    return _lib


def _u32(a):
    a = np.ascontiguousarray(a, dtype=np.uint32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32))


def t16_value(window: int) -> int:
    """T16 codebook value t (0..510) of one 16-bit window."""
    return int(lib().oracle_t16(int(window) & 0xFFFFFFFF))


def code(window: int) -> int:
    """Centred code c = t - 255 of one 16-bit window."""
    return int(lib().oracle_code(int(window) & 0xFFFFFFFF))


def window(words, n_bits: int, K: int, p: int) -> int:
    """16-bit window of position p in a tail-biting stream of n_bits bits."""
    a, ptr = _u32(words)
    return int(lib().oracle_window(ptr, n_bits, K, p))


def decode_stream(words, n: int, K: int) -> np.ndarray:
    """Codes of the n positions of a tail-biting stream of n*K bits."""
    a, ptr = _u32(words)
    assert a.size * 32 >= n * K
    out = np.empty(n, dtype=np.int32)
    lib().oracle_decode_stream(ptr, n, K, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    return out


def decode_tile(tile_words, K: int) -> np.ndarray:
    """Codes [16, 16] (row, column) of one tile of 8*K words."""
    a, ptr = _u32(tile_words)
    assert a.size == 8 * K
    out = np.empty((16, 16), dtype=np.int32)
    lib().oracle_decode_tile(ptr, K, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    return out


def decode_matrix(bits, K: int, rows: int, cols: int) -> np.ndarray:
    """Codes [rows, cols] of a bit stream laid out as row-major 16x16 tiles."""
    a, ptr = _u32(bits)
    assert a.size == (rows // 16) * (cols // 16) * 8 * K
    out = np.empty((rows, cols), dtype=np.int32)
    rc = lib().oracle_decode_matrix(ptr, K, rows, cols,
                                    out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if rc:
        raise ValueError("oracle_decode_matrix: bad arguments (%d)" % rc)
    return out


def decode_rows(bits, K: int, rows: int, cols: int, row_ids) -> np.ndarray:
    """Codes [len(row_ids), cols] of selected rows of a tiled bit stream."""
    a, ptr = _u32(bits)
    assert a.size == (rows // 16) * (cols // 16) * 8 * K
    ids = np.ascontiguousarray(row_ids, dtype=np.int64)
    out = np.empty((ids.size, cols), dtype=np.int32)
    rc = lib().oracle_decode_rows(ptr, K, rows, cols,
                                  ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), ids.size,
                                  out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if rc:
        raise ValueError("oracle_decode_rows: bad arguments (%d)" % rc)
    return out

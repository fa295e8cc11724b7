"""CPU oracle for MoE token dispatch and combine (ctypes front end).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library.  The arithmetic lives in
``moe_oracle.c`` (plain single-threaded C, built by ``make -C oracle``); this
file only converts numpy arrays to pointers and allocates outputs.

All functions take and return numpy arrays; bf16 data travels as raw uint16
bits, E4M3 data as uint8 codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_DIR, "moe_oracle.c")
# MOE_ORACLE_LIB names a prebuilt oracle library to load instead (the
# mutation tests point it at deliberately broken copies)
_LIB = os.environ.get("MOE_ORACLE_LIB") or os.path.join(_DIR, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

TILE = 128
OK, ERR_INVALID_ARG, ERR_EXPERT_RANGE, ERR_DUPLICATE_EXPERT, ERR_CAPACITY = 0, 1, 2, 3, 4

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(dtype=np.uint32, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int


def build() -> str:
    """Compile the oracle if its library is missing or older than its source."""
    if os.environ.get("MOE_ORACLE_LIB"):
        return _LIB
    with _lock:
        if (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            subprocess.run(["make", "-s", "-C", _DIR], check=True)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    lib.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_decode.restype = ctypes.c_double
    lib.oracle_bf16_encode.argtypes = [ctypes.c_double]
    lib.oracle_bf16_encode.restype = ctypes.c_uint16
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_padded_capacity.argtypes = [_i64, _int, _int]
    lib.oracle_padded_capacity.restype = _i64
    lib.oracle_layout.argtypes = [_i32p, _i64, _int, _int, _int, _i32p, _i32p, _i32p, _i32p,
                                  _i32p, _i32p, _i64]
    lib.oracle_layout.restype = _int
    lib.oracle_permute_rows.argtypes = [_vp, _i64, _i64, _i64, _i32p, _int, _i32p, _i32p, _int,
                                        _vp]
    lib.oracle_permute_rows.restype = None
    lib.oracle_combine.argtypes = [_u16p, _i64, _i32p, _f32p, _vp, _i64, _int, _u16p]
    lib.oracle_combine.restype = None
    lib.oracle_combine_bwd.argtypes = [_u16p, _u16p, _i64, _f32p, _i32p, _i32p, _i32p, _int,
                                       _i64, _int, _u16p, _f32p]
    lib.oracle_combine_bwd.restype = None
    lib.oracle_dispatch_bwd.argtypes = [_u16p, _i64, _i32p, _i64, _int, _u16p]
    lib.oracle_dispatch_bwd.restype = None
    lib.oracle_quantize_e4m3.argtypes = [_u16p, _i64, _i64, _i64, _u8p, _f32p]
    lib.oracle_quantize_e4m3.restype = _int
    lib.oracle_dequantize_e4m3.argtypes = [_u8p, _f32p, _i64, _i64, _f32p]
    lib.oracle_dequantize_e4m3.restype = None
    lib.oracle_tile_checksums.argtypes = [_vp, _i64, _vp, _i64, _i64, _u32p]
    lib.oracle_tile_checksums.restype = None
    _lib = lib
    return lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def bf16_decode(bits: int) -> float:
    return _load().oracle_bf16_decode(int(bits))


def bf16_encode(v: float) -> int:
    return int(_load().oracle_bf16_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return _load().oracle_e4m3_decode(int(code))


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def padded_capacity(T: int, K: int, E: int) -> int:
    return int(_load().oracle_padded_capacity(T, K, E))


# --------------------------------------------------------------------------
# dispatch
# --------------------------------------------------------------------------
class Layout:
    __slots__ = ("status", "counts", "offsets", "rank_counts", "rank_offsets", "dst_row",
                 "row_src", "P", "P_cap")

    def __repr__(self):
        return f"Layout(status={self.status}, P={self.P}, P_cap={self.P_cap})"


def layout(ids: np.ndarray, E: int, R: int, P_cap: int | None = None) -> Layout:
    ids = _c(ids, np.int32)
    T, K = ids.shape
    if P_cap is None:
        P_cap = padded_capacity(T, K, E)
    L = Layout()
    L.counts = np.zeros(E, np.int32)
    L.offsets = np.zeros(E + 1, np.int32)
    L.rank_counts = np.zeros(R, np.int32)
    L.rank_offsets = np.zeros(R + 1, np.int32)
    L.dst_row = np.zeros(T * K, np.int32)
    L.row_src = np.zeros(max(P_cap, 1), np.int32)
    L.status = _load().oracle_layout(ids.reshape(-1), T, K, E, R, L.counts, L.offsets,
                                     L.rank_counts, L.rank_offsets, L.dst_row, L.row_src,
                                     P_cap)
    L.row_src = L.row_src[:P_cap]
    L.P = int(L.offsets[E])
    L.P_cap = P_cap
    return L


def permute_rows(x: np.ndarray, dst_row: np.ndarray, K: int, counts: np.ndarray,
                 offsets: np.ndarray, xp: np.ndarray) -> np.ndarray:
    """Byte-exact scatter of the rows of ``x`` (2-D, any dtype, rows may be strided)
    into ``xp`` (2-D, same dtype and row length, contiguous), in place."""
    assert x.ndim == 2 and xp.ndim == 2 and x.dtype == xp.dtype and x.shape[1] == xp.shape[1]
    assert xp.flags.c_contiguous and x.strides[1] == x.itemsize
    T = x.shape[0]
    row_bytes = x.shape[1] * x.itemsize
    _load().oracle_permute_rows(x.ctypes.data_as(_vp), T, row_bytes, x.strides[0],
                                _c(dst_row, np.int32), K, _c(counts, np.int32),
                                _c(offsets, np.int32), len(counts), xp.ctypes.data_as(_vp))
    return xp


# --------------------------------------------------------------------------
# combine and the backward calls
# --------------------------------------------------------------------------
def combine(y: np.ndarray, dst_row: np.ndarray, scales: np.ndarray,
            shared: np.ndarray | None = None) -> np.ndarray:
    y = _c(y, np.uint16)
    scales = _c(scales, np.float32)
    T, K = scales.shape
    H = y.shape[1]
    out = np.empty((T, H), np.uint16)
    sh = None
    if shared is not None:
        shared = _c(shared, np.uint16)
        sh = shared.ctypes.data_as(_vp)
    _load().oracle_combine(y, H, _c(dst_row, np.int32), scales, sh, T, K, out)
    return out


def combine_bwd(g: np.ndarray, y: np.ndarray, scales: np.ndarray, dst_row: np.ndarray,
                counts: np.ndarray, offsets: np.ndarray, grad_y: np.ndarray):
    """Fills ``grad_y`` (uint16 [P_cap, H], in place) and returns grad_scales [T, K]."""
    g = _c(g, np.uint16)
    y = _c(y, np.uint16)
    scales = _c(scales, np.float32)
    T, K = scales.shape
    H = g.shape[1]
    assert grad_y.dtype == np.uint16 and grad_y.flags.c_contiguous
    gs = np.empty((T, K), np.float32)
    _load().oracle_combine_bwd(g, y, H, scales, _c(dst_row, np.int32), _c(counts, np.int32),
                               _c(offsets, np.int32), len(counts), T, K, grad_y, gs)
    return gs


def dispatch_bwd(grad_xp: np.ndarray, dst_row: np.ndarray, T: int, K: int) -> np.ndarray:
    grad_xp = _c(grad_xp, np.uint16)
    H = grad_xp.shape[1]
    out = np.empty((T, H), np.uint16)
    _load().oracle_dispatch_bwd(grad_xp, H, _c(dst_row, np.int32), T, K, out)
    return out


# --------------------------------------------------------------------------
# FP8
# --------------------------------------------------------------------------
def quantize_e4m3(x: np.ndarray):
    x = _c(x, np.uint16)
    T, H = x.shape
    q = np.empty((T, H), np.uint8)
    s = np.empty((T, H // 128), np.float32)
    st = _load().oracle_quantize_e4m3(x, T, H, H, q, s)
    if st != OK:
        raise ValueError("H must be a multiple of 128")
    return q, s


def dequantize_e4m3(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = _c(q, np.uint8)
    s = _c(s, np.float32)
    T, H = q.shape
    out = np.empty((T, H), np.float32)
    _load().oracle_dequantize_e4m3(q, s, T, H, out)
    return out


def tile_checksums(xp: np.ndarray, n_tiles: int, xs: np.ndarray | None = None) -> np.ndarray:
    assert xp.flags.c_contiguous
    row_bytes = xp.shape[1] * xp.itemsize
    out = np.zeros(n_tiles, np.uint32)
    if xs is not None:
        assert xs.flags.c_contiguous
        sp, sb = xs.ctypes.data_as(_vp), xs.shape[1] * xs.itemsize
    else:
        sp, sb = None, 0
    _load().oracle_tile_checksums(xp.ctypes.data_as(_vp), row_bytes, sp, sb, n_tiles, out)
    return out

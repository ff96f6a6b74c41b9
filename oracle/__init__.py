"""Plain CPU oracle for factorized causal self-attention (Sparse Transformer).

TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package; the CUDA library never
does, and this package never imports the library.

The arithmetic lives in ``oracle.cpp`` (C++17, fp64, OpenMP), built into
``liboracle.so`` by :func:`build`. This module only marshals numpy arrays.
Index-set definitions and their sources are listed at the top of
``oracle.cpp``; ``reference_np.py`` holds a second, numpy-only restatement
used on tiny sizes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC_PATH = os.path.join(HERE, "oracle.cpp")

STRIDED, FIXED, DENSE_CAUSAL = 0, 1, 2
SPLIT, MERGED = 0, 1
KIND = {"strided": STRIDED, "fixed": FIXED, "dense": DENSE_CAUSAL}
MODE = {"split": SPLIT, "merged": MERGED}

_lib = None
_i64 = ctypes.c_int64
_P = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile liboracle.so with g++ (-O2, OpenMP) if it is missing or stale."""
    stale = (not os.path.exists(LIB_PATH)
             or os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC_PATH))
    if force or stale:
        tmp = LIB_PATH + ".tmp"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, SRC_PATH])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        L.orc_max_threads.restype = ctypes.c_int
        L.orc_row_set.restype = _i64
        L.orc_row_set.argtypes = [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, _i64, _P, _i64]
        L.orc_nnz.restype = _i64
        L.orc_nnz.argtypes = [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, _i64]
        common = [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, _i64, _i64, _i64, ctypes.c_double]
        L.orc_forward.restype = None
        L.orc_forward.argtypes = common + [_P, _P, _P, _P, _P, ctypes.c_int]
        L.orc_forward_rows.restype = None
        L.orc_forward_rows.argtypes = common + [_P, _P, _P, _i64, _P, _P, _P, _P, ctypes.c_int]
        L.orc_backward.restype = None
        L.orc_backward.argtypes = common + [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int]
        L.orc_backward_query_rows.restype = None
        L.orc_backward_query_rows.argtypes = common + [_P, _P, _P, _P, _i64, _P, _P, _P, ctypes.c_int]
        L.orc_backward_key_rows.restype = None
        L.orc_backward_key_rows.argtypes = common + [_P, _P, _P, _P, _i64, _P, _P, _P, _P,
                                                     ctypes.c_int]
        L.orc_num_head_classes.restype = ctypes.c_int
        L.orc_num_head_classes.argtypes = [ctypes.c_int, ctypes.c_int]
        L.orc_num_segments.restype = ctypes.c_int
        L.orc_num_segments.argtypes = [ctypes.c_int, ctypes.c_int]
        L.orc_segment_views.restype = None
        L.orc_segment_views.argtypes = [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, ctypes.c_int,
                                        ctypes.c_int, _P, _P]
        L.orc_layout_tiles.restype = _i64
        L.orc_layout_tiles.argtypes = [ctypes.c_int, ctypes.c_int, _i64, _i64, _i64, ctypes.c_int,
                                       ctypes.c_int, _P, _P, _P, _i64]
        _lib = L
    return _lib


def _k(kind):
    return KIND[kind] if isinstance(kind, str) else int(kind)


def _m(mode):
    return MODE[mode] if isinstance(mode, str) else int(mode)


def _f32(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(lib().orc_max_threads())


def row_set(kind, mode, l, c, h, i) -> np.ndarray:
    """The sorted index set S_{h,i} (int64)."""
    cap = int(i) + 1
    out = np.zeros(cap, dtype=np.int64)
    n = lib().orc_row_set(_k(kind), _m(mode), int(l), int(c), int(h), int(i), _ptr(out), cap)
    return out[:n].copy()


def nnz(kind, mode, T, l, c, h) -> int:
    """Number of live (i, j) pairs of head h (sum of |S_{h,i}|)."""
    return int(lib().orc_nnz(_k(kind), _m(mode), int(T), int(l), int(c), int(h)))


def _scale(scale, d):
    return float(scale) if scale and scale > 0 else 1.0 / float(np.sqrt(d))


def forward(kind, mode, q, k, v, l, c, scale=None, threads=0):
    """Returns (O [B,H,T,d] float64, LSE [B,H,T] float64) for all rows."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, d = q.shape
    o = np.zeros((B, H, T, d), dtype=np.float64)
    lse = np.zeros((B, H, T), dtype=np.float64)
    lib().orc_forward(_k(kind), _m(mode), B, H, T, d, int(l), int(c), _scale(scale, d),
                      _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(threads))
    return o, lse


def forward_rows(kind, mode, q, k, v, l, c, bh, rows, scale=None, threads=0):
    """O and LSE for the listed rows: row r is (bh[r], rows[r]) with bh = b*H + h."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, d = q.shape
    bh = np.ascontiguousarray(bh, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = len(rows)
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    lib().orc_forward_rows(_k(kind), _m(mode), B, H, T, d, int(l), int(c), _scale(scale, d),
                           _ptr(q), _ptr(k), _ptr(v), n, _ptr(bh), _ptr(rows), _ptr(o), _ptr(lse),
                           int(threads))
    return o, lse


def backward(kind, mode, q, k, v, dout, l, c, scale=None, threads=0):
    """Returns (dQ, dK, dV), each [B,H,T,d] float64, with P recomputed."""
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, H, T, d = q.shape
    dq = np.zeros((B, H, T, d), dtype=np.float64)
    dk = np.zeros_like(dq)
    dv = np.zeros_like(dq)
    lib().orc_backward(_k(kind), _m(mode), B, H, T, d, int(l), int(c), _scale(scale, d),
                       _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                       int(threads))
    return dq, dk, dv


def backward_query_rows(kind, mode, q, k, v, dout, l, c, bh, rows, scale=None, threads=0):
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, H, T, d = q.shape
    bh = np.ascontiguousarray(bh, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = len(rows)
    dq = np.zeros((n, d), dtype=np.float64)
    lib().orc_backward_query_rows(_k(kind), _m(mode), B, H, T, d, int(l), int(c),
                                  _scale(scale, d), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), n,
                                  _ptr(bh), _ptr(rows), _ptr(dq), int(threads))
    return dq


def backward_key_rows(kind, mode, q, k, v, dout, l, c, bh, keys, scale=None, threads=0):
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, H, T, d = q.shape
    bh = np.ascontiguousarray(bh, dtype=np.int64)
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    n = len(keys)
    dk = np.zeros((n, d), dtype=np.float64)
    dv = np.zeros((n, d), dtype=np.float64)
    lib().orc_backward_key_rows(_k(kind), _m(mode), B, H, T, d, int(l), int(c),
                                _scale(scale, d), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), n,
                                _ptr(bh), _ptr(keys), _ptr(dk), _ptr(dv), int(threads))
    return dk, dv


def num_head_classes(kind, mode) -> int:
    return int(lib().orc_num_head_classes(_k(kind), _m(mode)))


def num_segments(kind, mode) -> int:
    return int(lib().orc_num_segments(_k(kind), _m(mode)))


def segment_views(kind, mode, T, l, c, hc, seg):
    qv = ctypes.c_int(0)
    kv = ctypes.c_int(0)
    lib().orc_segment_views(_k(kind), _m(mode), int(T), int(l), int(c), int(hc), int(seg),
                            ctypes.byref(qv), ctypes.byref(kv))
    return qv.value, kv.value


def layout_tiles(kind, mode, T, l, c, hc, seg):
    """(qtile, ktile, live) int64 arrays of one segment, sorted by (qtile, ktile).

    seg = -1 gives the plain natural-order 128 x 128 tiling of the whole set."""
    L = lib()
    n = L.orc_layout_tiles(_k(kind), _m(mode), int(T), int(l), int(c), int(hc), int(seg),
                           None, None, None, 0)
    qt = np.zeros(n, dtype=np.int64)
    kt = np.zeros(n, dtype=np.int64)
    live = np.zeros(n, dtype=np.int64)
    L.orc_layout_tiles(_k(kind), _m(mode), int(T), int(l), int(c), int(hc), int(seg),
                       _ptr(qt), _ptr(kt), _ptr(live), n)
    return qt, kt, live

"""fp64 CPU oracle for block-sparse spatio-temporal attention (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()`` and by the
bench's CPU-baseline leg. The product path (the CUDA library and its binding) never imports
it. See ``svg_oracle.c`` for the definitions and the passages each routine follows.

Parity status of each routine (what pins it, in tests/test_oracle_pins.py):
  or_keep / or_retained_pairs   pinned: closed-form retained counts, sink invariant
  or_tile_counts                pinned: interval-derived tile classes (tiny + pages' shape rows)
  or_rounded_class              pinned: rounded == exact where no tile is boundary; hand cases
  or_attention_rows             pinned: Q=0 => mean of kept V; all-kept == textbook softmax;
                                        V=1 => O=1 (rows sum to 1); LSE(Q=0) = ln(#kept);
                                        numpy brute force with an explicit N x N mask
  or_perm_table                 pinned: bijection, closed-form positions of corner tokens
  or_route_errors               pinned: masks equal to dense give zero error; constant V gives a
                                        tie; planted spatial / temporal structure is recovered
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svg_oracle.c")
_LIB = os.path.join(_HERE, "libsvgoracle.so")

ROUTE_SPATIAL, ROUTE_TEMPORAL = 0, 1
LAYOUT_SINK_PREFIX, LAYOUT_FULL_SPACE_MAJOR = 0, 1
MASK_EXACT, MASK_ROUNDED, MASK_ALL = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp). Building the checker is not using it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, u32p, u8p = ctypes.c_int64, ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint8)
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.or_position.restype = i64
        L.or_position.argtypes = [ctypes.c_int, ctypes.c_int, i64, i64, i64, i64, i64]
        L.or_perm_table.argtypes = [ctypes.c_int, ctypes.c_int, i64, i64, i64, i64p]
        L.or_inverse_table.argtypes = [ctypes.c_int, ctypes.c_int, i64, i64, i64, i64p]
        L.or_keep.restype = ctypes.c_int
        L.or_keep.argtypes = [ctypes.c_int, i64, i64, i64, i64, i64, i64]
        L.or_tile_counts.argtypes = [ctypes.c_int, ctypes.c_int, i64, i64, i64, i64, i64, i64, i64,
                                     i64p, i64, u32p, u8p]
        L.or_rounded_class.restype = ctypes.c_uint8
        L.or_rounded_class.argtypes = [ctypes.c_uint32, i64]
        L.or_retained_pairs.restype = ctypes.c_uint64
        L.or_retained_pairs.argtypes = [ctypes.c_int, i64, i64, i64, i64, i64]
        L.or_attention_rows.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, i64, i64,
                                        ctypes.c_double, ctypes.c_int, ctypes.c_int, i64, i64, i64, i64,
                                        i64, ctypes.c_int, ctypes.c_void_p, i64, i64, i64p, i64,
                                        ctypes.c_void_p, ctypes.c_void_p]
        L.or_num_threads.restype = ctypes.c_int
        L.or_route_errors.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, i64, i64, ctypes.c_double,
                                      i64, i64, i64, i64, i64, i64p, i64, ctypes.c_void_p]
        _lib = L
    return _lib


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    return int(lib().or_num_threads())


def position(route, layout, T, S, F0, t, s) -> int:
    return int(lib().or_position(route, layout, T, S, F0, t, s))


def perm_table(route, layout, T, S, F0) -> np.ndarray:
    """pi[i] = position of original token i in the head's token order."""
    pi = np.empty(T * S, dtype=np.int64)
    lib().or_perm_table(route, layout, T, S, F0, _p(pi, ctypes.c_int64))
    return pi


def inverse_table(route, layout, T, S, F0) -> np.ndarray:
    inv = np.empty(T * S, dtype=np.int64)
    lib().or_inverse_table(route, layout, T, S, F0, _p(inv, ctypes.c_int64))
    return inv


def keep(route, S, k, b, F0, i, j) -> int:
    return int(lib().or_keep(route, S, k, b, F0, i, j))


def tile_counts(route, layout, T, S, k, b, F0, bq, bk, qts=None):
    """Brute-force (count, class) arrays of shape [len(qts), nk] for the listed q-tiles."""
    N = T * S
    nq, nk = -(-N // bq), -(-N // bk)
    qts = np.arange(nq, dtype=np.int64) if qts is None else np.ascontiguousarray(qts, dtype=np.int64)
    cnt = np.empty((len(qts), nk), dtype=np.uint32)
    cls = np.empty((len(qts), nk), dtype=np.uint8)
    lib().or_tile_counts(route, layout, T, S, k, b, F0, bq, bk, _p(qts, ctypes.c_int64), len(qts),
                         _p(cnt, ctypes.c_uint32), _p(cls, ctypes.c_uint8))
    return cnt, cls


def tile_areas(N, bq, bk, qts=None) -> np.ndarray:
    """In-range area of each (qt, kt) tile."""
    nq, nk = -(-N // bq), -(-N // bk)
    qts = np.arange(nq) if qts is None else np.asarray(qts)
    rows = np.minimum(N, (qts + 1) * bq) - qts * bq
    kts = np.arange(nk)
    cols = np.minimum(N, (kts + 1) * bk) - kts * bk
    return rows[:, None].astype(np.int64) * cols[None, :].astype(np.int64)


def rounded_classes(counts: np.ndarray, areas: np.ndarray) -> np.ndarray:
    """Apply the oracle's rounding rule tile by tile."""
    f = lib().or_rounded_class
    out = np.empty(counts.shape, dtype=np.uint8)
    for idx in np.ndindex(counts.shape):
        out[idx] = f(int(counts[idx]), int(areas[idx]))
    return out


def retained_pairs(route, T, S, k, b, F0) -> int:
    return int(lib().or_retained_pairs(route, T, S, k, b, F0))


def attention_rows(q, k, v, rows, *, route, layout, T, S, frame_window, band, F0, scale=None,
                   mask_kind=MASK_EXACT, rcls=None, bq=1, bk=1):
    """fp64 masked softmax attention for the listed original query rows of ONE head.

    q, k, v: bf16 tensors/arrays [N, d] in original token order (torch bf16 or np.uint16 bits).
    Returns (out [n_rows, d] float64, lse [n_rows] float64)."""
    def bits(x):
        try:
            import torch
            if isinstance(x, torch.Tensor):
                return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))
        except ImportError:  # pragma: no cover
            pass
        return np.ascontiguousarray(x, dtype=np.uint16)
    qb, kb, vb = bits(q), bits(k), bits(v)
    N, d = qb.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((len(rows), d), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d)
    rc = None
    if mask_kind == MASK_ROUNDED:
        rc = np.ascontiguousarray(rcls, dtype=np.uint8)
    lib().or_attention_rows(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, N, d, float(scale),
                            route, layout, T, S, frame_window, band, F0, mask_kind,
                            rc.ctypes.data if rc is not None else None, bq, bk,
                            _p(rows, ctypes.c_int64), len(rows), out.ctypes.data, lse.ctypes.data)
    return out, lse


def _bits(x):
    import torch
    if isinstance(x, torch.Tensor):
        return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))
    return np.ascontiguousarray(x, dtype=np.uint16)


def route_errors(q, k, v, rows, *, T, S, frame_window, band, F0, scale=None):
    """(E_spatial, E_temporal, E_dense) of one head over the sampled original rows (fp64)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    N, d = qb.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty(3, dtype=np.float64)
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(d)
    lib().or_route_errors(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, N, d, float(scale), T, S, frame_window,
                          band, F0, _p(rows, ctypes.c_int64), len(rows), out.ctypes.data)
    return float(out[0]), float(out[1]), float(out[2])


def route(q, k, v, rows, **kw) -> int:
    es, et, _ = route_errors(q, k, v, rows, **kw)
    return ROUTE_SPATIAL if es <= et else ROUTE_TEMPORAL

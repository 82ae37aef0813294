"""ORACLE — TEST INFRASTRUCTURE ONLY.

A plain, slow CPU statement of what prefix-sliding attention over a ring-buffer
KV cache computes, used to check the CUDA library.  Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import it; the library never
does, and this package imports nothing from the library.

- ``attention.c`` (float64): the pages' reference model, masked softmax
  attention over an explicit history list (blog section 2.1; digest section 03
  visibility rule).
- ``listmodel.py``: the cache's list and ring models (blog sections 2.3-3.4).

Every function here is pinned by ``tests/test_oracle_*.py`` to facts that do not
come from this code: hand-derived golden cases, closed forms, special cases that
reduce to a textbook routine, and brute force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import listmodel  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "attention.c")
_lib = None


def build(force: bool = False) -> str:
    """Compile attention.c (gcc -O2, no fast-math) into liboracle.so."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _SO, _SRC,
                               "-lm", "-lpthread"])
    return _SO


class _Problem(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int64), ("W", ctypes.c_int64), ("t", ctypes.c_int64),
                ("scale", ctypes.c_double), ("G", ctypes.c_int32), ("d", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("nh", ctypes.c_int64), ("hpos", ctypes.c_void_p),
                ("hk", ctypes.c_void_p), ("hv", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("nvis", ctypes.c_int64)]


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.oracle_is_visible.restype = ctypes.c_int
        lib.oracle_is_visible.argtypes = [ctypes.c_int64] * 4
        lib.oracle_visible_mask.restype = None
        lib.oracle_visible_mask.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_void_p]
        lib.oracle_attend.restype = ctypes.c_int64
        lib.oracle_attend.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p]
        lib.oracle_attend_many.restype = None
        lib.oracle_attend_many.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int64, ctypes.c_int]
        _lib = lib
    return _lib


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def is_visible(P: int, W: int, t: int, p: int) -> bool:
    return bool(_load().oracle_is_visible(P, W, t, p))


def visible_mask(P: int, W: int, t: int, p0: int, n: int) -> np.ndarray:
    m = np.empty(max(n, 0), np.uint8)
    if n > 0:
        _load().oracle_visible_mask(P, W, t, p0, n, m.ctypes.data)
    return m.astype(bool)


def visible_positions(P: int, W: int, t: int) -> np.ndarray:
    """All visible positions for the query at t, by testing every p in [0, t]."""
    return np.nonzero(visible_mask(P, W, t, 0, t + 1))[0].astype(np.int64)


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def attend(P: int, W: int, t: int, scale: float, q, hist_pos, hist_k, hist_v) -> np.ndarray:
    """Masked softmax attention of q ([G][d]) over history rows (positions
    [nh], keys/values [nh][d]); float64 [G][d]."""
    q = _f64(q)
    G, d = q.shape
    hp = np.ascontiguousarray(hist_pos, dtype=np.int64)
    hk = _f64(hist_k)
    hv = _f64(hist_v)
    nh = hp.shape[0]
    assert hk.shape == (nh, d) and hv.shape == (nh, d)
    out = np.empty((G, d), np.float64)
    z = np.empty(max(nh, 1), np.float64)
    nvis = _load().oracle_attend(P, W, t, scale, G, d, q.ctypes.data, nh, hp.ctypes.data,
                                 hk.ctypes.data, hv.ctypes.data, out.ctypes.data, z.ctypes.data)
    if nvis == 0:
        raise ValueError("no visible row in the history given")
    return out


class Batch:
    """A set of independent problems solved on host threads by attend_many."""

    def __init__(self):
        self._probs = []
        self._keep = []

    def add(self, P, W, t, scale, q, hist_pos, hist_k, hist_v) -> np.ndarray:
        q = _f64(q)
        G, d = q.shape
        hp = np.ascontiguousarray(hist_pos, dtype=np.int64)
        hk = _f64(hist_k)
        hv = _f64(hist_v)
        nh = hp.shape[0]
        assert hk.shape == (nh, d) and hv.shape == (nh, d)
        out = np.empty((G, d), np.float64)
        self._keep += [q, hp, hk, hv, out]
        self._probs.append((int(P), int(W), int(t), float(scale), G, d, q, nh, hp, hk, hv, out))
        return out

    def run(self, nthreads: int | None = None) -> None:
        n = len(self._probs)
        arr = (_Problem * max(n, 1))()
        for i, (P, W, t, scale, G, d, q, nh, hp, hk, hv, out) in enumerate(self._probs):
            arr[i] = _Problem(P, W, t, scale, G, d, q.ctypes.data, nh, hp.ctypes.data,
                              hk.ctypes.data, hv.ctypes.data, out.ctypes.data, 0)
        _load().oracle_attend_many(arr, n, nthreads or host_threads())
        for i in range(n):
            if arr[i].nvis == 0:
                raise ValueError(f"problem {i}: no visible row in the history given")

"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds no attention or cache arithmetic.  It maps coordinates
(seed, tensor id, sequence, head, position, channel) to N(0,1) samples with a
counter-based hash (SplitMix64 + Box-Muller, see ``gen.c``), so any row of any
history position can be regenerated independently of every other row.

Values are produced as float32 (``dtype="f32"``) or as bfloat16 bit patterns
(``dtype="bf16"``, uint16, round-to-nearest-even from the float32 value).
``to_f64`` widens either form to float64 exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "gen.c")

# Tensor ids: one independent stream per kind of input.
TID_Q = 1
TID_K = 2
TID_V = 3
TID_KSCALE = 4
TID_PLEN = 5
TID_TLEN = 6
TID_HEAD = 7
TID_QBLK = 8

_lib = None


def build(force: bool = False) -> str:
    """Compile gen.c into libsynth.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-o", _SO, _SRC, "-lm", "-lpthread"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                     ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_uniform_int.restype = ctypes.c_int64
        lib.synth_uniform_int.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                          ctypes.c_int64, ctypes.c_int64]
        lib.synth_fill_rows.restype = None
        lib.synth_fill_rows.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                        ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int]
        lib.synth_f32_to_bf16.restype = None
        lib.synth_f32_to_bf16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
        _lib = lib
    return _lib


def _nthreads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def normal(seed: int, tid: int, seq: int, head: int, pos: int, dim: int) -> float:
    """One N(0,1) sample (float64) at the given coordinates."""
    return _load().synth_normal(seed, tid, seq, head, pos, dim)


def uniform_int(seed: int, tid: int, index: int, lo: int, hi: int) -> int:
    """Uniform integer in [lo, hi] (inclusive) for draw `index` of stream `tid`."""
    return int(_load().synth_uniform_int(seed, tid, index, lo, hi))


def rows(seed: int, tid: int, seq: int, H: int, pos0: int, npos: int, d: int,
         dtype: str = "f32", chan_scale: np.ndarray | None = None) -> np.ndarray:
    """Rows for positions [pos0, pos0+npos) of one sequence, token-major [npos][H][d].

    Returns float32 values (dtype "f32") or bfloat16 bit patterns as uint16
    (dtype "bf16").  ``chan_scale`` ([H][d] float64) multiplies each sample
    before the float32 rounding.
    """
    lib = _load()
    shape = (int(npos), int(H), int(d))
    f32 = np.empty(shape, np.float32) if dtype == "f32" else None
    b16 = np.empty(shape, np.uint16) if dtype == "bf16" else None
    if dtype not in ("f32", "bf16"):
        raise ValueError(dtype)
    cs = None
    if chan_scale is not None:
        cs = np.ascontiguousarray(chan_scale, dtype=np.float64)
        assert cs.shape == (H, d)
    if npos > 0:
        lib.synth_fill_rows(seed, tid, seq, H, pos0, npos, d,
                            None if cs is None else cs.ctypes.data,
                            None if f32 is None else f32.ctypes.data,
                            None if b16 is None else b16.ctypes.data, _nthreads())
    return f32 if dtype == "f32" else b16


def chan_scale(seed: int, H: int, d: int) -> np.ndarray:
    """Per (head, channel) log-normal(0,1) multipliers, float64 [H][d]."""
    z = rows(seed, TID_KSCALE, 0, H, 0, 1, d, "f32")[0].astype(np.float64)
    return np.exp(z)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (round to nearest even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().synth_f32_to_bf16(x.ctypes.data, out.ctypes.data, x.size)
    return out


def to_f64(x: np.ndarray) -> np.ndarray:
    """Widen float32 values or bfloat16 bit patterns (uint16) to float64, exactly."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)

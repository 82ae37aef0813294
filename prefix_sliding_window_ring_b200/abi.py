"""Python binding of the C ABI in include/ps.h (argument marshalling only).

Every ``ps_*`` function here calls the function of the same name in
``libps.so`` and raises ``PSError`` on a non-zero status.  Device arguments may
be torch tensors (their ``data_ptr()`` is passed) or integer addresses; host
index arrays may be any integer sequence.  ``stream`` defaults to torch's
current CUDA stream.  There is no fallback: if the library is missing, importing
this module fails.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libps.so")

PS_OK, PS_EINVAL, PS_ENOMEM, PS_EPOS, PS_ESTATE, PS_ECUDA, PS_EUNSUPPORTED = 0, -1, -2, -3, -4, -5, -6
PS_F32, PS_BF16 = 0, 1
STATUS_NAMES = {0: "PS_OK", -1: "PS_EINVAL", -2: "PS_ENOMEM", -3: "PS_EPOS", -4: "PS_ESTATE",
                -5: "PS_ECUDA", -6: "PS_EUNSUPPORTED"}

# Every entry point declared in include/ps.h: name -> (restype, argtypes)
_vp, _i, _i64, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float


class SeqInfo(ctypes.Structure):
    _fields_ = [("state", ctypes.c_int32), ("P", ctypes.c_int32), ("next_pos", ctypes.c_int64),
                ("head", ctypes.c_int32), ("count", ctypes.c_int32)]


SIGNATURES = {
    "ps_cache_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "ps_cache_bytes_paged": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "ps_cache_create_paged": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp,
                                   ctypes.POINTER(_vp)]),
    "ps_ring_pages_free": (_i, [_vp]),
    "ps_cache_create": (_i, [_i, _i, _i, _i, _i, _i, _vp, _sz, _vp, ctypes.POINTER(_vp)]),
    "ps_cache_destroy": (None, [_vp]),
    "ps_seq_reset": (_i, [_vp, _i, _i, _vp]),
    "ps_seq_info_get": (_i, [_vp, _i, ctypes.POINTER(SeqInfo)]),
    "ps_prefill_prefix": (_i, [_vp, _i, _vp, _vp, _i, _vp]),
    "ps_append_kv": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp]),
    "ps_decode_workspace_bytes": (_sz, [_vp, _i, _i]),
    "ps_attend_decode": (_i, [_vp, _vp, _vp, _vp, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "ps_attend_decode_static": (_i, [_vp, _vp, _vp, _vp, _i, _i, _f, _vp, _vp]),
    "ps_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp, _vp, _sz, _vp]),
    "ps_attend_chunk": (_i, [_vp, _i, _vp, _vp, _vp, _i64, _i, _i, _f, _vp, _i, _vp]),
    "ps_set_chunk_small_max": (_i, [_vp, _i]),
    "ps_attend_prompt": (_i, [_vp, _i, _vp, _i64, _i, _i, _f, _vp, _vp]),
    "ps_attend_chunk_batch": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _f, _vp, _i, _vp]),
    "ps_attend_prompt_batch": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _f, _vp, _vp]),
    "ps_share_prefix": (_i, [_vp, _i, _i, _vp]),
    "ps_debug_wait_timeout": (_i, [_vp, ctypes.c_longlong, _vp]),
    "ps_export_window": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "ps_import_window": (_i, [_vp, _i, _i64, _vp, _vp, _i, _i, _vp]),
    "ps_debug_visible": (_i, [_vp, _i, _i64, _vp, _vp, _vp]),
    "ps_device_error": (_i, [_vp, ctypes.POINTER(ctypes.c_int32), _vp]),
    "ps_last_error": (ctypes.c_char_p, []),
    "ps_version": (ctypes.c_char_p, []),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python prefix_sliding_window_ring_b200/build.py`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


class PSError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code
        self.fn = fn


def _check(fn: str, rc: int) -> None:
    if rc != PS_OK:
        raise PSError(fn, rc, _lib.ps_last_error().decode())


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _ints(seq, ctype):
    vals = [int(v) for v in seq]
    return (ctype * max(1, len(vals)))(*vals), len(vals)


def ps_version() -> str:
    return _lib.ps_version().decode()


def ps_last_error() -> str:
    return _lib.ps_last_error().decode()


def ps_cache_bytes(W, P_max, Hkv, d, dtype, max_seqs) -> int:
    return int(_lib.ps_cache_bytes(W, P_max, Hkv, d, dtype, max_seqs))


def ps_cache_create(W, P_max, Hkv, d, dtype, max_seqs, dev_buf, dev_bytes, stream=None):
    h = _vp()
    _check("ps_cache_create", _lib.ps_cache_create(W, P_max, Hkv, d, dtype, max_seqs, _ptr(dev_buf),
                                                   dev_bytes, _stream(stream), ctypes.byref(h)))
    return h


def ps_cache_bytes_paged(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages) -> int:
    return int(_lib.ps_cache_bytes_paged(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages))


def ps_cache_create_paged(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages, dev_buf,
                          dev_bytes, stream=None):
    h = _vp()
    _check("ps_cache_create_paged",
           _lib.ps_cache_create_paged(W, P_max, Hkv, d, dtype, max_seqs, page_rows, num_pages,
                                      _ptr(dev_buf), dev_bytes, _stream(stream), ctypes.byref(h)))
    return h


def ps_ring_pages_free(cache) -> int:
    r = int(_lib.ps_ring_pages_free(cache))
    if r < 0:
        _check("ps_ring_pages_free", r)
    return r


def ps_cache_destroy(cache) -> None:
    _lib.ps_cache_destroy(cache)


def ps_seq_reset(cache, seq, ring_head_offset=0, stream=None) -> None:
    _check("ps_seq_reset", _lib.ps_seq_reset(cache, seq, ring_head_offset, _stream(stream)))


def ps_seq_info_get(cache, seq) -> SeqInfo:
    info = SeqInfo()
    _check("ps_seq_info_get", _lib.ps_seq_info_get(cache, seq, ctypes.byref(info)))
    return info


def ps_prefill_prefix(cache, seq, k, v, P_s, stream=None) -> None:
    _check("ps_prefill_prefix", _lib.ps_prefill_prefix(cache, seq, _ptr(k), _ptr(v), P_s,
                                                       _stream(stream)))


def ps_append_kv(cache, seq_ids, k, v, n, stream=None) -> None:
    ids, B = _ints(seq_ids, ctypes.c_int)
    _check("ps_append_kv", _lib.ps_append_kv(cache, ids, B, _ptr(k), _ptr(v), n, _stream(stream)))


def ps_decode_workspace_bytes(cache, B, Hq) -> int:
    return int(_lib.ps_decode_workspace_bytes(cache, B, Hq))


def ps_attend_decode(cache, q, seq_ids, t, Hq, scale, out, workspace, workspace_bytes,
                     stream=None) -> None:
    ids, B = _ints(seq_ids, ctypes.c_int)
    ts, Bt = _ints(t, ctypes.c_int64)
    if Bt != B:
        raise ValueError("seq_ids and t differ in length")
    _check("ps_attend_decode", _lib.ps_attend_decode(cache, _ptr(q), ids, ts, B, Hq, scale,
                                                     _ptr(out), _ptr(workspace), workspace_bytes,
                                                     _stream(stream)))


def ps_decode_step(cache, q, k_new, v_new, seq_ids, t, Hq, scale, out, workspace,
                   workspace_bytes, stream=None) -> None:
    """Append the token at t == next_pos of each sequence, then attend at t (one pass)."""
    ids, B = _ints(seq_ids, ctypes.c_int)
    ts, Bt = _ints(t, ctypes.c_int64)
    if Bt != B:
        raise ValueError("seq_ids and t differ in length")
    _check("ps_decode_step", _lib.ps_decode_step(cache, _ptr(q), _ptr(k_new), _ptr(v_new), ids,
                                                 ts, B, Hq, scale, _ptr(out), _ptr(workspace),
                                                 workspace_bytes, _stream(stream)))


def ps_attend_decode_static(cache, q, seq_ids, t, Hq, scale, out, stream=None) -> None:
    """Decode with the library's fixed device scratch (no workspace, allocates nothing)."""
    ids, B = _ints(seq_ids, ctypes.c_int)
    ts, Bt = _ints(t, ctypes.c_int64)
    if Bt != B:
        raise ValueError("seq_ids and t differ in length")
    _check("ps_attend_decode_static", _lib.ps_attend_decode_static(cache, _ptr(q), ids, ts, B, Hq,
                                                                   scale, _ptr(out),
                                                                   _stream(stream)))


def ps_attend_chunk(cache, seq, q, k_blk, v_blk, t0, n, Hq, scale, out, append_after=0,
                    stream=None) -> None:
    _check("ps_attend_chunk", _lib.ps_attend_chunk(cache, seq, _ptr(q), _ptr(k_blk), _ptr(v_blk),
                                                   t0, n, Hq, scale, _ptr(out), int(append_after),
                                                   _stream(stream)))


def ps_set_chunk_small_max(cache, n_max) -> None:
    _check("ps_set_chunk_small_max", _lib.ps_set_chunk_small_max(cache, int(n_max)))


def _entries(seq_ids, t0, n):
    ids, B = _ints(seq_ids, ctypes.c_int)
    ts, Bt = _ints(t0, ctypes.c_int64)
    ns, Bn = _ints(n, ctypes.c_int)
    if not B == Bt == Bn:
        raise ValueError("seq_ids, t0 and n differ in length")
    return ids, ts, ns, B


def ps_attend_chunk_batch(cache, seq_ids, t0, n, q, k_blk, v_blk, Hq, scale, out, append_after=0,
                          stream=None) -> None:
    """Chunks of several sequences in one launch; rows packed end to end in entry order."""
    ids, ts, ns, B = _entries(seq_ids, t0, n)
    _check("ps_attend_chunk_batch", _lib.ps_attend_chunk_batch(
        cache, ids, ts, ns, B, _ptr(q), _ptr(k_blk), _ptr(v_blk), Hq, scale, _ptr(out),
        int(append_after), _stream(stream)))


def ps_attend_prompt_batch(cache, seq_ids, t0, n, q, Hq, scale, out, stream=None) -> None:
    """Prompt attention of several sequences in one launch; rows packed in entry order."""
    ids, ts, ns, B = _entries(seq_ids, t0, n)
    _check("ps_attend_prompt_batch", _lib.ps_attend_prompt_batch(
        cache, ids, ts, ns, B, _ptr(q), Hq, scale, _ptr(out), _stream(stream)))


def ps_share_prefix(cache, seq, src, stream=None) -> None:
    """Empty sequence `seq` reads the pinned prefix of sequence `src`."""
    _check("ps_share_prefix", _lib.ps_share_prefix(cache, seq, src, _stream(stream)))


def ps_attend_prompt(cache, seq, q, t0, n, Hq, scale, out, stream=None) -> None:
    """Causal attention of prompt tokens t0..t0+n-1 (inside the pinned prefix)."""
    _check("ps_attend_prompt", _lib.ps_attend_prompt(cache, seq, _ptr(q), t0, n, Hq, scale,
                                                     _ptr(out), _stream(stream)))


def ps_debug_wait_timeout(cache, limit_cycles, stream=None) -> None:
    """Run one bounded wait that nothing satisfies (sets the time-out bit)."""
    _check("ps_debug_wait_timeout", _lib.ps_debug_wait_timeout(cache, limit_cycles,
                                                               _stream(stream)))


def ps_export_window(cache, seq, k, v, pos, count_out, stream=None) -> None:
    _check("ps_export_window", _lib.ps_export_window(cache, seq, _ptr(k), _ptr(v), _ptr(pos),
                                                     _ptr(count_out), _stream(stream)))


def ps_import_window(cache, seq, next_pos, k, v, n, ring_head_offset=0, stream=None) -> None:
    _check("ps_import_window", _lib.ps_import_window(cache, seq, next_pos, _ptr(k), _ptr(v), n,
                                                     ring_head_offset, _stream(stream)))


def ps_debug_visible(cache, seq, t, pos_out, n_out, stream=None) -> None:
    _check("ps_debug_visible", _lib.ps_debug_visible(cache, seq, t, _ptr(pos_out), _ptr(n_out),
                                                     _stream(stream)))


def ps_device_error(cache, stream=None) -> int:
    code = ctypes.c_int32(0)
    _check("ps_device_error", _lib.ps_device_error(cache, ctypes.byref(code), _stream(stream)))
    return int(code.value)

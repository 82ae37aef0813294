"""The C-ABI library loads and exports every entry point include/ps.h declares;
host-only calls and argument checks that run before any CUDA call (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^PS_API\s+[\w\s\*]+?\b(ps_\w+)\s*\(", src, re.M)
    return names


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    for must in ["ps_cache_create", "ps_prefill_prefix", "ps_append_kv", "ps_attend_decode",
                 "ps_attend_chunk", "ps_export_window", "ps_import_window", "ps_debug_visible"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    from prefix_sliding_window_ring_b200 import abi
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in abi.SIGNATURES, f"binding lacks {name}"
    assert set(abi.SIGNATURES) == set(declared_symbols())


def test_cache_bytes_layout():
    from prefix_sliding_window_ring_b200 import abi
    n = abi.ps_cache_bytes(4096, 128, 8, 128, abi.PS_BF16, 8)
    slab = 8 * 8 * (128 + 4096) * 128 * 2
    assert n >= 2 * slab + 8 * 4096 * 8
    assert n < 2 * slab + 8 * 4096 * 8 + 8192
    assert abi.ps_cache_bytes(0, 1, 1, 64, abi.PS_F32, 1) == 0       # W = 0 rejected
    assert abi.ps_cache_bytes(4, 1, 1, 96, abi.PS_F32, 1) == 0       # head_dim 96 unsupported
    assert abi.ps_cache_bytes(4, -1, 1, 64, abi.PS_F32, 1) == 0
    assert abi.ps_cache_bytes(4, 1, 1, 64, 7, 1) == 0                # unknown dtype


def test_create_rejects_bad_arguments_before_touching_cuda():
    from prefix_sliding_window_ring_b200 import abi
    with pytest.raises(abi.PSError) as e:
        abi.ps_cache_create(4, 1, 1, 64, abi.PS_F32, 1, None, 1 << 20, 0)
    assert e.value.code == abi.PS_EINVAL
    with pytest.raises(abi.PSError) as e:
        abi.ps_cache_create(0, 1, 1, 64, abi.PS_F32, 1, 256, 1 << 20, 0)
    assert e.value.code == abi.PS_EINVAL
    with pytest.raises(abi.PSError) as e:
        abi.ps_cache_create(4, 1, 1, 80, abi.PS_F32, 1, 256, 1 << 20, 0)
    assert e.value.code == abi.PS_EUNSUPPORTED
    with pytest.raises(abi.PSError) as e:
        abi.ps_cache_create(4, 1, 1, 64, abi.PS_F32, 1, 256, 16, 0)
    assert e.value.code == abi.PS_ENOMEM
    assert "needs" in abi.ps_last_error()
    assert abi.ps_decode_workspace_bytes(None, 1, 1) == 0


def test_paged_cache_bytes_and_argument_checks():
    from prefix_sliding_window_ring_b200 import abi
    unpaged = abi.ps_cache_bytes(512, 64, 2, 128, abi.PS_BF16, 4)
    # one page per sequence holds the same rows as the unpaged layout plus a small page table
    same = abi.ps_cache_bytes_paged(512, 64, 2, 128, abi.PS_BF16, 4, 512, 4)
    assert unpaged <= same <= unpaged + 4096
    half = abi.ps_cache_bytes_paged(512, 64, 2, 128, abi.PS_BF16, 4, 128, 8)   # 8 of 16 pages
    assert half < same
    assert abi.ps_cache_bytes_paged(512, 64, 2, 128, abi.PS_BF16, 4, 100, 8) == 0  # 512 % 100
    assert abi.ps_cache_bytes_paged(512, 64, 2, 128, abi.PS_BF16, 4, 1024, 8) == 0  # page > W
    assert abi.ps_cache_bytes_paged(512, 64, 2, 128, abi.PS_BF16, 4, 128, 0) == 0  # no pages
    assert abi.ps_cache_bytes_paged(512, 64, 2, 128, abi.PS_BF16, 4, 0, 8) == 0
    with pytest.raises(abi.PSError) as e:
        abi.ps_cache_create_paged(512, 64, 2, 128, abi.PS_BF16, 4, 0, 8, 256, 1 << 20)
    assert e.value.code == abi.PS_EINVAL
    with pytest.raises(abi.PSError) as e:
        abi.ps_ring_pages_free(None)
    assert e.value.code == abi.PS_EINVAL


def test_every_call_rejects_a_null_cache_before_touching_cuda():
    from prefix_sliding_window_ring_b200 import abi
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name, (res, args) in abi.SIGNATURES.items():
        getattr(lib, name).restype, getattr(lib, name).argtypes = res, args
    ids = (ctypes.c_int * 2)(0, 1)
    ts = (ctypes.c_int64 * 2)(5, 6)
    ns = (ctypes.c_int * 2)(1, 1)
    info = abi.SeqInfo()
    calls = {
        "ps_seq_info_get": (None, 0, ctypes.byref(info)),
        "ps_seq_reset": (None, 0, 0, None),
        "ps_prefill_prefix": (None, 0, None, None, 1, None),
        "ps_share_prefix": (None, 1, 0, None),
        "ps_append_kv": (None, ids, 2, None, None, 1, None),
        "ps_attend_decode": (None, None, ids, ts, 2, 2, 1.0, None, None, 0, None),
        "ps_attend_decode_static": (None, None, ids, ts, 2, 2, 1.0, None, None),
        "ps_decode_step": (None, None, None, None, ids, ts, 2, 2, 1.0, None, None, 0, None),
        "ps_attend_chunk": (None, 0, None, None, None, 5, 1, 2, 1.0, None, 0, None),
        "ps_attend_chunk_batch": (None, ids, ts, ns, 2, None, None, None, 2, 1.0, None, 0, None),
        "ps_attend_prompt": (None, 0, None, 0, 1, 2, 1.0, None, None),
        "ps_attend_prompt_batch": (None, ids, ts, ns, 2, None, 2, 1.0, None, None),
        "ps_export_window": (None, 0, None, None, None, None, None),
        "ps_import_window": (None, 0, 5, None, None, 1, 0, None),
        "ps_debug_visible": (None, 0, 5, None, None, None),
        "ps_debug_wait_timeout": (None, 1000, None),
        "ps_device_error": (None, None, None),
        "ps_ring_pages_free": (None,),
    }
    for name, a in calls.items():
        assert getattr(lib, name)(*a) == abi.PS_EINVAL, name
        assert abi.ps_last_error(), name
    assert lib.ps_decode_workspace_bytes(None, 1, 1) == 0
    lib.ps_cache_destroy(None)  # deleting NULL is a no-op

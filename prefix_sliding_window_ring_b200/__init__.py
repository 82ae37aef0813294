"""Prefix-sliding attention over a ring-buffer KV cache, for B200 (sm_100a).

The work happens in ``libps.so`` (hand-written CUDA, C ABI in include/ps.h);
``abi`` binds it call for call and ``Cache`` owns the torch device buffers a
cache lives in.  Importing fails loudly if the library has not been built.
"""
from .abi import (PS_BF16, PS_EINVAL, PS_ENOMEM, PS_EPOS, PS_ESTATE, PS_F32,  # noqa: F401
                  PSError, ps_append_kv, ps_attend_chunk, ps_attend_decode, ps_attend_prompt,
                  ps_attend_decode_static, ps_cache_bytes, ps_cache_create, ps_cache_destroy,
                  ps_debug_visible, ps_decode_step, ps_decode_workspace_bytes, ps_device_error,
                  ps_export_window, ps_import_window, ps_last_error, ps_prefill_prefix,
                  ps_seq_info_get, ps_seq_reset, ps_share_prefix, ps_version)
from .cache import Cache  # noqa: F401

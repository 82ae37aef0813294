"""A cache bound to torch-allocated device memory (plumbing around the C ABI)."""
from __future__ import annotations

import torch

from . import abi

TORCH_DTYPE = {abi.PS_F32: torch.float32, abi.PS_BF16: torch.bfloat16}


class Cache:
    """Owns the device buffer of one ps_cache and forwards calls to the C ABI."""

    def __init__(self, W: int, P_max: int, Hkv: int, d: int, dtype: int, max_seqs: int,
                 device="cuda", stream=None, page_rows: int = 0, num_pages: int = 0):
        """page_rows > 0 makes a paged ring (num_pages physical pages of page_rows slots)."""
        self.W, self.P_max, self.Hkv, self.d, self.dtype, self.max_seqs = W, P_max, Hkv, d, dtype, max_seqs
        self.torch_dtype = TORCH_DTYPE[dtype]
        if page_rows > 0:
            self.nbytes = abi.ps_cache_bytes_paged(W, P_max, Hkv, d, dtype, max_seqs, page_rows,
                                                   num_pages)
        else:
            self.nbytes = abi.ps_cache_bytes(W, P_max, Hkv, d, dtype, max_seqs)
        if self.nbytes == 0:
            raise abi.PSError("ps_cache_bytes", abi.PS_EINVAL, "invalid cache shape")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        if page_rows > 0:
            self.handle = abi.ps_cache_create_paged(W, P_max, Hkv, d, dtype, max_seqs, page_rows,
                                                    num_pages, self.buf, self.nbytes, stream)
        else:
            self.handle = abi.ps_cache_create(W, P_max, Hkv, d, dtype, max_seqs, self.buf,
                                              self.nbytes, stream)
        self._ws = {}

    def ring_pages_free(self) -> int:
        return abi.ps_ring_pages_free(self.handle)

    def close(self) -> None:
        if getattr(self, "handle", None) is not None:
            abi.ps_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the binding may already be gone
            pass

    # ---- calls, same names as the C ABI without the ps_ prefix ----
    def seq_reset(self, seq, ring_head_offset=0, stream=None):
        abi.ps_seq_reset(self.handle, seq, ring_head_offset, stream)

    def seq_info(self, seq):
        return abi.ps_seq_info_get(self.handle, seq)

    def prefill_prefix(self, seq, k, v, P_s, stream=None):
        abi.ps_prefill_prefix(self.handle, seq, k, v, P_s, stream)

    def append_kv(self, seq_ids, k, v, n, stream=None):
        abi.ps_append_kv(self.handle, seq_ids, k, v, n, stream)

    def decode_workspace(self, B: int, Hq: int) -> torch.Tensor:
        nb = abi.ps_decode_workspace_bytes(self.handle, B, Hq)
        key = (B, Hq)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nb:
            ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=self.buf.device)
            self._ws[key] = ws
        return ws

    def attend_decode(self, q, seq_ids, t, Hq, scale, out, workspace=None, stream=None):
        B = len(seq_ids)
        ws = workspace if workspace is not None else self.decode_workspace(B, Hq)
        abi.ps_attend_decode(self.handle, q, seq_ids, t, Hq, scale, out, ws, ws.numel(), stream)

    def decode_step(self, q, k_new, v_new, seq_ids, t, Hq, scale, out, workspace=None,
                    stream=None):
        B = len(seq_ids)
        ws = workspace if workspace is not None else self.decode_workspace(B, Hq)
        abi.ps_decode_step(self.handle, q, k_new, v_new, seq_ids, t, Hq, scale, out, ws,
                           ws.numel(), stream)

    def attend_chunk(self, seq, q, k_blk, v_blk, t0, n, Hq, scale, out, append_after=0, stream=None):
        abi.ps_attend_chunk(self.handle, seq, q, k_blk, v_blk, t0, n, Hq, scale, out, append_after,
                            stream)

    def set_chunk_small_max(self, n_max):
        abi.ps_set_chunk_small_max(self.handle, n_max)

    def attend_chunk_batch(self, seq_ids, t0, n, q, k_blk, v_blk, Hq, scale, out, append_after=0,
                           stream=None):
        abi.ps_attend_chunk_batch(self.handle, seq_ids, t0, n, q, k_blk, v_blk, Hq, scale, out,
                                  append_after, stream)

    def attend_prompt_batch(self, seq_ids, t0, n, q, Hq, scale, out, stream=None):
        abi.ps_attend_prompt_batch(self.handle, seq_ids, t0, n, q, Hq, scale, out, stream)

    def share_prefix(self, seq, src, stream=None):
        abi.ps_share_prefix(self.handle, seq, src, stream)

    def attend_prompt(self, seq, q, t0, n, Hq, scale, out, stream=None):
        abi.ps_attend_prompt(self.handle, seq, q, t0, n, Hq, scale, out, stream)

    def export_window(self, seq, stream=None):
        k = torch.empty((self.W, self.Hkv, self.d), dtype=self.torch_dtype, device=self.buf.device)
        v = torch.empty_like(k)
        pos = torch.empty(self.W, dtype=torch.int64, device=self.buf.device)
        cnt = torch.empty(1, dtype=torch.int32, device=self.buf.device)
        abi.ps_export_window(self.handle, seq, k, v, pos, cnt, stream)
        n = int(cnt.item())
        return k[:n], v[:n], pos[:n]

    def import_window(self, seq, next_pos, k, v, n, ring_head_offset=0, stream=None):
        abi.ps_import_window(self.handle, seq, next_pos, k, v, n, ring_head_offset, stream)

    def debug_visible(self, seq, t, stream=None):
        pos = torch.empty(self.P_max + self.W, dtype=torch.int64, device=self.buf.device)
        n = torch.empty(1, dtype=torch.int32, device=self.buf.device)
        abi.ps_debug_visible(self.handle, seq, t, pos, n, stream)
        return pos[: int(n.item())]

    def device_error(self, stream=None) -> int:
        return abi.ps_device_error(self.handle, stream)

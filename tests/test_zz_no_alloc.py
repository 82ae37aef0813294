"""ps_attend_decode_static: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace -- a host runtime that owns all
device memory through its own pool, or a latency-critical loop that must not
call cudaMalloc (it synchronises the device).  This entry point runs the same
decode with its scratch in a fixed array inside the library.  These tests call
it through the C ABI and compare it with ps_attend_decode (caller workspace) on
two calls in a row, within the bf16 tolerances used by every parity test.
The file is named to be collected last.
"""
import math

import pytest
import torch

from prefix_sliding_window_ring_b200 import Cache, PSError, abi
from tests.helpers import SeqData, check_close, ps_dtype, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _setup(B, Hq, Hkv, d, P, W, t, seed=5):
    c = Cache(W, P, Hkv, d, ps_dtype("bf16"), B)
    sds = [SeqData(seed, b, Hq, Hkv, d, "bf16") for b in range(B)]
    for b, sd in enumerate(sds):
        c.prefill_prefix(b, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
        n = min(W, t - P)
        c.import_window(b, t, to_torch(sd.k(t - n, n)), to_torch(sd.v(t - n, n)), n, (7 * b) % W)
    return c, sds


def test_static_scratch_matches_workspace_decode_twice():
    B, Hq, Hkv, d, P, W = 8, 16, 8, 128, 128, 4096
    t0 = 20000
    c, sds = _setup(B, Hq, Hkv, d, P, W, t0)
    ids = list(range(B))
    scale = 1.0 / math.sqrt(d)
    ws = c.decode_workspace(B, Hq)
    for step in range(2):                     # two calls in a row
        t = t0 + step
        c.append_kv(ids, torch.stack([to_torch(sd.k(t, 1))[0] for sd in sds]),
                    torch.stack([to_torch(sd.v(t, 1))[0] for sd in sds]), 1)
        q = torch.stack([to_torch(sd.q(t, 1))[0] for sd in sds])
        ref = torch.empty_like(q)
        got = torch.empty_like(q)
        abi.ps_attend_decode(c.handle, q, ids, [t] * B, Hq, scale, ref, ws, ws.numel())
        abi.ps_attend_decode_static(c.handle, q, ids, [t] * B, Hq, scale, got)
        torch.cuda.synchronize()
        check_close(to_f64(got), to_f64(ref), "bf16", f"static vs workspace, call {step + 1}")
    assert c.device_error() == 0


def test_static_scratch_rejects_batches_over_its_size():
    B, Hq, Hkv, d, P, W = 128, 64, 8, 128, 1, 256
    c = Cache(W, P, Hkv, d, ps_dtype("bf16"), B)
    sd = SeqData(1, 0, Hq, Hkv, d, "bf16")
    kp, vp = to_torch(sd.k(0, P)), to_torch(sd.v(0, P))
    for b in range(B):
        c.prefill_prefix(b, kp, vp, P)
    k = to_torch(sd.k(P, W)).unsqueeze(0).expand(B, -1, -1, -1).contiguous()
    v = to_torch(sd.v(P, W)).unsqueeze(0).expand(B, -1, -1, -1).contiguous()
    c.append_kv(list(range(B)), k, v, W)
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(PSError) as e:
        abi.ps_attend_decode_static(c.handle, q, list(range(B)), [P + W - 1] * B, Hq, 0.1, out)
    assert e.value.code == abi.PS_ENOMEM
    assert "scratch" in str(e.value)

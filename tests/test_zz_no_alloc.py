"""ps_attend_decode_static: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace -- a host runtime that owns all
device memory through its own pool, or a latency-critical loop that must not
call cudaMalloc (it synchronises the device).  This entry point runs the same
decode with its scratch in a fixed array inside the library.  These tests call
it through the C ABI and compare it with ps_attend_decode (caller workspace) on
two calls in a row: the same kernels with the same slot layout, so the outputs
must be bit-identical (which is within the bf16 tolerances of every parity
test); both are also checked against the float64 oracle.  The file is named to
be collected last.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from prefix_sliding_window_ring_b200 import Cache, PSError, abi
from tests.helpers import SeqData, check_close, oracle_decode, ps_dtype, to_f64, to_torch

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
        assert torch.equal(got, ref), f"static vs workspace differ, call {step + 1}"
        check_close(to_f64(got), to_f64(ref), "bf16", f"static vs workspace, call {step + 1}")
        batch = oracle.Batch()
        q64 = to_f64(q)
        exp = [oracle_decode(batch, sd, P, W, t, scale, q64[b]) for b, sd in enumerate(sds)]
        batch.run()
        want = np.stack([np.concatenate(e, axis=0) for e in exp])
        check_close(to_f64(got), want, "bf16", f"static vs oracle, call {step + 1}")
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


def test_static_scratch_checks_arguments_first():
    """Bad arguments are reported as by ps_attend_decode (not as a set-up
    failure), and an empty batch is a no-op."""
    c, sds = _setup(2, 4, 2, 128, 8, 64, 100)
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    abi.ps_attend_decode_static(c.handle, q, [], [], 4, 0.1, out)          # B = 0
    with pytest.raises(PSError) as e:
        abi.ps_attend_decode_static(c.handle, q, [0, 1], [100, 100], 4, 0.1, out)
    assert e.value.code == abi.PS_EPOS                                      # t is not next_pos-1
    with pytest.raises(PSError) as e:
        abi.ps_attend_decode_static(c.handle, q, [0, 0], [99, 99], 4, 0.1, out)
    assert e.value.code == abi.PS_EINVAL                                    # duplicate id
    with pytest.raises(PSError) as e:
        abi.ps_attend_decode_static(c.handle, q, [0, 1], [99, 99], 3, 0.1, out)
    assert e.value.code == abi.PS_EINVAL                                    # Hq % Hkv
    assert c.device_error() == 0

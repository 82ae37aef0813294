"""GPU parity at full size: the single-model decode (B=8, t in {2048, 4224,
16384, 65536}) and the ragged 64-sequence serving batch, every output element
against the float64 oracle; plus batch-size edge cases."""
import numpy as np
import pytest
import torch

import oracle
import synth
from prefix_sliding_window_ring_b200 import Cache
from synth import workloads
from tests.helpers import (SeqData, check_close, default_scale, expected_window, oracle_decode,
                           ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu


def setup_seq(c, sd, seq, P, t, W, h0):
    """Prefix [0,P), window as it stands before position t, then append token t."""
    c.seq_reset(seq, 0)
    c.prefill_prefix(seq, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    n = min(W, t - P)
    c.import_window(seq, t, to_torch(sd.k(t - n, n)), to_torch(sd.v(t - n, n)), n, h0)
    c.append_kv([seq], to_torch(sd.k(t, 1)), to_torch(sd.v(t, 1)), 1)


def decode_and_check(c, sds, Ps, ts, W, Hq, d, dtype, what):
    B = len(sds)
    scale = default_scale(d)
    q = torch.stack([to_torch(sd.q(t, 1))[0] for sd, t in zip(sds, ts)])
    out = torch.empty_like(q)
    c.attend_decode(q, list(range(B)), ts, Hq, scale, out)
    assert c.device_error() == 0
    batch = oracle.Batch()
    exp = []
    for sd, P, t, qb in zip(sds, Ps, ts, to_f64(q)):
        exp.append(oracle_decode(batch, sd, P, W, t, scale, qb))
    batch.run()
    exp = np.stack([np.concatenate(e, axis=0) for e in exp])
    return check_close(to_f64(out), exp, dtype, what)


@pytest.mark.parametrize("t", workloads.DECODE["t_values"])
def test_single_model_decode(t):
    s = workloads.DECODE["shape"]
    B = workloads.DECODE["B"]
    ks = synth.chan_scale(0, s.Hkv, s.d)
    c = Cache(s.W, s.P, s.Hkv, s.d, ps_dtype(s.dtype), B)
    sds = [SeqData(0, b, s.Hq, s.Hkv, s.d, s.dtype, k_scale=ks) for b in range(B)]
    for b, sd in enumerate(sds):
        setup_seq(c, sd, b, s.P, t, s.W, h0=(b * 997) % s.W)
    decode_and_check(c, sds, [s.P] * B, [t] * B, s.W, s.Hq, s.d, s.dtype, f"decode t={t}")
    # ring of the last sequence holds exactly lastWindow of its history
    k, v, pos = c.export_window(B - 1)
    assert pos.cpu().tolist() == expected_window(s.P, s.W, t + 1)


def test_ragged_serving_batch():
    s = workloads.ragged_shape()
    draws = workloads.ragged_draws(0)
    B = len(draws)
    c = Cache(s.W, s.P, s.Hkv, s.d, ps_dtype(s.dtype), B)
    sds = [SeqData(0, b, s.Hq, s.Hkv, s.d, s.dtype) for b in range(B)]
    for b, (sd, r) in enumerate(zip(sds, draws)):
        setup_seq(c, sd, b, r.P, r.t, s.W, r.h0)
    decode_and_check(c, sds, [r.P for r in draws], [r.t for r in draws], s.W, s.Hq, s.d, s.dtype,
                     "ragged")


@pytest.mark.parametrize("B,Hq,d", [(3, 16, 128), (10, 16, 128), (3, 64, 128), (10, 8, 64)],
                         ids=["24pairs-G2", "80pairs-G2", "24pairs-G8", "80pairs-G1-d64"])
def test_cluster_sizes(B, Hq, d):
    """Few equal pairs run in cluster mode, where each CTA hands its merged
    state to the peers that own the output slices.  24 (sequence, kv head)
    pairs take clusters of 8 CTAs, 80 pairs clusters of 2 (the headline
    decode, 64 pairs, takes 4); G = 8 makes a slice span whole rows of the
    outputs, d = 64 halves them.  Every output against the float64 oracle."""
    W, P, t, Hkv = 2048, 64, 3000, 8
    c = Cache(W, P, Hkv, d, ps_dtype("bf16"), B)
    sds = [SeqData(11, b, Hq, Hkv, d, "bf16") for b in range(B)]
    for b, sd in enumerate(sds):
        setup_seq(c, sd, b, P, t, W, (331 * b) % W)
    decode_and_check(c, sds, [P] * B, [t] * B, W, Hq, d, "bf16", f"B={B} Hq={Hq} d={d}")


def test_batch_larger_than_one_launch():
    """300 sequences (more than one launch's worth of batch entries), fp32 d=64."""
    W, P, Hq, Hkv, d = 8, 2, 4, 2, 64
    B = 300
    c = Cache(W, P, Hkv, d, ps_dtype("f32"), B)
    sds = [SeqData(3, b, Hq, Hkv, d, "f32") for b in range(B)]
    ts = [P + (b % 19) for b in range(B)]
    for b, sd in enumerate(sds):
        c.seq_reset(b, b % W)
        c.prefill_prefix(b, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    # bulk append of 19 tokens to everyone, then trim by per-sequence import
    k = torch.stack([to_torch(sd.k(P, 19)) for sd in sds])
    v = torch.stack([to_torch(sd.v(P, 19)) for sd in sds])
    c.append_kv(list(range(B)), k, v, 19)
    for b, sd in enumerate(sds):
        info = c.seq_info(b)
        assert info.next_pos == P + 19 and info.count == W
        _, _, pos = c.export_window(b) if b % 50 == 0 else (None, None, None)
        if pos is not None:
            assert pos.cpu().tolist() == expected_window(P, W, P + 19)
    for b, sd in enumerate(sds):
        t = ts[b]
        n = min(W, t - P)
        c.import_window(b, t, to_torch(sd.k(t - n, n)), to_torch(sd.v(t - n, n)), n, (3 * b) % W)
    k1 = torch.stack([to_torch(sd.k(t, 1)) for sd, t in zip(sds, ts)])
    v1 = torch.stack([to_torch(sd.v(t, 1)) for sd, t in zip(sds, ts)])
    c.append_kv(list(range(B)), k1, v1, 1)
    decode_and_check(c, sds, [P] * B, ts, W, Hq, d, "f32", "B=300")


def test_empty_calls_are_noops():
    c = Cache(4, 2, 1, 64, ps_dtype("f32"), 2)
    sd = SeqData(1, 0, 1, 1, 64, "f32")
    c.prefill_prefix(0, to_torch(sd.k(0, 2)), to_torch(sd.v(0, 2)), 2)
    c.append_kv([], torch.empty(0, device="cuda"), torch.empty(0, device="cuda"), 1)
    c.append_kv([0], torch.empty(0, device="cuda"), torch.empty(0, device="cuda"), 0)
    assert c.seq_info(0).next_pos == 2
    c.attend_decode(torch.empty(0, device="cuda"), [], [], 1, 0.1,
                    torch.empty(0, device="cuda"),
                    workspace=torch.zeros(256, dtype=torch.uint8, device="cuda"))
    k, v, pos = c.export_window(0)
    assert pos.numel() == 0
    assert c.device_error() == 0


def test_bulk_append_longer_than_window_equals_single_steps():
    """n > W tokens in one call leave the ring exactly as n single steps (run = foldl step)."""
    W, P, Hkv, d = 5, 3, 2, 128
    sd = SeqData(2, 0, 2, Hkv, d, "bf16")
    a = Cache(W, P, Hkv, d, ps_dtype("bf16"), 1)
    b = Cache(W, P, Hkv, d, ps_dtype("bf16"), 1)
    for c in (a, b):
        c.seq_reset(0, 2)
        c.prefill_prefix(0, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    n = 17
    kk, vv = to_torch(sd.k(P, n)), to_torch(sd.v(P, n))
    a.append_kv([0], kk, vv, n)
    for i in range(n):
        b.append_kv([0], kk[i:i + 1], vv[i:i + 1], 1)
    ka, va, pa = a.export_window(0)
    kb, vb, pb = b.export_window(0)
    assert pa.tolist() == pb.tolist() == expected_window(P, W, P + n)
    assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
    assert torch.equal(va.view(torch.int16), vb.view(torch.int16))
    ia, ib = a.seq_info(0), b.seq_info(0)
    assert (ia.head, ia.count, ia.next_pos) == (ib.head, ib.count, ib.next_pos)

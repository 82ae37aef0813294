"""GPU parity of ps_decode_step (append the token, then attend, in one pass).

The fused step must leave exactly the state, and give exactly the output, of
ps_append_kv (n = 1) followed by ps_attend_decode: both run here side by side
on two caches fed the same rows, and are compared bit for bit; the outputs are
also checked against the float64 oracle and the rings against lastWindow.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from prefix_sliding_window_ring_b200 import PS_EPOS, Cache, PSError
from synth import workloads
from tests.helpers import (SeqData, check_close, default_scale, expected_window, oracle_decode,
                           ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu


def _bits(x):
    return x.view(torch.int32 if x.dtype == torch.float32 else torch.int16)


def _same_state(a, b, seqs, what):
    for s in seqs:
        ia, ib = a.seq_info(s), b.seq_info(s)
        assert (ia.next_pos, ia.head, ia.count, ia.P) == (ib.next_pos, ib.head, ib.count, ib.P), what
        ka, va, pa = a.export_window(s)
        kb, vb, pb = b.export_window(s)
        assert pa.tolist() == pb.tolist(), f"{what}: ring positions of sequence {s}"
        assert torch.equal(_bits(ka), _bits(kb)), f"{what}: ring keys of sequence {s}"
        assert torch.equal(_bits(va), _bits(vb)), f"{what}: ring values of sequence {s}"


STEP_CASES = [(1, 0, "f32", 0), (2, 1, "bf16", 1), (5, 3, "f32", 2), (129, 100, "bf16", 77),
              (128, 0, "f32", 5)]


@pytest.mark.parametrize("W,P,dtype,h0", STEP_CASES,
                         ids=[f"W{W}-P{P}-{dt}-h{h}" for W, P, dt, h in STEP_CASES])
def test_step_equals_append_then_decode(W, P, dtype, h0):
    """One sequence from an empty window through the not-full, just-full,
    first-eviction and wrap phases: every step's output and the whole ring state
    equal those of append + decode, and the output matches the oracle."""
    s = workloads.sweep_shape(W, P, dtype)
    sd = SeqData(4, 0, s.Hq, s.Hkv, s.d, dtype)
    scale = default_scale(s.d)
    T = P + 3 * W + 2
    kall, vall = to_torch(sd.k(0, T)), to_torch(sd.v(0, T))
    qall = to_torch(sd.q(P, T - P))
    fused = Cache(W, max(P, 1), s.Hkv, s.d, ps_dtype(dtype), 1)
    split = Cache(W, max(P, 1), s.Hkv, s.d, ps_dtype(dtype), 1)
    for c in (fused, split):
        c.seq_reset(0, h0)
        c.prefill_prefix(0, kall[:P], vall[:P], P)
    out_f = torch.empty((T - P, s.Hq, s.d), dtype=kall.dtype, device="cuda")
    out_s = torch.empty_like(out_f)
    for t in range(P, T):
        i = t - P
        fused.decode_step(qall[i:i + 1], kall[t:t + 1], vall[t:t + 1], [0], [t], s.Hq, scale,
                          out_f[i:i + 1])
        split.append_kv([0], kall[t:t + 1], vall[t:t + 1], 1)
        split.attend_decode(qall[i:i + 1], [0], [t], s.Hq, scale, out_s[i:i + 1])
        if W <= 5 or i % 37 == 0 or t == T - 1:
            _same_state(fused, split, [0], f"t={t}")
            assert fused.export_window(0)[2].tolist() == expected_window(P, W, t + 1)
    assert torch.equal(_bits(out_f), _bits(out_s)), "fused and split outputs differ"
    assert fused.device_error() == 0 and split.device_error() == 0
    steps = list(range(P, T, max(1, (T - P) // 40))) + [T - 1]
    batch = oracle.Batch()
    exp = [oracle_decode(batch, sd, P, W, t, scale, to_f64(qall[t - P])) for t in steps]
    batch.run()
    exp = np.stack([np.concatenate(e, axis=0) for e in exp])
    check_close(to_f64(out_f)[[t - P for t in steps]], exp, dtype, f"step W={W} P={P}")


def _prepare(c, sd, seq, P, t, W, h0):
    """Prefix [0,P) and the window as it stands before position t."""
    c.seq_reset(seq, 0)
    c.prefill_prefix(seq, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    n = min(W, t - P)
    c.import_window(seq, t, to_torch(sd.k(t - n, n)), to_torch(sd.v(t - n, n)), n, h0)


def _fused_vs_split(shape, sds, Ps, ts, h0s, what):
    s = shape
    B = len(sds)
    scale = default_scale(s.d)
    fused = Cache(s.W, s.P, s.Hkv, s.d, ps_dtype(s.dtype), B)
    split = Cache(s.W, s.P, s.Hkv, s.d, ps_dtype(s.dtype), B)
    for c in (fused, split):
        for b, sd in enumerate(sds):
            _prepare(c, sd, b, Ps[b], ts[b], s.W, h0s[b])
    q = torch.stack([to_torch(sd.q(t, 1))[0] for sd, t in zip(sds, ts)])
    kn = torch.stack([to_torch(sd.k(t, 1))[0] for sd, t in zip(sds, ts)])
    vn = torch.stack([to_torch(sd.v(t, 1))[0] for sd, t in zip(sds, ts)])
    ids = list(range(B))
    out_f, out_s = torch.empty_like(q), torch.empty_like(q)
    fused.decode_step(q, kn, vn, ids, ts, s.Hq, scale, out_f)
    split.append_kv(ids, kn, vn, 1)
    split.attend_decode(q, ids, ts, s.Hq, scale, out_s)
    assert fused.device_error() == 0 and split.device_error() == 0
    assert torch.equal(_bits(out_f), _bits(out_s)), f"{what}: fused and split outputs differ"
    _same_state(fused, split, [0, B // 2, B - 1], what)
    batch = oracle.Batch()
    exp = [oracle_decode(batch, sd, P, s.W, t, scale, qb)
           for sd, P, t, qb in zip(sds, Ps, ts, to_f64(q))]
    batch.run()
    exp = np.stack([np.concatenate(e, axis=0) for e in exp])
    return check_close(to_f64(out_f), exp, s.dtype, what)


@pytest.mark.parametrize("t", [4224, 65536])
def test_step_single_model(t):
    """The decode workload (B=8, Hq=16, Hkv=8, d=128, P=128, W=4096, bf16)."""
    s = workloads.DECODE["shape"]
    B = workloads.DECODE["B"]
    ks = synth.chan_scale(0, s.Hkv, s.d)
    sds = [SeqData(0, b, s.Hq, s.Hkv, s.d, s.dtype, k_scale=ks) for b in range(B)]
    _fused_vs_split(s, sds, [s.P] * B, [t] * B, [(b * 613) % s.W for b in range(B)],
                    f"step t={t}")


def test_step_ragged_serving_batch():
    s = workloads.ragged_shape()
    draws = workloads.ragged_draws(0)
    sds = [SeqData(0, b, s.Hq, s.Hkv, s.d, s.dtype) for b in range(len(draws))]
    _fused_vs_split(s, sds, [r.P for r in draws], [r.t for r in draws], [r.h0 for r in draws],
                    "ragged step")


def test_step_rejects_wrong_positions_without_side_effects():
    W, P, Hq, Hkv, d = 8, 2, 2, 1, 64
    c = Cache(W, P, Hkv, d, ps_dtype("f32"), 1)
    sd = SeqData(6, 0, Hq, Hkv, d, "f32")
    c.prefill_prefix(0, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    q, out = to_torch(sd.q(P, 1)), torch.empty((1, Hq, d), device="cuda")
    kn, vn = to_torch(sd.k(P, 1)), to_torch(sd.v(P, 1))
    for bad_t in (P + 1, P - 1):
        with pytest.raises(PSError) as e:
            c.decode_step(q, kn, vn, [0], [bad_t], Hq, 0.125, out)
        assert e.value.code == PS_EPOS
    info = c.seq_info(0)
    assert (info.next_pos, info.count) == (P, 0)
    c.decode_step(q, kn, vn, [0], [P], Hq, 0.125, out)
    assert c.seq_info(0).next_pos == P + 1 and c.device_error() == 0


SHAPES = [("f32", 64, 1, 1), ("bf16", 64, 4, 2), ("bf16", 128, 8, 2), ("f32", 128, 2, 2),
          ("bf16", 128, 1, 4)]


@pytest.mark.parametrize("dtype,d,G,Hkv", SHAPES,
                         ids=[f"{dt}-d{d}-G{G}-Hkv{h}" for dt, d, G, h in SHAPES])
def test_step_every_head_shape(dtype, d, G, Hkv):
    """Every head_dim / GQA group size the decode kernel is built for: a few
    steps across the just-full boundary, fused vs split bit-exact, oracle."""
    W, P = 40, 7
    Hq = G * Hkv
    sd = SeqData(12, 3, Hq, Hkv, d, dtype)
    scale = default_scale(d)
    T = P + W + 6
    kall, vall = to_torch(sd.k(0, T)), to_torch(sd.v(0, T))
    qall = to_torch(sd.q(0, T))
    fused = Cache(W, P, Hkv, d, ps_dtype(dtype), 1)
    split = Cache(W, P, Hkv, d, ps_dtype(dtype), 1)
    for c in (fused, split):
        c.seq_reset(0, 11)
        c.prefill_prefix(0, kall[:P], vall[:P], P)
        c.append_kv([0], kall[P:P + W - 3], vall[P:P + W - 3], W - 3)
    steps = list(range(P + W - 3, T))
    out_f = torch.empty((len(steps), Hq, d), dtype=kall.dtype, device="cuda")
    out_s = torch.empty_like(out_f)
    for i, t in enumerate(steps):
        fused.decode_step(qall[t:t + 1], kall[t:t + 1], vall[t:t + 1], [0], [t], Hq, scale,
                          out_f[i:i + 1])
        split.append_kv([0], kall[t:t + 1], vall[t:t + 1], 1)
        split.attend_decode(qall[t:t + 1], [0], [t], Hq, scale, out_s[i:i + 1])
    assert fused.device_error() == 0 and split.device_error() == 0
    assert torch.equal(_bits(out_f), _bits(out_s))
    _same_state(fused, split, [0], "every-shape")
    batch = oracle.Batch()
    exp = [oracle_decode(batch, sd, P, W, t, scale, to_f64(qall[t])) for t in steps]
    batch.run()
    exp = np.stack([np.concatenate(e, axis=0) for e in exp])
    check_close(to_f64(out_f), exp, dtype, f"step {dtype} d={d} G={G}")


def test_step_batch_larger_than_one_launch():
    """150 sequences in one call (two launches of at most 128 entries)."""
    W, P, Hq, Hkv, d, B = 16, 3, 4, 2, 64, 150
    scale = default_scale(d)
    sds = [SeqData(13, b, Hq, Hkv, d, "f32") for b in range(B)]
    ts = [P + 5 + (b % 23) for b in range(B)]
    fused = Cache(W, P, Hkv, d, ps_dtype("f32"), B)
    split = Cache(W, P, Hkv, d, ps_dtype("f32"), B)
    for c in (fused, split):
        for b, (sd, t) in enumerate(zip(sds, ts)):
            c.seq_reset(b, b % W)
            c.prefill_prefix(b, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
            n = min(W, t - P)
            c.import_window(b, t, to_torch(sd.k(t - n, n)), to_torch(sd.v(t - n, n)), n, (5 * b) % W)
    q = torch.stack([to_torch(sd.q(t, 1))[0] for sd, t in zip(sds, ts)])
    kn = torch.stack([to_torch(sd.k(t, 1))[0] for sd, t in zip(sds, ts)])
    vn = torch.stack([to_torch(sd.v(t, 1))[0] for sd, t in zip(sds, ts)])
    ids = list(range(B))
    out_f, out_s = torch.empty_like(q), torch.empty_like(q)
    fused.decode_step(q, kn, vn, ids, ts, Hq, scale, out_f)
    split.append_kv(ids, kn, vn, 1)
    split.attend_decode(q, ids, ts, Hq, scale, out_s)
    assert fused.device_error() == 0 and split.device_error() == 0
    assert torch.equal(_bits(out_f), _bits(out_s))
    _same_state(fused, split, [0, 127, 128, 149], "B=150")

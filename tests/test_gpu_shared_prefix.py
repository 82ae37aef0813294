"""GPU parity of ps_share_prefix (prompt reuse): sequences that read another
sequence's pinned prefix give exactly the results of sequences holding a private
copy of the same rows -- decode steps, chunks on both chunk kernels and prompt
attention are compared bit for bit, and the decode against the oracle -- and
the sharing rules (no reset of a prefix others read; empty targets only) hold."""
import numpy as np
import pytest
import torch

import oracle
import synth
from prefix_sliding_window_ring_b200 import PS_EINVAL, PS_ESTATE, Cache, PSError
from tests.helpers import (SeqData, check_close, default_scale, history_positions, ps_dtype,
                           to_f64, to_torch)

pytestmark = pytest.mark.gpu


def _bits(x):
    return x.view(torch.int32 if x.dtype == torch.float32 else torch.int16)


def _pair_of_caches(W, P, Hkv, d, dtype, S, src_sd, sds, ts, h0s):
    """`shared`: sequence 0 holds the prefix of src_sd, 1..S-1 share it;
    `private`: every sequence holds its own copy of the same prefix rows.
    Both then get the windows of sds[s] as they stand before ts[s]."""
    kp, vp = to_torch(src_sd.k(0, P)), to_torch(src_sd.v(0, P))
    shared = Cache(W, P, Hkv, d, ps_dtype(dtype), S)
    private = Cache(W, P, Hkv, d, ps_dtype(dtype), S)
    for s in range(S):
        shared.seq_reset(s, h0s[s])
        private.seq_reset(s, h0s[s])
        if s == 0:
            shared.prefill_prefix(0, kp, vp, P)
        else:
            shared.share_prefix(s, 0)
        private.prefill_prefix(s, kp, vp, P)
    for c in (shared, private):
        for s, (sd, t) in enumerate(zip(sds, ts)):
            n = min(W, t - P)
            if n > 0:
                c.import_window(s, t, to_torch(sd.k(t - n, n)), to_torch(sd.v(t - n, n)), n,
                                h0s[s])
    return shared, private


def test_decode_steps_with_a_shared_prefix():
    W, P, Hq, Hkv, d, S = 256, 160, 8, 2, 128, 5
    src = SeqData(21, 99, Hq, Hkv, d, "bf16")
    sds = [SeqData(21, s, Hq, Hkv, d, "bf16") for s in range(S)]
    ts = [P, P + 5, P + W - 1, P + W + 17, P + 3 * W + 2]
    h0s = [(37 * s) % W for s in range(S)]
    shared, private = _pair_of_caches(W, P, Hkv, d, "bf16", S, src, sds, ts, h0s)
    scale = default_scale(d)
    ids = list(range(S))
    outs = []
    for step in range(3):
        tt = [t + step for t in ts]
        q = torch.stack([to_torch(sd.q(t, 1))[0] for sd, t in zip(sds, tt)])
        kn = torch.stack([to_torch(sd.k(t, 1))[0] for sd, t in zip(sds, tt)])
        vn = torch.stack([to_torch(sd.v(t, 1))[0] for sd, t in zip(sds, tt)])
        a, b = torch.empty_like(q), torch.empty_like(q)
        shared.decode_step(q, kn, vn, ids, tt, Hq, scale, a)
        private.decode_step(q, kn, vn, ids, tt, Hq, scale, b)
        assert torch.equal(_bits(a), _bits(b)), f"shared and private prefixes differ at step {step}"
        outs.append((tt, q, a))
    assert shared.device_error() == 0 and private.device_error() == 0
    # oracle: prefix rows of the source sequence, window rows of each sequence
    Kp, Vp = synth.to_f64(src.k(0, P)), synth.to_f64(src.v(0, P))
    G = Hq // Hkv
    tt, q, a = outs[-1]
    batch = oracle.Batch()
    exp = []
    for s, (sd, t) in enumerate(zip(sds, tt)):
        hp = history_positions(P, W, t)
        win = hp[hp >= P]
        K = np.concatenate([Kp, synth.to_f64(sd.k(int(win[0]), len(win)))]) if len(win) else Kp
        V = np.concatenate([Vp, synth.to_f64(sd.v(int(win[0]), len(win)))]) if len(win) else Vp
        q64 = to_f64(q[s])
        exp.append([batch.add(P, W, t, scale, q64[g * G:(g + 1) * G], hp,
                              np.ascontiguousarray(K[:, g]), np.ascontiguousarray(V[:, g]))
                    for g in range(Hkv)])
    batch.run()
    exp = np.stack([np.concatenate(e, axis=0) for e in exp])
    check_close(to_f64(a), exp, "bf16", "shared-prefix decode")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_chunk_and_prompt_with_a_shared_prefix(dtype, d):
    W, P, Hq, Hkv, S = 128, 300, 4, 2, 3
    src = SeqData(22, 50, Hq, Hkv, d, dtype)
    sds = [SeqData(22, s, Hq, Hkv, d, dtype) for s in range(S)]
    ts = [P + 40, P + 400, P]
    h0s = [5, 77, 0]
    shared, private = _pair_of_caches(W, P, Hkv, d, dtype, S, src, sds, ts, h0s)
    scale = default_scale(d)
    n = 200
    for s, (sd, t0) in enumerate(zip(sds, ts)):
        q, kb, vb = to_torch(sd.q(t0, n)), to_torch(sd.k(t0, n)), to_torch(sd.v(t0, n))
        a, b = torch.empty_like(q), torch.empty_like(q)
        shared.attend_chunk(s, q, kb, vb, t0, n, Hq, scale, a)
        private.attend_chunk(s, q, kb, vb, t0, n, Hq, scale, b)
        assert torch.equal(_bits(a), _bits(b)), f"chunk of sequence {s}"
    qp = to_torch(src.q(0, P))
    a, b = torch.empty_like(qp), torch.empty_like(qp)
    shared.attend_prompt(2, qp, 0, P, Hq, scale, a)   # a sharer
    private.attend_prompt(2, qp, 0, P, Hq, scale, b)
    assert torch.equal(_bits(a), _bits(b))
    assert shared.device_error() == 0 and private.device_error() == 0


def test_sharing_rules():
    W, P, Hkv, d = 8, 4, 1, 64
    c = Cache(W, P, Hkv, d, ps_dtype("f32"), 4)
    sd = SeqData(23, 0, 2, Hkv, d, "f32")
    c.prefill_prefix(0, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)

    def code(fn, *a):
        with pytest.raises(PSError) as e:
            fn(*a)
        return e.value.code

    assert code(c.share_prefix, 1, 2) == PS_ESTATE    # source has no prefix
    assert code(c.share_prefix, 0, 0) == PS_EINVAL    # itself
    c.share_prefix(1, 0)
    c.share_prefix(2, 1)                             # from a sharer: reads sequence 0's rows
    assert c.seq_info(2).P == P and c.seq_info(2).next_pos == P
    assert code(c.share_prefix, 1, 0) == PS_ESTATE    # target not empty
    assert code(c.seq_reset, 0, 0) == PS_ESTATE       # two sequences read its prefix
    c.seq_reset(1, 0)
    assert code(c.seq_reset, 0, 0) == PS_ESTATE       # one still does
    c.seq_reset(2, 0)
    c.seq_reset(0, 0)                                 # released
    assert c.seq_info(0).state == 0
    assert c.device_error() == 0

"""GPU parity of the batched chunk and prompt calls (ps_attend_chunk_batch,
ps_attend_prompt_batch): one launch over several sequences, rows packed end
to end, gives bit for bit the outputs of one call per sequence -- on the
tensor-core kernel (with more query-tile CTAs than SMs, so the launch runs in
several waves across sequences) and on the CUDA-core kernel -- appends the
same rows to the rings, matches the oracle on sampled rows, and rejects a bad
batch before anything runs."""
import numpy as np
import pytest
import torch

import oracle
from prefix_sliding_window_ring_b200 import PS_EINVAL, PS_ENOMEM, PS_EPOS, Cache, PSError
from tests.helpers import (SeqData, check_close, default_scale, expected_window, history_positions,
                           history_rows, ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu


def _bits(x):
    return x.view(torch.int32 if x.dtype == torch.float32 else torch.int16)


def _setup(dtype, d, Hq, Hkv, W, P, starts, heads, page=0, seed=41):
    """Two identical caches.  Small blocks stay on the chunk kernels (bound 0):
    a call takes the split decode path for small blocks only when all its
    blocks are small, so a batch and its single calls may take different paths
    (tests/test_gpu_chunk_small.py covers that path)."""
    S = len(starts)
    sds = [SeqData(seed, s, Hq, Hkv, d, dtype) for s in range(S)]
    caches = []
    for _ in range(2):
        c = Cache(W, P, Hkv, d, ps_dtype(dtype), S, page_rows=page,
                  num_pages=S * (W // page) if page else 0)
        c.set_chunk_small_max(0)
        for s, (sd, t) in enumerate(zip(sds, starts)):
            c.seq_reset(s, heads[s])
            c.prefill_prefix(s, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
            nw = min(W, t - P)
            if nw > 0:
                c.import_window(s, t, to_torch(sd.k(t - nw, nw)), to_torch(sd.v(t - nw, nw)), nw,
                                heads[s])
        caches.append(c)
    return sds, caches


# dtype, d, Hq, Hkv, W, P, page_rows, block lengths.  The tensor-core cases have
# 182 query-tile CTAs (more than the 148 SMs: the launch runs in waves that mix
# sequences), while each sequence alone has fewer.
CASES = [
    ("bf16", 128, 4, 2, 512, 96, 0, [3000, 0, 129, 2500, 63]),
    ("bf16", 128, 8, 1, 256, 40, 128, [2000, 0, 129, 700, 63]),
    ("f32", 64, 4, 2, 48, 6, 0, [90, 0, 33, 70, 5]),
]


@pytest.mark.parametrize("dtype,d,Hq,Hkv,W,P,page,ns", CASES,
                         ids=[f"{c[0]}-d{c[1]}-G{c[2] // c[3]}-W{c[4]}-pg{c[6]}" for c in CASES])
@pytest.mark.parametrize("append", [0, 1])
def test_chunk_batch_equals_one_call_per_sequence(dtype, d, Hq, Hkv, W, P, page, ns, append):
    starts = [P, P + 7, P + W - 3, P + 3 * W + 11, P + 1]
    heads = [0, 5 % W, W - 1, W // 2, 1]
    sds, (one, bat) = _setup(dtype, d, Hq, Hkv, W, P, starts, heads, page)
    scale = default_scale(d)
    q = torch.cat([to_torch(sd.q(t, n)) for sd, t, n in zip(sds, starts, ns)])
    kb = torch.cat([to_torch(sd.k(t, n)) for sd, t, n in zip(sds, starts, ns)])
    vb = torch.cat([to_torch(sd.v(t, n)) for sd, t, n in zip(sds, starts, ns)])
    out_b = torch.full_like(q, 7.0)
    bat.attend_chunk_batch(list(range(len(ns))), starts, ns, q, kb, vb, Hq, scale, out_b, append)
    out_1 = torch.full_like(q, 7.0)
    r0 = 0
    for s, (t, n) in enumerate(zip(starts, ns)):
        if n:
            one.attend_chunk(s, q[r0:r0 + n], kb[r0:r0 + n], vb[r0:r0 + n], t, n, Hq, scale,
                             out_1[r0:r0 + n], append)
        r0 += n
    torch.cuda.synchronize()
    assert one.device_error() == 0 and bat.device_error() == 0
    assert torch.equal(_bits(out_b), _bits(out_1))
    for s, (t, n) in enumerate(zip(starts, ns)):
        a_, b_ = one.seq_info(s), bat.seq_info(s)
        assert (a_.next_pos, a_.head, a_.count) == (b_.next_pos, b_.head, b_.count)
        assert a_.next_pos == t + (n if append else 0)
        ka, va, pa = one.export_window(s)
        kb2, vb2, pb = bat.export_window(s)
        assert pa.tolist() == pb.tolist() == expected_window(P, W, a_.next_pos)
        assert torch.equal(_bits(ka), _bits(kb2)) and torch.equal(_bits(va), _bits(vb2))
    # sampled rows of the batch output against the oracle
    G = Hq // Hkv
    batch = oracle.Batch()
    exp, got = [], []
    r0 = 0
    for s, (sd, t, n) in enumerate(zip(sds, starts, ns)):
        for i in sorted({0, n // 2, n - 1}) if n else []:
            tq = t + i
            hp = history_positions(P, W, tq)
            K, V = history_rows(sd, hp)
            q64 = to_f64(q[r0 + i])
            exp.append([batch.add(P, W, tq, scale, q64[g * G:(g + 1) * G], hp,
                                  np.ascontiguousarray(K[:, g]), np.ascontiguousarray(V[:, g]))
                        for g in range(Hkv)])
            got.append(to_f64(out_b[r0 + i]))
        r0 += n
    batch.run()
    check_close(np.stack(got), np.stack([np.concatenate(e, axis=0) for e in exp]), dtype,
                "batched chunk")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_prompt_batch_equals_one_call_per_sequence(dtype, d):
    Hq, Hkv, W, P = 4, 2, 128, 1500 if dtype == "bf16" else 150
    starts = [0, 0, 0, 0]
    sds, (one, bat) = _setup(dtype, d, Hq, Hkv, W, P, [P] * 4, [0, 3, 9, 100])
    scale = default_scale(d)
    t0s = [0, 37, 0, P - 1]
    ns = [P, P - 37 - 1, 0, 1]
    q = torch.cat([to_torch(sd.q(t, n)) for sd, t, n in zip(sds, t0s, ns)])
    out_b = torch.full_like(q, 7.0)
    bat.attend_prompt_batch([0, 1, 2, 3], t0s, ns, q, Hq, scale, out_b)
    out_1 = torch.full_like(q, 7.0)
    r0 = 0
    for s, (t, n) in enumerate(zip(t0s, ns)):
        if n:
            one.attend_prompt(s, q[r0:r0 + n], t, n, Hq, scale, out_1[r0:r0 + n])
        r0 += n
    torch.cuda.synchronize()
    assert torch.equal(_bits(out_b), _bits(out_1))
    assert one.device_error() == 0 and bat.device_error() == 0
    del starts


def test_many_entries_span_several_launches():
    # more entries than one launch takes (64): the batch is split, results unchanged
    W, P, Hq, Hkv, d, S = 256, 16, 2, 1, 128, 70
    starts = [P + (s % 5) * 97 for s in range(S)]
    sds, (one, bat) = _setup("bf16", d, Hq, Hkv, W, P, starts, [s % W for s in range(S)])
    ns = [1 + (7 * s) % 40 for s in range(S)]
    scale = default_scale(d)
    q = torch.cat([to_torch(sd.q(t, n)) for sd, t, n in zip(sds, starts, ns)])
    kb = torch.cat([to_torch(sd.k(t, n)) for sd, t, n in zip(sds, starts, ns)])
    vb = torch.cat([to_torch(sd.v(t, n)) for sd, t, n in zip(sds, starts, ns)])
    out_b = torch.empty_like(q)
    bat.attend_chunk_batch(list(range(S)), starts, ns, q, kb, vb, Hq, scale, out_b, 1)
    out_1 = torch.empty_like(q)
    r0 = 0
    for s, (t, n) in enumerate(zip(starts, ns)):
        one.attend_chunk(s, q[r0:r0 + n], kb[r0:r0 + n], vb[r0:r0 + n], t, n, Hq, scale,
                         out_1[r0:r0 + n], 1)
        r0 += n
    torch.cuda.synchronize()
    assert torch.equal(_bits(out_b), _bits(out_1))
    assert all(bat.seq_info(s).next_pos == starts[s] + ns[s] for s in range(S))
    assert bat.device_error() == 0


def test_bad_batches_change_nothing():
    W, P, Hq, Hkv, d = 128, 8, 2, 1, 128
    starts = [P + 10, P + 200]
    sds, (c, _) = _setup("bf16", d, Hq, Hkv, W, P, starts, [0, 0], page=128)
    scale = default_scale(d)
    n = [20, 30]
    q = torch.cat([to_torch(sd.q(t, m)) for sd, t, m in zip(sds, starts, n)])
    kb = torch.cat([to_torch(sd.k(t, m)) for sd, t, m in zip(sds, starts, n)])
    out = torch.empty_like(q)
    before = [(c.seq_info(s).next_pos, c.seq_info(s).count) for s in range(2)]

    def code(*args):
        with pytest.raises(PSError) as e:
            c.attend_chunk_batch(*args)
        return e.value.code

    assert code([0, 0], starts, n, q, kb, kb, Hq, scale, out, 1) == PS_EINVAL   # repeated id
    assert code([0, 1], [starts[0], starts[1] + 1], n, q, kb, kb, Hq, scale, out, 1) == PS_EPOS
    assert code([0, 1], starts, [20, -1], q, kb, kb, Hq, scale, out, 1) == PS_EINVAL
    free = c.ring_pages_free()
    assert free == 0  # both rings hold a page already; the pool had exactly two pages
    # sequence 0 fills its ring slot by slot: appending 20 rows at slot 10 stays in its page,
    # sequence 1's ring is full: no new page either, so this batch succeeds ...
    c.attend_chunk_batch([0, 1], starts, n, q, kb, kb, Hq, scale, out, 1)
    after = [(c.seq_info(s).next_pos, c.seq_info(s).count) for s in range(2)]
    assert after == [(before[0][0] + 20, before[0][1] + 20), (before[1][0] + 30, W)]
    assert c.device_error() == 0


def test_batch_exhausting_the_page_pool_changes_nothing():
    W, P, Hq, Hkv, d, page = 256, 8, 2, 1, 128, 128
    sds = [SeqData(43, s, Hq, Hkv, d, "bf16") for s in range(2)]
    c = Cache(W, P, Hkv, d, ps_dtype("bf16"), 2, page_rows=page, num_pages=3)
    for s, sd in enumerate(sds):
        c.prefill_prefix(s, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    n = [200, 200]  # two pages each: four pages wanted, three in the pool
    q = torch.cat([to_torch(sd.q(P, m)) for sd, m in zip(sds, n)])
    kb = torch.cat([to_torch(sd.k(P, m)) for sd, m in zip(sds, n)])
    out = torch.empty_like(q)
    with pytest.raises(PSError) as e:
        c.attend_chunk_batch([0, 1], [P, P], n, q, kb, kb, Hq, default_scale(d), out, 1)
    assert e.value.code == PS_ENOMEM
    assert c.ring_pages_free() == 3
    assert [c.seq_info(s).next_pos for s in range(2)] == [P, P]
    c.attend_chunk_batch([0], [P], [200], q[:200], kb[:200], kb[:200], Hq, default_scale(d),
                         out[:200], 1)
    assert c.ring_pages_free() == 1 and c.device_error() == 0

"""GPU parity of the paged ring (ps_cache_create_paged): the same sequence of
calls on a paged cache and on an unpaged one gives bit-identical outputs and
windows -- decode steps, bulk appends, window imports, chunks with appends on
both chunk kernels, prompt attention -- and matches the oracle; pages are taken
only when a slot is first written, return on reset, and an exhausted pool
fails cleanly."""
import numpy as np
import pytest
import torch

import oracle
from prefix_sliding_window_ring_b200 import PS_ENOMEM, Cache, PSError
from tests.helpers import (SeqData, check_close, default_scale, expected_window, oracle_decode,
                           ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu


def _bits(x):
    return x.view(torch.int32 if x.dtype == torch.float32 else torch.int16)


CASES = [  # dtype, d, G, Hkv, W, P, page_rows (bf16 d=128: tensor-core chunks; else CUDA cores)
    ("bf16", 128, 2, 2, 512, 96, 128),
    ("bf16", 128, 4, 2, 256, 40, 256),
    ("f32", 64, 2, 2, 40, 6, 8),
    ("bf16", 64, 1, 2, 48, 5, 16),
]


@pytest.mark.parametrize("dtype,d,G,Hkv,W,P,page", CASES,
                         ids=[f"{c[0]}-d{c[1]}-G{c[2]}-W{c[4]}-pg{c[6]}" for c in CASES])
def test_paged_equals_unpaged(dtype, d, G, Hkv, W, P, page):
    Hq, S = G * Hkv, 3
    scale = default_scale(d)
    sds = [SeqData(31, s, Hq, Hkv, d, dtype) for s in range(S)]
    plain = Cache(W, P, Hkv, d, ps_dtype(dtype), S)
    paged = Cache(W, P, Hkv, d, ps_dtype(dtype), S, page_rows=page, num_pages=S * (W // page))
    npages = S * (W // page)
    h0s = [0, W // 3, W - 1]
    t_imp = P + W + 17          # sequence 1 gets its window by import
    for c in (plain, paged):
        for s, sd in enumerate(sds):
            c.seq_reset(s, h0s[s])
            c.prefill_prefix(s, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
        n = min(W, t_imp - P)
        c.import_window(1, t_imp, to_torch(sds[1].k(t_imp - n, n)), to_torch(sds[1].v(t_imp - n, n)),
                        n, h0s[1])
    assert paged.ring_pages_free() == npages - W // page   # only the imported window took pages
    nxt = [P, t_imp, P]
    outs = {"plain": [], "paged": []}

    def run(c, key):
        pos = list(nxt)
        # bulk append to sequences 0 and 2 (17 tokens), then decode steps for all three
        k17 = torch.stack([to_torch(sds[s].k(pos[s], 17)) for s in (0, 2)])
        v17 = torch.stack([to_torch(sds[s].v(pos[s], 17)) for s in (0, 2)])
        c.append_kv([0, 2], k17, v17, 17)
        pos[0] += 17
        pos[2] += 17
        for step in range(4):
            q = torch.stack([to_torch(sd.q(p, 1))[0] for sd, p in zip(sds, pos)])
            kn = torch.stack([to_torch(sd.k(p, 1))[0] for sd, p in zip(sds, pos)])
            vn = torch.stack([to_torch(sd.v(p, 1))[0] for sd, p in zip(sds, pos)])
            o = torch.empty_like(q)
            c.decode_step(q, kn, vn, [0, 1, 2], pos, Hq, scale, o)
            outs[key].append(o)
            pos = [p + 1 for p in pos]
        # a chunk with append on sequence 2 (crosses the window fill and pages)
        n = W // 2 + 3
        qb, kb, vb = to_torch(sds[2].q(pos[2], n)), to_torch(sds[2].k(pos[2], n)), to_torch(sds[2].v(pos[2], n))
        ob = torch.empty_like(qb)
        c.attend_chunk(2, qb, kb, vb, pos[2], n, Hq, scale, ob, append_after=1)
        outs[key].append(ob)
        pos[2] += n
        # prompt attention of sequence 0
        qp = to_torch(sds[0].q(0, P))
        op = torch.empty_like(qp)
        c.attend_prompt(0, qp, 0, P, Hq, scale, op)
        outs[key].append(op)
        return pos

    pos_a = run(plain, "plain")
    pos_b = run(paged, "paged")
    assert pos_a == pos_b
    assert plain.device_error() == 0 and paged.device_error() == 0
    for a, b in zip(outs["plain"], outs["paged"]):
        assert torch.equal(_bits(a), _bits(b))
    for s in range(S):
        ka, va, pa = plain.export_window(s)
        kb_, vb_, pb = paged.export_window(s)
        assert pa.tolist() == pb.tolist() == expected_window(P, W, pos_a[s])
        assert torch.equal(_bits(ka), _bits(kb_)) and torch.equal(_bits(va), _bits(vb_))
    # the last decode step against the oracle
    last = outs["paged"][3]
    tl = [p - 1 for p in (pos_a[0], pos_a[1], pos_a[2] - (W // 2 + 3))]
    batch = oracle.Batch()
    exp = [oracle_decode(batch, sd, P, W, t, scale, to_f64(q))
           for sd, t, q in zip(sds, tl, [to_torch(sd.q(t, 1))[0] for sd, t in zip(sds, tl)])]
    batch.run()
    exp = np.stack([np.concatenate(e, axis=0) for e in exp])
    check_close(to_f64(last), exp, dtype, "paged decode")


def test_page_pool_accounting_and_exhaustion():
    W, P, Hkv, d, page = 32, 2, 1, 64, 8
    c = Cache(W, P, Hkv, d, ps_dtype("f32"), 3, page_rows=page, num_pages=5)
    sds = [SeqData(32, s, 2, Hkv, d, "f32") for s in range(3)]
    for s, sd in enumerate(sds):
        c.prefill_prefix(s, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    assert c.ring_pages_free() == 5                   # nothing written to a ring yet
    c.append_kv([0], to_torch(sds[0].k(P, 9)).unsqueeze(0), to_torch(sds[0].v(P, 9)).unsqueeze(0), 9)
    assert c.ring_pages_free() == 3                   # slots 0..8: two pages
    c.append_kv([0], to_torch(sds[0].k(P + 9, 40)).unsqueeze(0),
                to_torch(sds[0].v(P + 9, 40)).unsqueeze(0), 40)
    assert c.ring_pages_free() == 1                   # the whole ring: four pages
    with pytest.raises(PSError) as e:                 # 9 tokens for sequence 1 need two pages
        c.append_kv([1], to_torch(sds[1].k(P, 9)).unsqueeze(0),
                    to_torch(sds[1].v(P, 9)).unsqueeze(0), 9)
    assert e.value.code == PS_ENOMEM
    info = c.seq_info(1)
    assert (info.next_pos, info.count) == (P, 0) and c.ring_pages_free() == 1
    c.seq_reset(0, 0)                                 # four pages back
    assert c.ring_pages_free() == 5
    c.append_kv([1], to_torch(sds[1].k(P, 9)).unsqueeze(0), to_torch(sds[1].v(P, 9)).unsqueeze(0), 9)
    assert c.ring_pages_free() == 3
    _, _, pos = c.export_window(1)
    assert pos.tolist() == expected_window(P, W, P + 9)
    assert c.device_error() == 0

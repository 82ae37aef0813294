"""GPU parity of chunked prefill/extend (ps_attend_chunk): small shapes with every
output element checked, and the full-size workload (4 sequences, 2048-query
blocks at t0=100000, W in {4096, 16384}): every row at W=4096, sampled query
rows at W=16384."""
import numpy as np
import pytest
import torch

import oracle
import synth
from prefix_sliding_window_ring_b200 import Cache
from synth import workloads
from tests.helpers import (EVICTED_MARGIN, SeqData, check_close, default_scale, expected_window,
                           history_rows, ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu


def chunk_history(P, W, t0, n, i_rows):
    """Prefix plus every position from the lowest window start (minus an evicted
    margin) to the end of the block; the oracle masks what each query must not see."""
    lo = max(P, t0 + min(i_rows) - W + 1 - EVICTED_MARGIN)
    return np.concatenate([np.arange(0, P), np.arange(lo, t0 + n)]).astype(np.int64)


def run_chunk(W, P, L, n, dtype, d, G, Hkv=2, seed=0, rows=None, seqs=1, h0=0, append=True,
              batched=False, page=0):
    """batched: all sequences' blocks in one ps_attend_chunk_batch call (the
    launch the benchmark times); otherwise one ps_attend_chunk call each.
    page > 0: a paged ring of page-row pages."""
    Hq = G * Hkv
    scale = default_scale(d)
    kw = dict(page_rows=page, num_pages=seqs * (W // page)) if page else {}
    c = Cache(W, max(P, 1), Hkv, d, ps_dtype(dtype), seqs, **kw)
    t0 = P + L
    sds = [SeqData(seed, s, Hq, Hkv, d, dtype) for s in range(seqs)]
    outs, qs, kbs, vbs = [], [], [], []
    for s, sd in enumerate(sds):
        c.seq_reset(s, 0)
        c.prefill_prefix(s, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
        nw = min(W, L)
        c.import_window(s, t0, to_torch(sd.k(t0 - nw, nw)), to_torch(sd.v(t0 - nw, nw)), nw,
                        (h0 + 31 * s) % W)
        q = to_torch(sd.q(t0, n))
        kb, vb = to_torch(sd.k(t0, n)), to_torch(sd.v(t0, n))
        if batched:
            kbs.append(kb)
            vbs.append(vb)
        else:
            out = torch.empty_like(q)
            c.attend_chunk(s, q, kb, vb, t0, n, Hq, scale, out, append_after=int(append))
            outs.append(out)
        qs.append(q)
    if batched:
        qall = torch.cat(qs)
        oall = torch.empty_like(qall)
        c.attend_chunk_batch(list(range(seqs)), [t0] * seqs, [n] * seqs, qall, torch.cat(kbs),
                             torch.cat(vbs), Hq, scale, oall, int(append))
        outs = list(oall.split(n))
    assert c.device_error() == 0
    if rows is None:
        rows = list(range(n))
    batch = oracle.Batch()
    exp = []
    for s, sd in enumerate(sds):
        hp = chunk_history(P, W, t0, n, rows)
        K, V = history_rows(sd, hp)
        # one contiguous copy per kv head, shared by every query's problem
        Kg = [np.ascontiguousarray(K[:, g]) for g in range(Hkv)]
        Vg = [np.ascontiguousarray(V[:, g]) for g in range(Hkv)]
        del K, V
        q64 = to_f64(qs[s])
        per = []
        for i in rows:
            for g in range(Hkv):
                per.append(batch.add(P, W, t0 + i, scale, q64[i, g * G:(g + 1) * G], hp,
                                     Kg[g], Vg[g]))
        exp.append(per)
    batch.run()
    got = np.stack([to_f64(o)[rows] for o in outs])
    want = np.stack([np.stack([np.concatenate(e[r * Hkv:(r + 1) * Hkv], axis=0)
                               for r in range(len(rows))]) for e in exp])
    stats = check_close(got, want, dtype, f"chunk W={W} P={P} L={L} n={n} {dtype}")
    if append:
        for s in range(seqs):
            _, _, pos = c.export_window(s)
            assert pos.cpu().tolist() == expected_window(P, W, t0 + n)
            info = c.seq_info(s)
            assert info.next_pos == t0 + n
    return stats


SMALL = [
    # W, P, L (window tokens before the block), n, dtype, d, G
    (5, 3, 0, 7, "f32", 64, 2),
    (5, 3, 2, 3, "bf16", 128, 2),
    (37, 0, 100, 50, "f32", 128, 1),
    (37, 17, 20, 100, "bf16", 64, 4),
    (128, 16, 1000, 300, "bf16", 128, 2),
    (129, 100, 129, 129, "f32", 128, 2),
    (1, 0, 5, 4, "bf16", 128, 2),
    (64, 5, 3, 1, "f32", 64, 8),
    (300, 40, 700, 260, "bf16", 128, 2),
    (256, 128, 256, 384, "bf16", 128, 2),
    # window not yet full before, and inside, the block (tensor-core kernel)
    (512, 64, 0, 700, "bf16", 128, 4),
    (4096, 256, 100, 2048, "bf16", 128, 2),
    (4096, 128, 3000, 2048, "bf16", 128, 2),
]


@pytest.mark.parametrize("W,P,L,n,dtype,d,G", SMALL)
def test_chunk_small(W, P, L, n, dtype, d, G):
    run_chunk(W, P, L, n, dtype, d, G)


@pytest.mark.parametrize("W", workloads.CHUNK["W_values"])
def test_chunk_full_size(W):
    """The chunk workload at full size, the four blocks in one batched launch as
    the benchmark runs it.  At W=4096 every output row of all four sequences is compared with the oracle
    (65536 problems of about 6.5k history rows each); at W=16384 a sample of rows
    that includes every query-tile edge class."""
    cfg = workloads.CHUNK
    s = cfg["shape_for"](W)
    n, t0 = cfg["n"], cfg["t0"]
    if W == 4096:
        rows = None
    else:
        rng = np.random.default_rng(11)
        rows = sorted(set([0, 1, 2, 63, 64, 127, 128, 129, 1023, 1024, n - 2, n - 1]) |
                      set(rng.integers(0, n, 6).tolist()))
    run_chunk(W, s.P, t0 - s.P, n, s.dtype, s.d, s.G, Hkv=s.Hkv, rows=rows, seqs=cfg["B"],
              h0=1234, append=True, batched=True)


@pytest.mark.parametrize("page", [8, 16, 32, 64])
def test_chunk_small_pages(page):
    """Paged rings whose pages are smaller than a 128-row key tile: the
    tensor-core kernel reads each ring tile as whole pages from a page edge
    (window full and wrapping, then window filling inside the block)."""
    run_chunk(512, 40, 700, 300, "bf16", 128, 2, h0=37, seqs=2, page=page, batched=True)
    run_chunk(256, 24, 100, 200, "bf16", 128, 4, h0=5, page=page)


@pytest.mark.parametrize("W,page", [(200, 8), (344, 8), (208, 16), (320, 64), (448, 64)])
def test_chunk_small_pages_ragged_ring(W, page):
    """A ring that is not a whole number of 128-row key tiles: the last ring
    tile of a run ends inside a tile, and its pages past the ring's end are
    copied as zeros and masked (window full and wrapping; window filling)."""
    run_chunk(W, 16, 3 * W + 11, 150, "bf16", 128, 2, h0=W // 3, seqs=2, page=page, batched=True)
    run_chunk(W, 40, W // 2, 90, "bf16", 128, 1, h0=7, page=page)


def test_chunk_full_size_16_row_pages():
    """The chunk workload (4 sequences x 2048 queries at t0=100000, W=4096) on
    a ring of 16-row pages, sampled rows of every query-tile edge class."""
    cfg = workloads.CHUNK
    s = cfg["shape_for"](4096)
    n, t0 = cfg["n"], cfg["t0"]
    rows = [0, 1, 63, 64, 127, 128, 129, 1023, 1024, n - 2, n - 1]
    run_chunk(4096, s.P, t0 - s.P, n, s.dtype, s.d, s.G, Hkv=s.Hkv, rows=rows, seqs=cfg["B"],
              h0=1234, append=True, batched=True, page=16)

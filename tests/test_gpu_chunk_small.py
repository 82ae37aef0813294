"""GPU parity of small chunk blocks routed to the split decode kernel
(ps_attend_chunk / ps_attend_chunk_batch, bf16: a call whose blocks all have
n <= ps_set_chunk_small_max's bound and whose (group, kv head) pairs fit the
GPU at once): block sizes 1, 2, 3 and the bound -1 / +0 / +1 (the last one
runs on the chunk kernel) on the chunk workload's shape, every GQA size, both
head sizes, windows shorter than the block, windows not yet full, paged rings,
batches that mix small blocks, large blocks and empty entries (the chunk
kernel then takes them all), one call per block, more pairs than fit at once
(the chunk kernel).  Every output row is compared with the oracle ("Prefix
Sliding" digest section 03 rule applied to each query of the block)."""
import numpy as np
import pytest
import torch

import oracle
from prefix_sliding_window_ring_b200 import Cache
from tests.helpers import (EVICTED_MARGIN, SeqData, check_close, default_scale, expected_window,
                           history_rows, ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu

BOUND = 16  # the small-block bound these tests set explicitly


def run_blocks(W, P, blocks, d=128, G=2, Hkv=8, small_max=BOUND, page=0, seed=3, h0=0,
               append=True, single=False):
    """blocks: per sequence (L, n): L window tokens before a block of n
    queries.  All blocks in one ps_attend_chunk_batch call (single: one
    ps_attend_chunk call each); every row checked."""
    dtype = "bf16"
    Hq = G * Hkv
    scale = default_scale(d)
    S = len(blocks)
    kw = {}
    if page:
        kw = dict(page_rows=page, num_pages=S * (W // page))
    c = Cache(W, max(P, 1), Hkv, d, ps_dtype(dtype), S, **kw)
    c.set_chunk_small_max(small_max)
    sds = [SeqData(seed, s, Hq, Hkv, d, dtype) for s in range(S)]
    qs, kbs, vbs, t0s, ns = [], [], [], [], []
    for s, (L, n) in enumerate(blocks):
        sd = sds[s]
        c.seq_reset(s, 0)
        c.prefill_prefix(s, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
        t0 = P + L
        nw = min(W, L)
        c.import_window(s, t0, to_torch(sd.k(t0 - nw, nw)), to_torch(sd.v(t0 - nw, nw)), nw,
                        (h0 + 37 * s) % W)
        qs.append(to_torch(sd.q(t0, n)) if n else torch.empty(0, Hq, d, dtype=torch.bfloat16,
                                                                device="cuda"))
        kbs.append(to_torch(sd.k(t0, n)) if n else torch.empty(0, Hkv, d, dtype=torch.bfloat16,
                                                                 device="cuda"))
        vbs.append(to_torch(sd.v(t0, n)) if n else torch.empty(0, Hkv, d, dtype=torch.bfloat16,
                                                                 device="cuda"))
        t0s.append(t0)
        ns.append(n)
    qall = torch.cat(qs)
    oall = torch.full_like(qall, float("nan"))
    if single:
        r0 = 0
        for s, n in enumerate(ns):
            if n:
                c.attend_chunk(s, qs[s], kbs[s], vbs[s], t0s[s], n, Hq, scale, oall[r0:r0 + n],
                               int(append))
            r0 += n
    else:
        c.attend_chunk_batch(list(range(S)), t0s, ns, qall, torch.cat(kbs), torch.cat(vbs), Hq,
                             scale, oall, int(append))
    assert c.device_error() == 0
    got = to_f64(oall)
    batch = oracle.Batch()
    exp = []
    for s, (L, n) in enumerate(blocks):
        if n == 0:
            continue
        t0 = t0s[s]
        lo = max(P, t0 - W + 1 - EVICTED_MARGIN)
        hp = np.concatenate([np.arange(0, P), np.arange(lo, t0 + n)]).astype(np.int64)
        K, V = history_rows(sds[s], hp)
        Kg = [np.ascontiguousarray(K[:, g]) for g in range(Hkv)]
        Vg = [np.ascontiguousarray(V[:, g]) for g in range(Hkv)]
        q64 = to_f64(qs[s])
        for i in range(n):
            for g in range(Hkv):
                exp.append(batch.add(P, W, t0 + i, scale, q64[i, g * G:(g + 1) * G], hp, Kg[g],
                                     Vg[g]))
    batch.run()
    N = sum(ns)
    want = np.stack([np.concatenate(exp[r * Hkv:(r + 1) * Hkv], axis=0) for r in range(N)])
    check_close(got, want, dtype, f"small chunk W={W} P={P} blocks={blocks} G={G} d={d}")
    if append:
        for s, (L, n) in enumerate(blocks):
            _, _, pos = c.export_window(s)
            assert pos.cpu().tolist() == expected_window(P, W, t0s[s] + n)
    c.close()


@pytest.mark.parametrize("n", [1, 2, 3, BOUND - 1, BOUND, BOUND + 1])
def test_block_sizes_around_the_bound(n):
    """The chunk workload's shape (4 sequences, Hq=16, Hkv=8, d=128, P=256,
    W=4096, window full) at block sizes 1, 2, 3 and bound-1 / bound (split
    decode) and bound+1 (chunk kernel)."""
    run_blocks(4096, 256, [(100000 - 256, n)] * 4, h0=1234)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
def test_gqa_and_head_sizes(G, d):
    run_blocks(300, 40, [(700, 5), (20, 9), (300, 1)], d=d, G=G, Hkv=2)


@pytest.mark.parametrize("W,P,L,n", [
    (1, 0, 5, 4),      # a one-slot window: each query sees only itself
    (3, 2, 10, 9),     # the window shorter than the block
    (5, 3, 2, 7),      # window not yet full before the block, full inside it
    (8, 0, 0, 8),      # no history at all before the block
    (64, 16, 63, 16),  # the block starts as the window fills
])
def test_short_windows_and_edges(W, P, L, n):
    run_blocks(W, P, [(L, n), (L + 3, max(1, n - 2))], Hkv=2, small_max=32)


@pytest.mark.parametrize("page", [4, 8, 16, 256])
def test_paged_ring(page):
    """Pages of 4 rows start an atom each (their own layout); 8, 16 and 256
    keep the unpaged one."""
    run_blocks(512, 64, [(1000, 3), (37, 12), (600, 1)], Hkv=4, page=page, h0=77)


def test_paged_ring_non_power_of_two_pages():
    """24-row pages: a multiple of 8 (the unpaged layout) whose page numbers
    need a division, not a shift."""
    run_blocks(480, 40, [(900, 5), (100, 9), (481, 1)], Hkv=4, page=24, h0=13)


def test_mixed_batch():
    """Small blocks, a chunk-kernel block and empty entries in one call: the
    two paths split the batch, each entry's rows stay in place."""
    run_blocks(1024, 128, [(2000, 3), (500, 200), (0, 0), (1500, 16), (900, 1), (10, 0),
                           (4000, 130)], Hkv=4, h0=5)


def test_every_block_on_the_split_path_and_none():
    """The same inputs with the bound at 0 (all chunk kernel) and at 64 (all
    split decode) both match the oracle."""
    for bound in (0, 64):
        run_blocks(512, 32, [(800, 40), (300, 64), (50, 7)], Hkv=4, small_max=bound, seed=8)


def test_one_call_per_block():
    run_blocks(700, 50, [(900, 3), (120, 16), (2000, 1), (10, 7)], Hkv=4, single=True, seed=4)


def test_more_pairs_than_fit_at_once():
    """24 sequences x 16 queries x 8 kv heads = 768 (group, head) pairs, more
    than the GPU holds at once: the call runs on the chunk kernel."""
    run_blocks(512, 16, [(600 + 13 * s, 16) for s in range(24)], small_max=64, seed=6)

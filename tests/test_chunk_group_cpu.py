"""Chunk mode of the tensor-core decode kernel (small chunk blocks), compiled
from the library's header as host code and run on the CPU.  A pair is a group
of nq consecutive queries of a block at t0 + i0 + k and one kv head; its tiles
hold the union of the group's visible sets and a per-row query mask cuts it
back.  For many ring states, block offsets and group sizes: for every query of
the group, the rows whose mask admits it are exactly the rows the query sees
("Prefix Sliding" digest section 03 rule, 0-indexed: the prefix, the window
[max(P, t - W + 1), t] with the block's own rows causal), each once; ring
pieces hold positions the ring still has, block pieces rows of the block up
to the group's last query; the atoms a piece's copy writes hold no other
piece's rows; a tile copied whole never needs a query mask."""
import os
import random
import shutil
import subprocess
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "native", "chunk_group_harness.cu")
CSRC = os.path.join(ROOT, "prefix_sliding_window_ring_b200", "csrc")
RUN_PREFIX, RUN_RING, RUN_NEW, RUN_BLK = 0, 1, 2, 3


def pad8(x):
    return (x + 7) // 8 * 8


@pytest.fixture(scope="module")
def layout():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    d = tempfile.mkdtemp(prefix="cgroup")
    exe = os.path.join(d, "chunk_group_harness")
    subprocess.check_call([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", CSRC, HARNESS, "-o", exe])

    def run(cases):
        text = "\n".join(" ".join(str(v) for v in c) for c in cases) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        res = []
        for line in out.strip().split("\n"):
            parts = line.split("|")
            head = [int(x) for x in parts[0].split()]
            tiles, wholes = [], []
            for t in parts[1:]:
                pieces, w = [], None
                for p in t.split():
                    if p.startswith("W"):
                        w = tuple(int(v) for v in p[1:].split(","))
                        continue
                    f = p.split(",")
                    masks = [int(v) for v in f[4].split(":")]
                    pieces.append((int(f[0]), int(f[1]), int(f[2]), int(f[3]), masks))
                tiles.append(pieces)
                wholes.append(w)
            assert len(tiles) == head[0]
            res.append((head, tiles, wholes))
        return res
    yield run
    shutil.rmtree(d, ignore_errors=True)


def _check(case, head, tiles, wholes):
    P, W, h0, count, t0, i0, nq, page, TR, csize = case
    ntiles, rows, padded, ring_ok = head
    assert ring_ok == 1
    base = t0 - count
    seen = [[] for _ in range(nq)]
    for j, pieces in enumerate(tiles):
        end = 0
        for src, row, sr, n, masks in pieces:
            assert len(masks) == n
            lead = sr % 8
            assert n >= 1 and sr - lead >= end, ("atoms shared", case, j)
            assert pad8(sr + n) <= TR, case
            end = pad8(sr + n)
            if src == RUN_PREFIX:
                assert 0 <= row and row + n <= P, case
                pos = list(range(row, row + n))
            elif src == RUN_RING:
                assert 0 <= row and row + n <= W, ("ring piece wraps", case)
                if page:
                    assert row // page == (row + n - 1) // page, ("crosses a page", case)
                pos0 = base + (row - h0) % W
                assert base <= pos0 and pos0 + n <= t0, ("not in the ring", case)
                pos = list(range(pos0, pos0 + n))
            else:
                assert src == RUN_BLK, case
                assert 0 <= row and row + n <= i0 + nq, ("block row", case)
                pos = [t0 + row + r for r in range(n)]
            for p, m in zip(pos, masks):
                for k in range(nq):
                    if (m >> k) & 1:
                        seen[k].append(p)
    for k in range(nq):
        need = [int(p) for p in oracle.visible_positions(P, W, t0 + i0 + k)]
        assert len(seen[k]) == len(set(seen[k])), ("a row counted twice", case, k)
        assert sorted(seen[k]) == need, ("coverage", case, k)
    if not csize:
        assert ntiles == (padded + TR - 1) // TR
    for pieces, w in zip(tiles, wholes):
        if w is not None:
            assert len(pieces) == 1 and pieces[0][:4] == (w[0], w[1], 0, TR), case
            assert all(m == 0xff for m in pieces[0][4]), case


def _cases(rng, n):
    out = []
    for _ in range(n):
        W = rng.choice([1, 2, 3, 7, 8, 9, 16, 63, 64, 65, 128, 130, 300, 1024, 4096])
        P = rng.choice([0, 1, 7, 8, 9, 37, 64, 128, 300])
        pages = [0] + [p for p in (1, 2, 4, 8, 16, 24, 64, 128, 256) if W % p == 0 and p <= W]
        page = rng.choice(pages)
        t0 = P + rng.randrange(0, 3 * W + 200)   # next_pos before the block
        count = min(W, t0 - P)
        h0 = rng.randrange(W)
        nblock = rng.choice([1, 2, 3, 4, 5, 8, 9, 16, 17, 40])
        cols = rng.choice([1, 2, 4, 8])
        gq = rng.choice([g for g in (1, 2, 4, 8) if g <= cols])
        Q = cols // gq
        i0 = rng.randrange(0, nblock, Q) if nblock > Q else 0
        nq = min(Q, nblock - i0)
        TR = 64
        csize = rng.choice([0, 0, 2, 4, 8])
        out.append((P, W, h0, count, t0, i0, nq, page, TR, csize))
    return out


def test_chunk_groups_see_exactly_their_rows(layout):
    rng = random.Random(29)
    cases = _cases(rng, 4000)
    for case, (head, tiles, wholes) in zip(cases, layout(cases)):
        _check(case, head, tiles, wholes)


def test_chunk_group_edge_states(layout):
    """Windows shorter than the group, window not yet full / just full / first
    eviction, every head offset of small rings, groups at the start, middle
    and end of a block, the chunk workload's shape."""
    cases = []
    for W in (1, 2, 3, 5, 8, 9):
        for P in (0, 3, 8):
            for t0 in range(P, P + 2 * W + 3):
                for h0 in range(W):
                    for i0, nq in ((0, 1), (0, 4), (3, 4), (0, 8), (5, 3)):
                        cases.append((P, W, h0, min(W, t0 - P), t0, i0, nq, 0, 64, 0))
    for h0 in (0, 1, 613, 4095):
        for page in (0, 16, 256):
            for i0, nq in ((0, 4), (4, 4), (12, 4), (0, 1), (7, 1)):
                for cs in (0, 2, 8):
                    cases.append((256, 4096, h0, 4096, 100000, i0, nq, page, 64, cs))
                    cases.append((256, 4096, h0, 1000, 1256, i0, nq, page, 64, cs))
    for case, (head, tiles, wholes) in zip(cases, layout(cases)):
        _check(case, head, tiles, wholes)

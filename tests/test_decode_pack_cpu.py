"""The tensor-core decode kernel's tile layout, compiled from the library's
header as host code and run on the CPU.  For many ring states (head offset,
fill level, wrap, paged and unpaged, plain decode and decode step): the pieces
of a pair's tiles cover exactly the rows the query at t sees (blog "Formal
verification of a sliding-window KV cache in Lean4" section 2.1 reference
model; "Prefix Sliding" digest section 03 rule), each once; a ring piece's
slots hold its positions and stay inside the ring and one page; a row sits
at its slot's offset within its 8-row atom, the atoms a piece's copy writes
stay inside the tile and hold no other piece's rows, and the copy starts in
the piece's own page; in a decode step the token at t is the last piece, read
from the caller's row (in a plain decode, the same piece read from t's ring
slot, so both lay out their tiles identically); with pages a multiple of 8
rows a paged ring has the unpaged ring's layout."""
import os
import random
import shutil
import subprocess
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "native", "decode_pack_harness.cu")
CSRC = os.path.join(ROOT, "prefix_sliding_window_ring_b200", "csrc")
RUN_PREFIX, RUN_RING, RUN_NEW = 0, 1, 2


def pad8(x):
    return (x + 7) // 8 * 8


@pytest.fixture(scope="module")
def layout():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    d = tempfile.mkdtemp(prefix="dpack")
    exe = os.path.join(d, "decode_pack_harness")
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
                ps_ = [tuple(int(v) for v in p.split(",")) for p in t.split() if not p.startswith("W")]
                ws = [tuple(int(v) for v in p[1:].split(",")) for p in t.split() if p.startswith("W")]
                tiles.append(ps_)
                wholes.append(ws[0] if ws else None)
            assert len(tiles) == head[0]
            res.append((head, tiles, wholes))
        return res
    yield run
    shutil.rmtree(d, ignore_errors=True)


def _check(case, head, tiles, wholes=None):
    P, W, h0, count, next_pos, t, page, step, TR, csize = case
    ntiles, rows, padded, ring_ok = head
    assert ring_ok == 1
    base = next_pos - count
    need = [int(p) for p in oracle.visible_positions(P, W, t)]
    got = []
    aligned = page == 0 or page % 8 == 0
    newest = tiles[-1][-1]
    for j, pieces in enumerate(tiles):
        assert pieces, ("empty tile", case, j)
        end = 0
        for src, row, sr, n in pieces:
            lead = sr % 8                  # the copy starts at the atom below sr
            assert n >= 1 and sr - lead >= end, ("atoms shared", case, j, sr, n)
            assert sr + n <= TR and pad8(sr + n) <= TR, (case, j, sr, n)
            end = pad8(sr + n)
            if j == len(tiles) - 1 and (src, row, sr, n) == newest:
                assert lead == 0, case     # the newest row starts an atom of its own
            elif src == RUN_PREFIX or (src == RUN_RING and aligned):
                assert row % 8 == lead, ("row not at its slot's offset", case)
            else:
                assert lead == 0, case
            if src == RUN_RING and page:
                assert row % page - lead >= 0, ("copy starts in another page", case)
            if src == RUN_PREFIX:
                assert 0 <= row and row + n <= P, case
                got.extend(range(row, row + n))
            elif src == RUN_RING:
                assert 0 <= row and row + n <= W, ("ring piece wraps", case)
                if page:
                    assert row // page == (row + n - 1) // page, ("crosses a page", case)
                pos0 = base + (row - h0) % W
                assert base <= pos0 and pos0 + n <= next_pos, case
                got.extend(range(pos0, pos0 + n))
            else:
                assert src == RUN_NEW and step and n == 1, case
                got.append(t)
    # the newest row (position t) is a piece of its own, the last one: the
    # appended token in a step, its ring slot in a plain decode
    src, row, sr, n = tiles[-1][-1]
    assert n == 1 and sr % 8 == 0 and tiles[-1][-1] not in tiles[-1][:-1], case
    if step:
        assert src == RUN_NEW, ("the token is the last row", case)
    else:
        assert src == RUN_RING and (row - h0) % W == t - base, ("t's slot", case)
    assert len(got) == len(set(got)), ("a row read twice", case)
    assert sorted(got) == need, ("coverage", case)
    assert rows == len(need) and padded % 8 == 0
    if not csize:
        assert ntiles == (padded + TR - 1) // TR
    for pieces, w in zip(tiles, wholes or [None] * len(tiles)):
        if w is not None:  # a whole tile is exactly one piece of TR rows from tile row 0
            assert pieces == [(w[0], w[1], 0, TR)] and w[1] % 8 == 0, (case, pieces, w)


def _cases(rng, n):
    out = []
    for _ in range(n):
        W = rng.choice([1, 2, 7, 8, 16, 63, 64, 65, 128, 130, 300, 512, 1024, 4096])
        P = rng.choice([0, 1, 7, 8, 9, 37, 64, 128, 300])
        pages = [0] + [p for p in (1, 2, 4, 8, 16, 24, 64, 128, 256) if W % p == 0 and p <= W]
        page = rng.choice(pages)
        step = rng.randrange(2)
        t = P + rng.randrange(0, 3 * W + 200)    # the query's position, t >= P
        next_pos = t + 1                          # the token at t is in the history
        count = min(W, next_pos - P)
        h0 = rng.randrange(W)
        TR = rng.choice([64, 128])
        csize = rng.choice([0, 0, 2, 4, 8])
        out.append((P, W, h0, count, next_pos, t, page, step, TR, csize))
    return out


def test_decode_tiles_cover_exactly_the_visible_rows(layout):
    rng = random.Random(17)
    cases = _cases(rng, 4000)
    for case, (head, tiles, wholes) in zip(cases, layout(cases)):
        _check(case, head, tiles, wholes)


def test_paged_layout_equals_unpaged(layout):
    """Pages of a multiple of 8 rows leave the tile layout unchanged (so the
    kernel's arithmetic, and its results, are bit-identical)."""
    rng = random.Random(23)
    cases, paged = [], []
    for _ in range(1500):
        W = rng.choice([8, 64, 128, 512, 4096])
        P = rng.choice([0, 5, 128])
        page = rng.choice([p for p in (8, 16, 64, 128, 256) if W % p == 0])
        step = rng.randrange(2)
        t = P + rng.randrange(0, 3 * W)
        h0 = rng.randrange(W)
        base = (P, W, h0, min(W, t + 1 - P), t + 1, t, 0, step, 64, rng.choice([0, 4]))
        cases.append(base)
        paged.append(base[:6] + (page,) + base[7:])
    for (ha, ta, _), (hb, tb, _) in zip(layout(cases), layout(paged)):
        assert ha == hb

        def rows(tiles):
            return [sorted((sr + k, src, row + k) for src, row, sr, n in t for k in range(n))
                    for t in tiles]
        # the same rows at the same tile rows (a page edge may split a piece in two)
        assert rows(ta) == rows(tb)


def test_decode_tiles_edge_states(layout):
    """Window not yet full, just full, first eviction, the wrap at every
    offset of a small ring, one-row windows, the decode workload's shape."""
    cases = []
    for W in (1, 8, 9, 16, 64):
        for P in (0, 3, 8):
            for step in (0, 1):
                for n in range(1, 2 * W + 3):
                    t = P + n - 1
                    for h0 in range(W):
                        cases.append((P, W, h0, min(W, n), t + 1, t, 0, step, 64, 0))
    for step in (0, 1):
        for h0 in (0, 1, 613, 4095):
            for cs in (0, 4):
                cases.append((128, 4096, h0, 4096, 65537, 65536, 0, step, 64, cs))
                cases.append((128, 4096, h0, 4096, 65537, 65536, 16, step, 64, cs))
                cases.append((128, 4096, h0, 1921, 2049, 2048, 0, step, 64, cs))
    for case, (head, tiles, wholes) in zip(cases, layout(cases)):
        _check(case, head, tiles, wholes)

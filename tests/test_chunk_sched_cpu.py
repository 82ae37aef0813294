"""The tensor-core chunk kernel's key-tile schedule, compiled from the
library's header as host code and run on the CPU.  For chunk and prompt query
tiles over many cache states (ring head, fill level, wrap, paged and unpaged):
the tiles cover every key any query of the tile sees, read no key that none of
them sees, read each key once, and address it correctly -- a ring tile's slots
hold its positions and never wrap; with pages of 128 rows or more a ring tile
stays inside one page, with smaller pages (8 to 64 rows) it starts on a page
edge, and its rows before the range hold positions below the schedule's
lowest ring key (rlo), which the kernel masks like the window's edge; prefix
and block rows are the positions themselves."""
import os
import random
import shutil
import subprocess

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "native", "chunk_sched_harness.cu")
CSRC = os.path.join(ROOT, "prefix_sliding_window_ring_b200", "csrc")
BN = 128


@pytest.fixture(scope="module")
def sched():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    import tempfile
    d = tempfile.mkdtemp(prefix="sched")
    exe = os.path.join(d, "chunk_sched_harness")
    subprocess.check_call([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", CSRC, HARNESS, "-o", exe])

    def run(cases):
        text = "\n".join(" ".join(str(v) for v in c) for c in cases) + "\n"
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        res = []
        for line in out.strip().split("\n"):
            f = line.split()
            tiles = [tuple(int(x) for x in t.split(",")) for t in f[2:]]
            assert len(tiles) == int(f[0])
            res.append((int(f[1]), tiles))
        return res
    yield run
    shutil.rmtree(d, ignore_errors=True)


def _chunk_cases(rng, n_cases):
    out = []
    for _ in range(n_cases):
        W = rng.choice([1, 7, 128, 130, 300, 512, 640, 1024])
        P = rng.choice([0, 1, 37, 128, 300])
        # the tensor-core kernel takes paged caches whose pages are 128-row
        # multiples or divide 128 and are multiples of 8 (other pages go to the
        # CUDA-core kernel, which maps rows one by one)
        page = rng.choice([0] + [p for p in (8, 16, 32, 64, 128, 256, 512, 1024)
                                 if W % p == 0 and p <= W])
        next_pos = P + rng.randrange(0, 3 * W + 300)
        count = min(W, next_pos - P)
        head = rng.randrange(W)
        n_blk = rng.randrange(1, 700)
        PT = rng.choice([16, 32, 64, 128])
        i0 = rng.randrange(0, n_blk, PT) if n_blk > PT else 0
        plo, phi = next_pos + i0, next_pos + min(i0 + PT, n_blk) - 1
        out.append((P, W, head, count, next_pos, next_pos, plo, phi, 0, page))
    return out


def _check(case, sched_out):
    P, W, head, count, next_pos, t0, plo, phi, prompt, page = case
    rlo, tiles = sched_out
    base = next_pos - count
    need = set()
    for t in range(plo, phi + 1):
        if prompt:
            need.update(range(0, t + 1))
        else:
            need.update(int(p) for p in oracle.visible_positions(P, W, t))
    got = []
    for src, row, pos0, valid in tiles:
        # rows the kernel masks by position below rlo (ring and block tiles)
        lead = 0 if src == 2 else max(0, rlo - pos0)
        assert 0 <= lead < valid <= BN, (case, src, row, pos0, valid, lead)
        assert lead == 0 or (src == 0 and 0 < page < BN and lead < page), case
        if src == 2:  # prefix rows are the positions
            assert row == pos0 and 0 <= row and row + valid <= P, case
        elif src == 1:  # block rows: position t0 + row, inside the block
            assert pos0 == t0 + row and row >= 0 and t0 + row + valid - 1 <= phi, case
        else:  # ring slots: contiguous, no wrap, holding their positions
            assert 0 <= row and row + valid <= W, case
            if page >= BN:  # inside one page
                assert row // page == (row + valid - 1) // page, case
            elif page:  # whole pages from a page edge
                assert row % page == 0, case
            assert base <= pos0 + lead and pos0 + valid <= next_pos, case
            assert (head + pos0 + lead - base) % W == row + lead, case
        got.extend(range(pos0 + lead, pos0 + valid))
    assert len(got) == len(set(got)), ("a key read twice", case)
    assert set(got) == need, ("coverage", case, sorted(need - set(got))[:5],
                              sorted(set(got) - need)[:5])


def test_chunk_tiles_cover_exactly_the_visible_keys(sched):
    rng = random.Random(5)
    cases = _chunk_cases(rng, 3000)
    for case, out in zip(cases, sched(cases)):
        _check(case, out)


def test_prompt_tiles_cover_exactly_the_causal_prefix(sched):
    rng = random.Random(6)
    cases = []
    for _ in range(800):
        P = rng.choice([1, 2, 127, 128, 129, 300, 1000])
        PT = rng.choice([16, 64, 128])
        plo = rng.randrange(0, P)
        phi = min(P - 1, plo + PT - 1)
        cases.append((P, 64, 0, 0, P, 0, plo, phi, 1, 0))
    for case, out in zip(cases, sched(cases)):
        _check(case, out)
        assert all(src == 2 for src, *_ in out[1])

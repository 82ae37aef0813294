"""The tensor-core chunk kernel's key-tile schedule, compiled from the
library's header as host code and run on the CPU.  For chunk and prompt query
tiles over many cache states (ring head, fill level, wrap, paged and unpaged):
the tiles cover every key any query of the tile sees, read no key that none of
them sees, read each key once, and address it correctly -- a ring tile's slots
hold its positions, never wrap and stay inside one page; prefix and block rows
are the positions themselves.  Pages are 128-row multiples, the only paged
caches this kernel is given."""
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
            tiles = [tuple(int(x) for x in t.split(",")) for t in f[1:]]
            assert len(tiles) == int(f[0])
            res.append(tiles)
        return res
    yield run
    shutil.rmtree(d, ignore_errors=True)


def _chunk_cases(rng, n_cases):
    out = []
    for _ in range(n_cases):
        W = rng.choice([1, 7, 128, 130, 300, 512, 640, 1024])
        P = rng.choice([0, 1, 37, 128, 300])
        # the tensor-core kernel takes paged caches whose pages are 128-row multiples
        # (smaller pages go to the CUDA-core kernel, which maps rows one by one)
        page = rng.choice([0] + [p for p in (128, 256, 512, 1024) if W % p == 0 and p <= W])
        next_pos = P + rng.randrange(0, 3 * W + 300)
        count = min(W, next_pos - P)
        head = rng.randrange(W)
        n_blk = rng.randrange(1, 700)
        PT = rng.choice([16, 32, 64, 128])
        i0 = rng.randrange(0, n_blk, PT) if n_blk > PT else 0
        plo, phi = next_pos + i0, next_pos + min(i0 + PT, n_blk) - 1
        out.append((P, W, head, count, next_pos, next_pos, plo, phi, 0, page))
    return out


def _check(case, tiles):
    P, W, head, count, next_pos, t0, plo, phi, prompt, page = case
    base = next_pos - count
    need = set()
    for t in range(plo, phi + 1):
        if prompt:
            need.update(range(0, t + 1))
        else:
            need.update(int(p) for p in oracle.visible_positions(P, W, t))
    got = []
    for src, row, pos0, valid in tiles:
        assert 1 <= valid <= BN, (case, src, row, pos0, valid)
        if src == 2:  # prefix rows are the positions
            assert row == pos0 and 0 <= row and row + valid <= P, case
        elif src == 1:  # block rows: position t0 + row, inside the block
            assert pos0 == t0 + row and row >= 0 and t0 + row + valid - 1 <= phi, case
        else:  # ring slots: contiguous, no wrap, one page, holding their positions
            assert 0 <= row and row + valid <= W, case
            if page:
                assert row // page == (row + valid - 1) // page, case
            assert base <= pos0 and pos0 + valid <= next_pos, case
            assert (head + pos0 - base) % W == row, case
        got.extend(range(pos0, pos0 + valid))
    assert len(got) == len(set(got)), ("a key read twice", case)
    assert set(got) == need, ("coverage", case, sorted(need - set(got))[:5],
                              sorted(set(got) - need)[:5])


def test_chunk_tiles_cover_exactly_the_visible_keys(sched):
    rng = random.Random(5)
    cases = _chunk_cases(rng, 3000)
    for case, tiles in zip(cases, sched(cases)):
        _check(case, tiles)


def test_prompt_tiles_cover_exactly_the_causal_prefix(sched):
    rng = random.Random(6)
    cases = []
    for _ in range(800):
        P = rng.choice([1, 2, 127, 128, 129, 300, 1000])
        PT = rng.choice([16, 64, 128])
        plo = rng.randrange(0, P)
        phi = min(P - 1, plo + PT - 1)
        cases.append((P, 64, 0, 0, P, 0, plo, phi, 1, 0))
    for case, tiles in zip(cases, sched(cases)):
        _check(case, tiles)
        assert all(src == 2 for src, *_ in tiles)

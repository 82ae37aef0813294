"""The paged ring's page planning (the library's host code, compiled from its
header with the host C++ compiler and run on the CPU): a write maps exactly the
ring pages its slots touch that had no page, takes them from the end of the
free list, records the page-table entries to set, leaves every other page
alone, and reports an exhausted pool."""
import os
import random
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "native", "page_plan_harness.cpp")
CSRC = os.path.join(ROOT, "prefix_sliding_window_ring_b200", "csrc")


@pytest.fixture(scope="module")
def plan():
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tempfile.mkdtemp(prefix="plan")
    exe = os.path.join(d, "page_plan_harness")
    subprocess.check_call([cxx, "-std=c++17", "-O1", "-I", CSRC, HARNESS, "-o", exe])

    def run(cases):
        text = "\n".join(f"{W} {pr} {seq} {s0} {n} | {' '.join(map(str, pages))} | "
                         f"{' '.join(map(str, avail))}" for W, pr, seq, s0, n, pages, avail in cases)
        out = subprocess.run([exe], input=text + "\n", capture_output=True, text=True,
                             check=True).stdout.strip().split("\n")
        res = []
        for line in out:
            ok, pages, avail, sets = line.split("|")
            res.append((ok.strip() == "1", [int(x) for x in pages.split()],
                        [int(x) for x in avail.split()],
                        [tuple(int(v) for v in x.split(":")) for x in sets.split()]))
        return res
    yield run
    shutil.rmtree(d, ignore_errors=True)


def test_a_write_maps_exactly_the_pages_it_touches(plan):
    rng = random.Random(11)
    cases = []
    for _ in range(3000):
        pr = rng.choice([1, 2, 3, 4, 8, 16, 128])
        npg = rng.randrange(1, 12)
        W = pr * npg
        seq = rng.randrange(0, 5)
        pages = [rng.choice([-1, -1, rng.randrange(100, 200)]) for _ in range(npg)]
        avail = rng.sample(range(0, 99), rng.randrange(0, 2 * npg + 1))
        slot0 = rng.randrange(0, 3 * W)
        n = rng.randrange(0, 3 * W)
        cases.append((W, pr, seq, slot0, n, pages, avail))
    for (W, pr, seq, slot0, n, pages, avail), (ok, pages2, avail2, sets) in zip(cases,
                                                                              plan(cases)):
        # planning takes min(n, W) slots from slot0 (callers pass the first slot that
        # survives a write longer than the ring)
        touched = {((slot0 % W + i) % W) // pr for i in range(min(n, W))}
        need = sorted(p for p in touched if pages[p] < 0)
        if len(need) > len(avail):
            assert not ok
            continue
        assert ok
        given = list(reversed(avail))[:len(need)]  # popped from the end, in page order
        assert [p for p, _ in sets] == [seq * (W // pr) + p for p in _order(W, pr, slot0, n, need)]
        assert sorted(v for _, v in sets) == sorted(given)
        assert avail2 == avail[:len(avail) - len(need)]
        for p in range(W // pr):
            if p in need:
                assert pages2[p] == dict((q - seq * (W // pr), v) for q, v in sets)[p]
            else:
                assert pages2[p] == pages[p]


def _order(W, pr, slot0, n, need):
    """The pages needing a page, in the order the write reaches them."""
    seen, out = set(), []
    for i in range(min(n, W)):
        p = ((slot0 % W + i) % W) // pr
        if p in need and p not in seen:
            seen.add(p)
            out.append(p)
    return out


def test_no_write_and_a_full_ring_write(plan):
    # n = 0 touches nothing; a write of >= W slots touches every page once
    (ok, pages, avail, sets), = plan([(8, 2, 1, 3, 0, [-1, -1, -1, -1], [7])])
    assert ok and pages == [-1, -1, -1, -1] and avail == [7] and sets == []
    (ok, pages, avail, sets), = plan([(8, 2, 1, 5, 20, [-1, 42, -1, -1], [1, 2, 3, 4])])
    assert ok and sorted(pages) == [2, 3, 4, 42] and avail == [1]
    assert sorted(i for i, _ in sets) == [4, 6, 7]  # seq 1 * 4 pages + pages 0, 2, 3

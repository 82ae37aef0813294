"""The library's visible-range derivation (the row ranges every kernel
streams) and its cache addressing, compiled from the library's own header as
host code and run on the CPU: for every small (P, W, ring head, length) and
every query position from the decode query to far past the window, the ranges
visit exactly the oracle's visible positions, in order, each once; every prefix
row, ring row and position entry of an unpaged or paged cache has its own
address."""
import os
import shutil
import subprocess

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "native", "segments_harness.cu")
CSRC = os.path.join(ROOT, "prefix_sliding_window_ring_b200", "csrc")


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    exe = str(tmp_path_factory.mktemp("seg") / "segments_harness")
    subprocess.check_call([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", CSRC, HARNESS, "-o", exe])

    def run(lines):
        out = subprocess.run([exe], input="\n".join(lines) + "\n", capture_output=True, text=True,
                             check=True).stdout
        return out.strip().split("\n")
    return run


def _cases():
    for W in (1, 2, 3, 5, 8):
        for P in (0, 1, 3):
            for head in range(W):
                for next_pos in range(P, P + 3 * W + 3):
                    count = min(W, next_pos - P)
                    # a decode query is next_pos - 1; chunk queries reach past next_pos
                    for t in range(max(next_pos - 1, 0), next_pos + 2 * W + 2):
                        if t < P:
                            continue  # prompt queries use the prompt schedule, not these ranges
                        yield P, W, head, count, next_pos, t


def test_ranges_visit_exactly_the_visible_positions(harness):
    cases = list(_cases())
    out = harness([f"seg {P} {W} {h} {c} {n} {t}" for P, W, h, c, n, t in cases])
    assert len(out) == len(cases)
    for (P, W, h, c, n, t), line in zip(cases, out):
        head_part, _, pos_part = line.partition(":")
        fields = head_part.split()
        ring_ok, total = int(fields[1]), int(fields[3])
        got = [int(x) for x in pos_part.split()]
        exp = [int(x) for x in oracle.visible_positions(P, W, t)]
        assert ring_ok == 1, (P, W, h, c, n, t)
        assert total == len(got) == len(exp), (P, W, h, c, n, t)
        assert got == exp, (P, W, h, c, n, t, got, exp)


def test_a_ring_missing_part_of_the_window_is_flagged(harness):
    # the ring holds 2 of the 4 window rows the query needs: the ranges stop at
    # what is held and the derivation says so
    out = harness(["seg 2 4 0 2 10 9"])
    fields = out[0].split(":")[0].split()
    assert int(fields[1]) == 0


@pytest.mark.parametrize("S,Hkv,P_max,W,page_rows,nphys", [
    (3, 2, 5, 8, 0, 0), (1, 1, 0, 1, 0, 0), (4, 3, 7, 12, 4, 9), (2, 2, 0, 16, 16, 3),
    (5, 1, 3, 6, 1, 13),
])
def test_every_row_and_position_entry_has_its_own_address(harness, S, Hkv, P_max, W, page_rows,
                                                           nphys):
    out = harness([f"addr {S} {Hkv} {P_max} {W} {page_rows} {nphys}"])
    f = out[0].split()
    rows, bad, shared, unused = int(f[1]), int(f[3]), int(f[5]), int(f[7])
    assert rows > 0 and bad == 0 and shared == 0 and unused == 0, out[0]

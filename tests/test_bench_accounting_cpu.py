"""The work bench.py divides by its timings, pinned to the visible sets of the
oracle (CPU only): decode bytes per step, chunk- and prompt-prefill flops per
step count exactly the keys each query sees."""
import os
import sys

import numpy as np

import oracle

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _visible(P, W, t):
    return len(oracle.visible_positions(P, W, t))


def test_decode_bytes_are_the_visible_rows_of_the_step():
    # every sequence of a step sits at t >= T_START, window full
    n = _visible(bench.P, bench.W, bench.T_START)
    assert n == bench.P + bench.W == 4224
    per_seq = bench.HKV * n * bench.D * 2 * 2  # K and V rows, 2 bytes each
    assert bench.kv_bytes_per_seq() == per_seq
    assert bench.kv_bytes_per_step() == bench.B * per_seq == 138412032


def test_prefill_flops_count_the_visible_pairs():
    for Wp, gflop in ((4096, 292.1), (16384, 1116.7)):
        # the visible count is the same for every query of a block far past the window
        ts = [bench.PF_T0, bench.PF_T0 + bench.PF_N // 2, bench.PF_T0 + bench.PF_N - 1]
        counts = {_visible(bench.PF_P, Wp, t) for t in ts}
        assert counts == {bench.PF_P + Wp}
        pairs = bench.PF_SEQS * bench.PF_N * (bench.PF_P + Wp)
        assert bench.prefill_flops(Wp) == 4.0 * bench.D * bench.HQ * pairs
        assert round(bench.prefill_flops(Wp) / 1e9, 1) == gflop


def test_prompt_flops_count_the_causal_pairs():
    P = bench.PR_P
    # prompt query t sees [0, t]; the oracle's rule for t < P with any window
    ts = np.arange(P)
    pairs = int(sum(len([p for p in range(t + 1) if oracle.is_visible(P, 64, int(t), p)])
                    for t in ts[:64]))  # spot check the first rows by brute force
    assert pairs == sum(t + 1 for t in range(64))
    assert bench.prompt_flops() == 4.0 * bench.D * bench.HQ * bench.PF_SEQS * P * (P + 1) / 2

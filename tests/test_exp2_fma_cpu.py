"""The FMA-pipe exponential of the tensor-core chunk kernel: 2^y as
2^floor(y) * p(y - floor(y)) with a cubic p fitted to 2^f on [0, 1) (Cody and
Waite's reduction).  The coefficients are read from the kernel source and the
method is replayed in float32 with numpy; the kernel itself is compared with
the float64 oracle by the GPU chunk tests.  Pinned: the relative error against
exact 2^y over the range the softmax feeds it (scaled scores minus the
running maximum, at most 2^8 above it), exact zeros at and below -127 (the
masked -inf included), and exact powers of two at integers."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "prefix_sliding_window_ring_b200", "csrc", "chunk_tc.cu")


def _coeffs():
    text = open(SRC).read()
    m = re.search(r"kExpC1 = ([0-9.e+-]+)f, kExpC2 = ([0-9.e+-]+)f, kExpC3 = ([0-9.e+-]+)f", text)
    assert m, "coefficients not found in the kernel source"
    return [np.float32(float(g)) for g in m.groups()]


def _exp2_fma(y):
    c1, c2, c3 = _coeffs()
    y = np.maximum(np.asarray(y, np.float32), np.float32(-127.0))
    fl = np.floor(y).astype(np.float32)
    f = (y - fl).astype(np.float32)
    q = ((c3 * f + c2) * f + c1) * f + np.float32(1.0)
    bits = q.view(np.uint32).astype(np.int64) + (fl.astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    y = np.linspace(-126.0, 8.0, 400001, dtype=np.float32)
    got = _exp2_fma(y).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < 2.7e-4
    # well below the relative rounding of the bf16 P it feeds (2^-9)
    assert 2.7e-4 < 2.0 ** -9


def test_masked_and_underflowing_inputs_give_exact_zero():
    y = np.array([-np.inf, -1e30, -1000.0, -127.5, -127.0], np.float32)
    out = _exp2_fma(y)
    assert np.all(out == 0.0) and not np.any(np.signbit(out))


def test_integers_give_exact_powers_of_two():
    k = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(_exp2_fma(k), np.exp2(k.astype(np.float64)).astype(np.float32))

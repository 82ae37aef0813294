"""Pins for the oracle's visibility rule and float64 attention (CPU only).

What pins them (none of it comes from the oracle itself):
- visible sets and counts hand-derived from the digest's section 03 rule,
  including its worked example (P=100, W=4096: 4196 positions);
- closed forms: |A(t)| = P + min(W, t-P+1); q = 0 gives the plain mean of the
  visible values; W=1, P=0 gives v_t; two keys give a logistic weight;
- special cases that reduce to a library routine: with the window covering
  the whole history the rule is plain causal attention, checked against
  torch's scaled_dot_product_attention in float64;
- the blog's section 4.2 corollary: attention over the full history with the
  window mask equals unmasked softmax attention over the truncated list
  (prefix ++ lastWindow), the list coming from the separately pinned list model
  and the softmax from torch;
- invariants: masked rows carry exactly zero weight, the row order of the
  history list does not matter;
- planted mistakes: mutated copies of attention.c, built on the CPU, must each
  fail at least one of these pins.
"""
import math
import os

import subprocess
import tempfile


import numpy as np
import pytest
import torch

import oracle
from oracle import listmodel as lm
from tests.golden import fixtures


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ pins ---

def pin_visible_golden():
    for P, W, t, exp in fixtures.visible_set_cases():
        assert list(oracle.visible_positions(P, W, t)) == exp, (P, W, t)
    for P, W, t, exp in fixtures.visible_count_cases():
        assert len(oracle.visible_positions(P, W, t)) == exp, (P, W, t)


def pin_visible_closed_form():
    for P in (0, 1, 3, 7):
        for W in (1, 2, 3, 5, 9):
            for t in range(0, P + 3 * W + 4):
                got = oracle.visible_positions(P, W, t)
                if t >= P:
                    assert len(got) == P + min(W, t - P + 1)
                    lo = max(P, t - W + 1)
                    assert list(got) == list(range(P)) + list(range(lo, t + 1))
                else:
                    assert list(got) == list(range(t + 1))
                if P == 0:                       # plain sliding window
                    assert list(got) == list(range(max(0, t - W + 1), t + 1))
                if W >= t - P + 1:               # window covers everything: causal
                    assert list(got) == list(range(t + 1))


def pin_zero_query_is_mean():
    r = _rng(1)
    d, T, P, W = 16, 40, 3, 7
    K, V = r.standard_normal((T, d)), r.standard_normal((T, d))
    for t in (0, 2, 5, 9, 20, 39):
        out = oracle.attend(P, W, t, 0.25, np.zeros((2, d)), np.arange(T), K, V)
        vis = oracle.visible_positions(P, W, t)
        mean = V[vis].sum(0) / len(vis)
        np.testing.assert_allclose(out, np.stack([mean, mean]), rtol=0, atol=1e-14)


def pin_window_one_is_last_value():
    r = _rng(2)
    d, T = 8, 12
    K, V = r.standard_normal((T, d)), r.standard_normal((T, d))
    for t in range(T):
        out = oracle.attend(0, 1, t, 0.3, r.standard_normal((3, d)), np.arange(T), K, V)
        assert np.array_equal(out, np.stack([V[t]] * 3))


def pin_two_keys_logistic():
    for a, b in [(0.0, 0.0), (1.5, -0.5), (-3.0, 2.0), (10.0, 9.0)]:
        q = np.array([[1.0, 0.0, 0.0, 0.0]])
        K = np.array([[a, 0, 0, 0], [b, 0, 0, 0]], dtype=np.float64)
        V = np.array([[0, 1, 0, 0], [0, 0, 1, 0]], dtype=np.float64)
        out = oracle.attend(0, 2, 1, 1.0, q, np.array([0, 1]), K, V)[0]
        w0 = 1.0 / (1.0 + math.exp(b - a))
        np.testing.assert_allclose(out, [0.0, w0, 1.0 - w0, 0.0], rtol=0, atol=1e-15)
        only_last = oracle.attend(0, 1, 1, 1.0, q, np.array([0, 1]), K, V)[0]
        assert np.array_equal(only_last, V[1])


def pin_causal_equals_sdpa():
    r = _rng(3)
    T, d, G = 33, 16, 2
    scale = 1.0 / math.sqrt(d)
    Q = r.standard_normal((G, T, d))
    K, V = r.standard_normal((T, d)), r.standard_normal((T, d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None, None].expand(1, G, T, d),
        torch.from_numpy(V)[None, None].expand(1, G, T, d), is_causal=True, scale=scale)[0]
    for P in (0, 3):
        for t in range(T):
            out = oracle.attend(P, T + 5, t, scale, Q[:, t], np.arange(T), K, V)
            np.testing.assert_allclose(out, ref[:, t].numpy(), rtol=0, atol=1e-12)


def pin_window_corollary():
    """Full history + masks == softmax over prefix ++ lastWindow (blog 4.2)."""
    r = _rng(4)
    d, T = 16, 60
    scale = 0.2
    K, V = r.standard_normal((T, d)), r.standard_normal((T, d))
    for P, W in [(0, 1), (0, 5), (3, 1), (3, 4), (5, 11), (2, 70)]:
        for t in range(T):
            q = r.standard_normal((2, d))
            out = oracle.attend(P, W, t, scale, q, np.arange(T), K, V)
            if t < P:
                keep = list(range(t + 1))
            else:
                hist = [(p, None) for p in range(P, t + 1)]
                keep = list(range(P)) + [c[0] for c in lm.last_window(W, hist)]
            Kt, Vt = torch.from_numpy(K[keep]), torch.from_numpy(V[keep])
            w = torch.softmax(scale * (torch.from_numpy(q) @ Kt.T), dim=-1)
            np.testing.assert_allclose(out, (w @ Vt).numpy(), rtol=0, atol=1e-12)


def pin_masked_rows_have_zero_weight():
    r = _rng(5)
    P, W, T, d = 4, 6, 30, 32
    K = r.standard_normal((T, d))
    V = np.eye(d)[:T]                     # v_p = e_p exposes the weight of p
    for t in range(T):
        out = oracle.attend(P, W, t, 0.5, r.standard_normal((1, d)), np.arange(T), K, V)[0]
        vis = set(oracle.visible_positions(P, W, t).tolist())
        for p in range(T):
            if p in vis:
                assert out[p] > 0
            else:
                assert out[p] == 0.0
        assert abs(out.sum() - 1.0) < 1e-14


def pin_row_order_and_masked_values_irrelevant():
    r = _rng(6)
    P, W, T, d = 3, 5, 25, 8
    K, V = r.standard_normal((T, d)), r.standard_normal((T, d))
    q = r.standard_normal((2, d))
    t = 17
    base = oracle.attend(P, W, t, 0.4, q, np.arange(T), K, V)
    perm = r.permutation(T)
    np.testing.assert_allclose(oracle.attend(P, W, t, 0.4, q, perm, K[perm], V[perm]), base,
                               rtol=0, atol=1e-14)
    vis = set(oracle.visible_positions(P, W, t).tolist())
    K2, V2 = K.copy(), V.copy()
    for p in range(T):
        if p not in vis:
            K2[p] = 1e6
            V2[p] = -1e6
    assert np.array_equal(oracle.attend(P, W, t, 0.4, q, np.arange(T), K2, V2), base)


PINS = [pin_visible_golden, pin_visible_closed_form, pin_zero_query_is_mean,
        pin_window_one_is_last_value, pin_two_keys_logistic, pin_causal_equals_sdpa,
        pin_window_corollary, pin_masked_rows_have_zero_weight,
        pin_row_order_and_masked_values_irrelevant]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_batch_matches_single():
    r = _rng(7)
    d, T = 16, 50
    K, V = r.standard_normal((T, d)), r.standard_normal((T, d))
    b = oracle.Batch()
    outs, singles = [], []
    for t in range(0, T, 3):
        q = r.standard_normal((2, d))
        outs.append(b.add(2, 9, t, 0.3, q, np.arange(T), K, V))
        singles.append(oracle.attend(2, 9, t, 0.3, q, np.arange(T), K, V))
    b.run(4)
    for a, s in zip(outs, singles):
        assert np.array_equal(a, s)


# --------------------------------------------------------- planted mistakes ---

MUTANTS = {
    "window one row too wide": ("int64_t lo = t - W + 1;", "int64_t lo = t - W;"),
    "query does not see itself": ("if (p < 0 || p > t) return 0;",
                                  "if (p < 0 || p >= t) return 0;"),
    "prefix one row too long": ("if (p < P) return 1;", "if (p <= P) return 1;"),
    "scale dropped": ("z[r] = scale * dot;", "z[r] = dot;"),
    "keys used as values": ("oh[c] += w * hv[(size_t)r * d + c];",
                            "oh[c] += w * hk[(size_t)r * d + c];"),
    "no normalisation": ("for (int c = 0; c < d; ++c) oh[c] /= den;", ""),
    "head 0 query for all heads": ("const double* qh = q + (size_t)h * d;",
                                   "const double* qh = q;"),
    "uniform denominator": ("den += w;", "den += 1.0;"),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attention.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, old
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "m.c")
        so = os.path.join(td, "m.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", so, c, "-lm", "-lpthread"])
        monkeypatch.setattr(oracle, "_lib", None)
        monkeypatch.setattr(oracle, "_SO", so)
        monkeypatch.setattr(oracle, "build", lambda force=False: so)
        failed = []
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
        assert failed, f"mutant '{name}' passed every pin"
    oracle._lib = None

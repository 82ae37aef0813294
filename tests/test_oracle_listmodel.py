"""Pins for the oracle's list and ring models (CPU only).

What pins them (none of it comes from the oracle itself):
- golden cases hand-derived from the blog's definitions, including the page's
  own executable example ``step 4 [] kv1 = [kv1]`` (tests/golden/*.txt);
- the key equation lastWindow(xs++[kv]) = step(lastWindow xs, kv) and the
  run_correct theorem (blog sections 2.4, 4.1, 4.2), checked by brute force
  over every history length up to 3w+3 for w = 1..9;
- the drop/append lemma of section 4.1, by brute force;
- closed forms: length min(w, len), base position P + max(0, len - W);
- the digest's generation loop (section 03) against the visibility rule.
"""
import itertools

import pytest

from oracle import listmodel as lm
from oracle import visible_positions
from tests.golden import fixtures


def cells(positions):
    return [(p, f"kv{p}") for p in positions]


def poss(c):
    return [cell[0] for cell in c]


@pytest.mark.parametrize("case", list(fixtures.last_window_cases()))
def test_last_window_golden(case):
    w, hist, exp = case
    assert poss(lm.last_window(w, cells(hist))) == exp


@pytest.mark.parametrize("case", list(fixtures.step_cases()))
def test_step_golden(case):
    w, cache, new, exp = case
    assert poss(lm.step(w, cells(cache), (new, f"kv{new}"))) == exp


@pytest.mark.parametrize("w", range(1, 10))
def test_key_equation_and_run_correct(w):
    """Blog section 2.4 key equation and section 4.2 run_correct, brute force."""
    for n in range(0, 3 * w + 4):
        xs = cells(range(n))
        kv = (n, f"kv{n}")
        assert lm.last_window(w, xs + [kv]) == lm.step(w, lm.last_window(w, xs), kv)
        c = lm.run(w, xs)
        assert lm.valid(w, xs, c)
        assert len(c) <= w and len(c) == min(w, n)          # length obligation
        assert lm.position_invariant(c)                      # position obligation


@pytest.mark.parametrize("w", range(1, 8))
def test_drop_append_lemma(w):
    """Blog section 4.1 drop/append lemma.  As extracted it reads
    (xs ++ [a]).drop(len + 1 - w) = xs.drop(len - w) ++ [a], which is false
    (the right side holds w + 1 cells; w=1, xs=[0] is a counter-example).
    The reading that holds, and that the full-window case of
    step_preserves_valid needs, drops the oldest cell on the right:
    (xs ++ [a]).drop(len + 1 - w) = (xs.drop(len - w) ++ [a]).drop(1)."""
    for n in range(w, 3 * w + 2):
        xs = list(range(n))
        a = -1
        assert (xs + [a])[n + 1 - w:] == (xs[n - w:] + [a])[1:]
    assert ([0] + [-1])[1:] != [0][0:] + [-1]      # the as-extracted form fails


@pytest.mark.parametrize("W", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("P", [0, 1, 3])
def test_window_positions_closed_form(W, P):
    """Position obligation (blog section 2.4): slot i holds base + i, with
    base = t - W + 1 once full; read as base = P + max(0, len - W) so that it
    also holds while the window is filling (section 5.2 warns about the
    truncated subtraction)."""
    for next_pos in range(P, P + 3 * W + 3):
        got = lm.expected_window_positions(P, W, next_pos)
        n = next_pos - P
        base = P + max(0, n - W)
        assert got == list(range(base, base + min(W, n)))


@pytest.mark.parametrize("w", range(1, 10))
def test_ring_simulates_list_model(w):
    """Blog section 3.4 second layer: the ring's push, read through
    ring_to_list, equals the list model's step, for every head offset, at
    the not-full, just-full, first-eviction and wrap-around phases."""
    for h0 in range(w):
        ring = lm.RingBuffer(w, head=h0)
        c = []
        for n in range(1, 3 * w + 3):
            kv = (n - 1, f"kv{n - 1}")
            ring.push(kv)
            c = lm.step(w, c, kv)
            assert ring.to_list() == c
            assert ring.count == min(w, n)
            if n <= w:
                assert ring.head == h0                      # no eviction yet
            else:
                assert ring.head == (h0 + n - w) % w        # one advance per eviction
        # every physical slot holds position p at (h0 + p) mod w
        for slot, cell in enumerate(ring.buf):
            assert slot == (h0 + cell[0]) % w


def test_phase_boundaries_explicit():
    w = 4
    ring = lm.RingBuffer(w, head=2)
    for p in range(3):
        ring.push((p, None))
    assert poss(ring.to_list()) == [0, 1, 2] and ring.head == 2          # not full
    ring.push((3, None))
    assert poss(ring.to_list()) == [0, 1, 2, 3] and ring.head == 2       # just full
    ring.push((4, None))
    assert poss(ring.to_list()) == [1, 2, 3, 4] and ring.head == 3       # first eviction
    for p in range(5, 8):
        ring.push((p, None))
    assert poss(ring.to_list()) == [4, 5, 6, 7] and ring.head == 2       # len == 2w
    for p in range(8, 12):
        ring.push((p, None))
    assert poss(ring.to_list()) == [8, 9, 10, 11] and ring.head == 2     # len == 3w


@pytest.mark.parametrize("P,W", [(0, 1), (0, 3), (2, 3), (3, 1), (4, 6)])
def test_generation_loop_matches_visibility_rule(P, W):
    """Digest section 03: the pseudocode's visible list (prefix ++ window)
    at each step equals the visibility rule A(t) for the query at the last
    token, as enumerated by the oracle's mask.  Two statements on the page,
    checked against each other."""
    prefix = [(p, None) for p in range(P)]
    seen = []

    def next_cell(visible):
        seen.append(visible)
        return (P + len(seen) - 1, None)

    # seed the window with the token at position P (the first generated cell)
    window_states = lm.prefix_sliding_generation(prefix, W, 4 * W + 3, next_cell)
    for k, visible in enumerate(window_states):
        if k == 0:
            continue  # empty window: no query token yet
        t = P + k - 1          # position of the last token in the window
        assert poss(visible) == list(visible_positions(P, W, t))


# ---- planted mistakes: each mutant of the list model must fail a pin above ----

def _step_le(w, c, kv):       # garbled branch read as <=
    c2 = list(c) + [kv]
    if w <= len(c2):
        c2 = c2[1:]
    return c2


def _last_window_off_by_one(w, hs):
    n = len(hs)
    return list(hs[max(0, n - min(w, n) - 1):])


def _ring_to_list_all_slots(w, buf, head, count):
    return [buf[(head + i) % w] for i in range(w)]


def test_mutants_are_caught(monkeypatch):
    caught = []
    for name, mutant in [("step", _step_le), ("last_window", _last_window_off_by_one),
                         ("ring_to_list", _ring_to_list_all_slots)]:
        with monkeypatch.context() as m:
            m.setattr(lm, name, mutant)
            try:
                for case in fixtures.step_cases():
                    test_step_golden(case)
                for case in fixtures.last_window_cases():
                    test_last_window_golden(case)
                test_key_equation_and_run_correct(3)
                test_ring_simulates_list_model(3)
            except AssertionError:
                caught.append(name)
    assert caught == ["step", "last_window", "ring_to_list"]


def test_exhaustive_small_streams():
    """Every w <= 4 and every stream length <= 8 over distinct payloads:
    run == lastWindow (the finite exhaustive check of blog section 5.4)."""
    for w, n in itertools.product(range(1, 5), range(0, 9)):
        xs = cells(range(10, 10 + n))
        assert lm.run(w, xs) == lm.last_window(w, xs)


# ---- negative pins: the obligations must reject caches that break them ----
# (blog section 2.3 Valid: the cache IS the last window, cells and order;
#  section 3.2 PositionInvariant: cell i holds base + i for one base)

def _bad_caches(w, n):
    """Caches that are NOT the last window of history cells(range(n)), n >= w + 2,
    each with the rule it breaks."""
    hs = cells(range(n))
    good = hs[n - w:]
    bad = {
        "reordered": good[::-1] if w > 1 else None,
        "oldest_stale": [hs[n - w - 1]] + good[1:],          # an evicted cell kept
        "one_too_many": hs[n - w - 1:],                       # w + 1 cells
        "newest_missing": good[:-1],                          # truncated at the end
        "oldest_missing": good[1:],                           # truncated at the start
        "shifted_back": hs[n - w - 1:n - 1],                  # the window one step late
        "gap": good[:1] + good[2:] + [hs[0]] if w > 2 else None,
        "payload_changed": good[:-1] + [(n - 1, "other")],
        "empty": [],
    }
    return hs, {k: v for k, v in bad.items() if v is not None}


@pytest.mark.parametrize("w", [1, 2, 3, 5, 8])
def test_valid_rejects_every_other_cache(w):
    n = 3 * w + 2
    hs, bad = _bad_caches(w, n)
    assert lm.valid(w, hs, hs[n - w:])
    for name, c in bad.items():
        assert not lm.valid(w, hs, c), name
    # while the history is shorter than w the whole history is the only valid cache
    short = cells(range(w - 1)) if w > 1 else []
    assert lm.valid(w, short, short)
    if short:
        assert not lm.valid(w, short, short[1:])
        assert not lm.valid(w, short, short + [(99, "x")])


def test_position_invariant_rejects_non_consecutive():
    assert lm.position_invariant(cells([7]))
    assert lm.position_invariant(cells([3, 4, 5, 6]))
    for name, ps in {"gap": [3, 4, 6], "descending": [6, 5, 4], "repeat": [4, 4, 5],
                     "late_gap": [0, 1, 2, 3, 5], "step_two": [0, 2, 4],
                     "first_off": [2, 4, 5, 6], "swapped_middle": [3, 5, 4, 6]}.items():
        assert not lm.position_invariant(cells(ps)), name


# mutants of the two predicates that accept too much; each must fail a pin above

def _valid_any_order(w, hs, c):
    return sorted(c) == sorted(lm.last_window(w, hs))


def _valid_subset(w, hs, c):
    lw = lm.last_window(w, hs)
    return all(cell in lw for cell in c)


def _valid_positions_only(w, hs, c):
    return [x[0] for x in c] == [x[0] for x in lm.last_window(w, hs)]


def _valid_length_only(w, hs, c):
    return len(c) == min(w, len(hs))


def _pi_nondecreasing(c):
    return all(c[i][0] >= c[0][0] + i for i in range(len(c)))


def _pi_endpoints(c):
    return not c or c[-1][0] - c[0][0] == len(c) - 1


def _pi_increasing(c):
    return all(c[i][0] < c[i + 1][0] for i in range(len(c) - 1))


def test_predicate_mutants_are_caught(monkeypatch):
    caught = []
    mutants = [("valid", _valid_any_order), ("valid", _valid_subset),
               ("valid", _valid_positions_only), ("valid", _valid_length_only),
               ("position_invariant", _pi_nondecreasing),
               ("position_invariant", _pi_endpoints),
               ("position_invariant", _pi_increasing)]
    for name, mutant in mutants:
        with monkeypatch.context() as m:
            m.setattr(lm, name, mutant)
            try:
                for w in [1, 2, 3, 5, 8]:
                    test_valid_rejects_every_other_cache(w)
                test_position_invariant_rejects_non_consecutive()
            except AssertionError:
                caught.append(mutant.__name__)
    assert caught == [f.__name__ for _, f in mutants]

"""Readers for the hand-derived golden fixtures in this folder."""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def _lines(name):
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line


def _ints(field):
    return [int(x) for x in field.split()]


def _ranges(field):
    out = []
    for tok in field.split():
        if "-" in tok:
            a, b = tok.split("-")
            out.extend(range(int(a), int(b) + 1))
        else:
            out.append(int(tok))
    return out


def last_window_cases():
    for line in _lines("last_window.txt"):
        w, hist, exp = line.split("|")
        yield int(w), _ints(hist), _ints(exp)


def step_cases():
    for line in _lines("step_cases.txt"):
        w, cache, new, exp = line.split("|")
        yield int(w), _ints(cache), int(new), _ints(exp)


def visible_set_cases():
    for line in _lines("visible_sets.txt"):
        head, exp = line.split("|")
        P, W, t = _ints(head)
        yield P, W, t, _ranges(exp)


def visible_count_cases():
    for line in _lines("visible_counts.txt"):
        head, exp = line.split("|")
        P, W, t = _ints(head)
        yield P, W, t, int(exp)

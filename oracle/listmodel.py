"""ORACLE — TEST INFRASTRUCTURE ONLY: the list model of the sliding-window cache.

Pure Python, written from "Formal verification of a sliding-window KV cache in
Lean4" (pnsm.cn blog) and the "Prefix Sliding" digest (longzhangge.com
PaperDaily).  Nothing here is shared with, or imported by, the CUDA library.

Cells are ``(pos, payload)`` tuples; the payload is opaque to the model.

- ``last_window`` / ``valid``: blog section 2.3.  The legal cache for history
  ``hs`` is ``hs`` with its first ``len(hs) - min(w, len(hs))`` cells dropped.
- ``step`` / ``run``: blog sections 3.3 and 4.2.  A token joins the end of the
  cache and only the newest ``w`` cells are kept; ``run`` folds ``step`` over a
  token stream from the empty cache.  The page's eviction condition is garbled;
  it is read as "evict when the grown cache holds more than w cells", the only
  reading under which the key equation of section 2.4 holds at the just-full
  boundary.
- ``position_invariant``: blog section 3.2 (some base with pos_i = base + i).
- ``RingBuffer`` / ``ring_to_list``: blog section 3.4 (fixed array plus head;
  logical cell i lives in slot (head + i) mod w).  The page maps all w slots;
  while the ring is not yet full that reads unwritten slots (the failure its
  section 5.1 describes), so the interpretation here maps only ``count`` slots.
- ``prefix_sliding_generation``: digest section 03 pseudocode (pinned prefix,
  window append, evict the oldest when longer than W).
"""
from __future__ import annotations

from typing import Any, Callable, Iterable, List, Sequence, Tuple

Cell = Tuple[int, Any]


def last_window(w: int, hs: Sequence[Cell]) -> List[Cell]:
    """The newest ``w`` cells of the history (all of it while it is shorter)."""
    return list(hs[max(0, len(hs) - w):])


def valid(w: int, hs: Sequence[Cell], c: Sequence[Cell]) -> bool:
    """The cache is exactly the last window of the history: same cells, same order."""
    return list(c) == last_window(w, hs)


def step(w: int, c: Sequence[Cell], kv: Cell) -> List[Cell]:
    """One token: the cache with the new cell at its end, cut back to its
    newest ``w`` cells.  For a cache of at most ``w`` cells that evicts exactly
    the oldest cell when the grown cache would hold ``w + 1``."""
    return [*c, kv][-w:]


def run(w: int, tokens: Iterable[Cell]) -> List[Cell]:
    c: List[Cell] = []
    for kv in tokens:
        c = step(w, c, kv)
    return c


def position_invariant(c: Sequence[Cell]) -> bool:
    """Some base position makes cell i hold position base + i (consecutive,
    increasing by one); the empty cache satisfies it."""
    if not c:
        return True
    base = c[0][0]
    return all(cell[0] == base + i for i, cell in enumerate(c))


class RingBuffer:
    """Physical ring: a fixed array of w slots, a head index and a fill count.

    ``push`` writes the next free slot while fewer than w cells are held;
    once full it overwrites the oldest cell (slot ``head``) and advances head.
    """

    def __init__(self, w: int, head: int = 0):
        if w < 1:
            raise ValueError("window must hold at least one cell")
        self.w = w
        self.buf: List[Any] = [None] * w
        self.head = head % w
        self.count = 0

    def push(self, kv: Cell) -> None:
        if self.count < self.w:
            self.buf[(self.head + self.count) % self.w] = kv
            self.count += 1
        else:
            self.buf[self.head] = kv
            self.head = (self.head + 1) % self.w

    def to_list(self) -> List[Cell]:
        return ring_to_list(self.w, self.buf, self.head, self.count)


def ring_to_list(w: int, buf: Sequence[Any], head: int, count: int) -> List[Any]:
    return [buf[(head + i) % w] for i in range(count)]


def prefix_sliding_generation(prefix: Sequence[Cell], W: int, T: int,
                              next_cell: Callable[[List[Cell]], Cell]) -> List[List[Cell]]:
    """Digest section 03 loop: at each step the visible cells are the pinned
    prefix followed by the window; the new cell joins the window, which then
    drops its oldest cell if it holds more than W.  Returns the visible list
    seen at each of the T steps."""
    window: List[Cell] = []
    seen = []
    for _ in range(T):
        visible = list(prefix) + list(window)
        seen.append(visible)
        window.append(next_cell(visible))
        if len(window) > W:
            window.pop(0)
    return seen


def expected_window_positions(P: int, W: int, next_pos: int) -> List[int]:
    """Positions the ring must hold once positions [P, next_pos) were appended:
    ``last_window`` of the window history, computed on the list itself."""
    hist = [(p, None) for p in range(P, next_pos)]
    return [cell[0] for cell in last_window(W, hist)]

"""Test helpers: synthetic histories from the shared generator, oracle
expectations, tolerance checks.  Used by the GPU parity tests."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import synth
from oracle import listmodel as lm

# Tolerances (stated with the workloads): fp32 max-abs 1e-5; bf16 (fp32
# accumulation, bf16 output) max-abs 2e-2 and relative L2 5e-3.
TOL_F32_ABS = 1e-5
TOL_BF16_ABS = 2e-2
TOL_BF16_RL2 = 5e-3

# Rows below the window start that the oracle is also handed (and must mask).
EVICTED_MARGIN = 64


def ps_dtype(dtype: str) -> int:
    from prefix_sliding_window_ring_b200 import PS_BF16, PS_F32
    return PS_F32 if dtype == "f32" else PS_BF16


def to_torch(arr: np.ndarray, device="cuda") -> torch.Tensor:
    """float32 values or bf16 bit patterns (uint16) -> torch tensor on device."""
    if arr.dtype == np.uint16:
        t = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr))
    return t.to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


class SeqData:
    """Synthetic history of one sequence: K/V rows by position, queries by position."""

    def __init__(self, seed: int, seq: int, Hq: int, Hkv: int, d: int, dtype: str,
                 k_scale: np.ndarray | None = None):
        self.seed, self.seq, self.Hq, self.Hkv, self.d, self.dtype = seed, seq, Hq, Hkv, d, dtype
        self.k_scale = k_scale

    def k(self, p0: int, n: int) -> np.ndarray:
        return synth.rows(self.seed, synth.TID_K, self.seq, self.Hkv, p0, n, self.d, self.dtype,
                          self.k_scale)

    def v(self, p0: int, n: int) -> np.ndarray:
        return synth.rows(self.seed, synth.TID_V, self.seq, self.Hkv, p0, n, self.d, self.dtype)

    def q(self, p0: int, n: int = 1) -> np.ndarray:
        return synth.rows(self.seed, synth.TID_Q, self.seq, self.Hq, p0, n, self.d, self.dtype)


def history_positions(P: int, W: int, t: int, margin: int = EVICTED_MARGIN) -> np.ndarray:
    """A superset of the visible rows for the query at t: the prefix plus the
    window with `margin` evicted rows below it (the oracle masks those)."""
    lo = max(P, t - W + 1 - margin)
    return np.concatenate([np.arange(0, P), np.arange(lo, t + 1)]).astype(np.int64)


def history_rows(sd: SeqData, positions: np.ndarray):
    """float64 K, V rows [n][Hkv][d] for the given sorted positions (runs fetched in bulk)."""
    n = len(positions)
    K = np.empty((n, sd.Hkv, sd.d), np.float64)
    V = np.empty((n, sd.Hkv, sd.d), np.float64)
    if n == 0:
        return K, V
    breaks = np.nonzero(np.diff(positions) != 1)[0] + 1
    starts = np.concatenate([[0], breaks])
    ends = np.concatenate([breaks, [n]])
    for a, b in zip(starts, ends):
        p0 = int(positions[a])
        K[a:b] = synth.to_f64(sd.k(p0, b - a))
        V[a:b] = synth.to_f64(sd.v(p0, b - a))
    return K, V


def oracle_decode(batch: oracle.Batch, sd: SeqData, P: int, W: int, t: int, scale: float,
                  q64: np.ndarray, hist=None) -> list:
    """Queue the oracle problems of one decode query (all Hq heads); returns the
    per-kv-head output arrays ([G][d] each) to be read after batch.run()."""
    G = sd.Hq // sd.Hkv
    if hist is None:
        hp = history_positions(P, W, t)
        K, V = history_rows(sd, hp)
    else:
        hp, K, V = hist
    outs = []
    for g in range(sd.Hkv):
        outs.append(batch.add(P, W, t, scale, q64[g * G:(g + 1) * G], hp,
                              np.ascontiguousarray(K[:, g]), np.ascontiguousarray(V[:, g])))
    return outs


def check_close(got: np.ndarray, exp: np.ndarray, dtype: str, what: str = "") -> dict:
    err = np.abs(got - exp)
    mx = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(got - exp) / max(np.linalg.norm(exp), 1e-300))
    if dtype == "f32":
        assert mx <= TOL_F32_ABS, f"{what}: max-abs {mx:.3e} > {TOL_F32_ABS}"
    else:
        assert mx <= TOL_BF16_ABS, f"{what}: max-abs {mx:.3e} > {TOL_BF16_ABS}"
        assert rl2 <= TOL_BF16_RL2, f"{what}: rel-L2 {rl2:.3e} > {TOL_BF16_RL2}"
    return {"max_abs": mx, "rel_l2": rl2}


def expected_window(P: int, W: int, next_pos: int) -> list:
    return lm.expected_window_positions(P, W, next_pos)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)

"""The five synthetic workloads (shapes and seeded draws only; no method arithmetic).

1. tiny fp32: B=1, Hq=2, Hkv=1, d=64, P=16, W=32, 200 decode steps at t=16..215.
2. boundary sweep: 1 sequence, Hq=4, Hkv=2, d=128, W in {1,2,127,128,129,4096},
   P in {0,1,100}, fp32 and bf16, decode t = P .. 3W+P.
3. decode: B=8, Hq=16, Hkv=8, d=128, P=128, W=4096, bf16, t in {2048,4224,16384,65536};
   K carries a per-(head, channel) log-normal(0,1) outlier scale.
4. ragged serving batch: 64 sequences, Hq=16, Hkv=8, d=128, W=4096, bf16,
   P_s ~ U[64,512], current length t_s ~ U[P_s, 131072], ring head h0 ~ U[0,W).
5. chunked prefill/extend: 4 sequences, 2048-query blocks at t0=100000, Hq=16,
   Hkv=8, d=128, P=256, W in {4096, 16384}, bf16.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import TID_HEAD, TID_PLEN, TID_TLEN, uniform_int


@dataclass
class Shape:
    Hq: int
    Hkv: int
    d: int
    P: int
    W: int
    dtype: str  # "f32" | "bf16"

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


TINY = dict(shape=Shape(Hq=2, Hkv=1, d=64, P=16, W=32, dtype="f32"), B=1,
            t_first=16, t_last=215, seed=0)

SWEEP_W = (1, 2, 127, 128, 129, 4096)
SWEEP_P = (0, 1, 100)
SWEEP_DTYPES = ("f32", "bf16")


def sweep_shape(W: int, P: int, dtype: str) -> Shape:
    return Shape(Hq=4, Hkv=2, d=128, P=P, W=W, dtype=dtype)


DECODE = dict(shape=Shape(Hq=16, Hkv=8, d=128, P=128, W=4096, dtype="bf16"), B=8,
              t_values=(2048, 4224, 16384, 65536), seed=0, k_outlier=True)

RAGGED_SEQS = 64
RAGGED_T_MAX = 131072
RAGGED_P_RANGE = (64, 512)


def ragged_shape() -> Shape:
    return Shape(Hq=16, Hkv=8, d=128, P=RAGGED_P_RANGE[1], W=4096, dtype="bf16")


@dataclass
class RaggedSeq:
    P: int      # pinned prefix length of this sequence
    t: int      # position decoded this step (the sequence's current length)
    h0: int     # ring-head offset of this sequence's ring buffer


def ragged_draws(seed: int = 0, nseq: int = RAGGED_SEQS, W: int = 4096,
                 t_max: int = RAGGED_T_MAX) -> list[RaggedSeq]:
    out = []
    for s in range(nseq):
        P = uniform_int(seed, TID_PLEN, s, RAGGED_P_RANGE[0], RAGGED_P_RANGE[1])
        t = uniform_int(seed, TID_TLEN, s, P, t_max)
        h0 = uniform_int(seed, TID_HEAD, s, 0, W - 1)
        out.append(RaggedSeq(P=P, t=t, h0=h0))
    return out


CHUNK = dict(B=4, n=2048, t0=100000, W_values=(4096, 16384), seed=0,
             shape_for=lambda W: Shape(Hq=16, Hkv=8, d=128, P=256, W=W, dtype="bf16"))

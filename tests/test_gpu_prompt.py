"""GPU parity of ps_attend_prompt: the prompt tokens themselves (t < P), which
attend causally to the pinned prefix rows [0, t].

Covers the tcgen05 kernel (bf16, head_dim 128, every GQA group size) and the
CUDA-core kernel (fp32, head_dim 64), prompts shorter than, equal to and longer
than one 128-row tile, prompts longer than the window (the window does not
limit prompt queries), chunked calls (bit-identical to one call), a 4096-token
prompt on sampled rows, and the argument checks."""
import numpy as np
import pytest
import torch

import oracle
from prefix_sliding_window_ring_b200 import PS_EPOS, PS_ESTATE, Cache, PSError
from tests.helpers import SeqData, check_close, default_scale, ps_dtype, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _bits(x):
    return x.view(torch.int32 if x.dtype == torch.float32 else torch.int16)


def _setup(P, W, Hq, Hkv, d, dtype, seed=8):
    sd = SeqData(seed, 0, Hq, Hkv, d, dtype)
    c = Cache(W, P, Hkv, d, ps_dtype(dtype), 1)
    c.prefill_prefix(0, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    return c, sd


def _oracle_rows(sd, P, W, rows, scale, q64):
    """float64 prompt outputs [len(rows)][Hq][d] for the given query positions."""
    import synth
    K = synth.to_f64(sd.k(0, P))
    V = synth.to_f64(sd.v(0, P))
    G = sd.Hq // sd.Hkv
    pos = np.arange(P, dtype=np.int64)
    batch = oracle.Batch()
    outs = []
    for t in rows:
        per = []
        for g in range(sd.Hkv):
            per.append(batch.add(P, W, t, scale, q64[t, g * G:(g + 1) * G], pos,
                                 np.ascontiguousarray(K[:, g]), np.ascontiguousarray(V[:, g])))
        outs.append(per)
    batch.run()
    return np.stack([np.concatenate(p, axis=0) for p in outs])


CASES = [("bf16", 128, 4, 2, P, W) for P in (1, 2, 127, 128, 129, 300) for W in (64, 4096)] + \
        [("bf16", 128, 2, 2, 257, 4096), ("bf16", 128, 8, 2, 257, 100), ("bf16", 128, 16, 2, 200, 33),
         ("f32", 64, 4, 2, 1, 8), ("f32", 64, 4, 2, 100, 16), ("bf16", 64, 8, 4, 77, 4096)]


@pytest.mark.parametrize("dtype,d,Hq,Hkv,P,W", CASES,
                         ids=[f"{dt}-d{d}-G{hq // hk}-P{P}-W{W}" for dt, d, hq, hk, P, W in CASES])
def test_prompt_matches_oracle(dtype, d, Hq, Hkv, P, W):
    c, sd = _setup(P, W, Hq, Hkv, d, dtype)
    scale = default_scale(d)
    q = to_torch(sd.q(0, P))
    out = torch.empty_like(q)
    info0 = c.seq_info(0)
    c.attend_prompt(0, q, 0, P, Hq, scale, out)
    assert c.device_error() == 0
    info1 = c.seq_info(0)
    assert (info1.next_pos, info1.count, info1.head) == (info0.next_pos, info0.count, info0.head)
    exp = _oracle_rows(sd, P, W, list(range(P)), scale, to_f64(q))
    check_close(to_f64(out), exp, dtype, f"prompt {dtype} d={d} Hq={Hq} P={P} W={W}")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_prompt_in_chunks_equals_one_call(dtype, d):
    P, W, Hq, Hkv = 300, 4096, 4, 2
    c, sd = _setup(P, W, Hq, Hkv, d, dtype)
    scale = default_scale(d)
    q = to_torch(sd.q(0, P))
    whole, parts = torch.empty_like(q), torch.empty_like(q)
    c.attend_prompt(0, q, 0, P, Hq, scale, whole)
    for a, b in [(0, 100), (100, 228), (228, 300)]:
        c.attend_prompt(0, q[a:b], a, b - a, Hq, scale, parts[a:b])
    assert c.device_error() == 0
    assert torch.equal(_bits(whole), _bits(parts))


def test_long_prompt_sampled_rows():
    """A 4096-token prompt, Hq=16, Hkv=8, bf16: every row computed, sampled rows
    (tile edges and ends) compared with the oracle."""
    P, W, Hq, Hkv, d = 4096, 4096, 16, 8, 128
    c, sd = _setup(P, W, Hq, Hkv, d, "bf16")
    scale = default_scale(d)
    q = to_torch(sd.q(0, P))
    out = torch.empty_like(q)
    c.attend_prompt(0, q, 0, P, Hq, scale, out)
    assert c.device_error() == 0
    rows = [0, 1, 63, 64, 127, 128, 129, 1000, 2047, 2048, 4094, 4095]
    exp = _oracle_rows(sd, P, W, rows, scale, to_f64(q))
    check_close(to_f64(out)[rows], exp, "bf16", "long prompt")


def test_prompt_argument_checks():
    P, W, Hq, Hkv, d = 10, 8, 2, 1, 64
    c, sd = _setup(P, W, Hq, Hkv, d, "f32")
    q = to_torch(sd.q(0, P))
    out = torch.empty_like(q)
    for t0, n in [(0, P + 1), (5, 6), (-1, 2)]:
        with pytest.raises(PSError) as e:
            c.attend_prompt(0, q, t0, n, Hq, 0.1, out)
        assert e.value.code == PS_EPOS
    empty = Cache(W, P, Hkv, d, ps_dtype("f32"), 2)
    with pytest.raises(PSError) as e:
        empty.attend_prompt(1, q, 0, 1, Hq, 0.1, out)
    assert e.value.code == PS_ESTATE
    c.attend_prompt(0, q, 3, 0, Hq, 0.1, out)  # empty range: no-op
    assert c.device_error() == 0

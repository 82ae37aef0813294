"""GPU parity: the tiny fp32 run and the boundary sweep (append + decode every step).

At every checked step the CUDA path is compared with the oracle:
- the rows the kernels visit (ps_debug_visible) against the visibility rule,
  bit-exact;
- the ring's logical contents (ps_export_window): positions against
  lastWindow of the window history, key/value bits against the generated rows;
- the decode output against float64 masked attention over the full history.
"""
import numpy as np
import pytest
import torch

import oracle
from prefix_sliding_window_ring_b200 import Cache
from synth import workloads
from tests.helpers import (SeqData, check_close, default_scale, expected_window, history_positions,
                           oracle_decode, ps_dtype, to_f64, to_torch)

pytestmark = pytest.mark.gpu


def phase_steps(P, W):
    """Decode positions at the not-full/just-full/first-eviction/wrap boundaries."""
    lens = {1, 2, W - 1, W, W + 1, W + 2, 2 * W - 1, 2 * W, 2 * W + 1, 3 * W, 3 * W + 1}
    return {P + n - 1 for n in lens if n >= 1}


def run_sweep(Hq, Hkv, d, P, W, dtype, t_last, seed=0, h0=0, every_visible=1, every_ring=1,
              every_out=1):
    sd = SeqData(seed, 0, Hq, Hkv, d, dtype)
    scale = default_scale(d)
    c = Cache(W, max(P, 1), Hkv, d, ps_dtype(dtype), 1)
    c.seq_reset(0, h0)
    T = t_last + 1
    k_np, v_np = sd.k(0, T), sd.v(0, T)
    kall, vall = to_torch(k_np), to_torch(v_np)
    qall = to_torch(sd.q(P, T - P))
    c.prefill_prefix(0, kall[:P], vall[:P], P)
    outs = torch.empty((T - P, Hq, d), dtype=kall.dtype, device="cuda")
    ws = c.decode_workspace(1, Hq)
    bits = torch.int32 if dtype == "f32" else torch.int16
    phases = phase_steps(P, W)
    out_steps = []
    for t in range(P, T):
        i = t - P
        c.append_kv([0], kall[t:t + 1], vall[t:t + 1], 1)
        c.attend_decode(qall[i:i + 1], [0], [t], Hq, scale, outs[i:i + 1], ws)
        if t in phases or i % every_visible == 0:
            vis = c.debug_visible(0, t).cpu().numpy()
            assert np.array_equal(vis, oracle.visible_positions(P, W, t)), f"visible set at t={t}"
        if t in phases or i % every_ring == 0:
            k, v, pos = c.export_window(0)
            exp = expected_window(P, W, t + 1)
            assert pos.cpu().tolist() == exp, f"ring positions at t={t}"
            idx = torch.tensor(exp, device="cuda", dtype=torch.long)
            assert torch.equal(k.view(bits), kall[idx].view(bits)), f"ring keys at t={t}"
            assert torch.equal(v.view(bits), vall[idx].view(bits)), f"ring values at t={t}"
        if t in phases or i % every_out == 0:
            out_steps.append(t)
    info = c.seq_info(0)
    assert info.next_pos == T and info.count == min(W, T - P)
    assert info.head == (h0 + max(0, T - P - W)) % W
    assert c.device_error() == 0
    # oracle over the full history (prefix + window + evicted margin, masked)
    K64, V64 = to_f64_rows(k_np), to_f64_rows(v_np)
    q64 = to_f64(qall)
    batch = oracle.Batch()
    exp_outs = []
    for t in out_steps:
        hp = history_positions(P, W, t)
        exp_outs.append(oracle_decode(batch, sd, P, W, t, scale, q64[t - P],
                                      hist=(hp, K64[hp], V64[hp])))
    batch.run()
    got = to_f64(outs)
    G = Hq // Hkv
    exp = np.stack([np.concatenate(e, axis=0) for e in exp_outs])
    stats = check_close(got[[t - P for t in out_steps]], exp, dtype,
                        f"W={W} P={P} {dtype}")
    assert exp.shape == (len(out_steps), G * Hkv, d)
    return outs, stats


def to_f64_rows(arr):
    import synth
    return synth.to_f64(arr)


def test_tiny_fp32():
    """Batch 1, 2 query heads on 1 kv head, d=64, P=16, W=32, decode t=16..215:
    ring, positions, visible set and output checked at every step."""
    cfg = workloads.TINY
    s = cfg["shape"]
    run_sweep(s.Hq, s.Hkv, s.d, s.P, s.W, s.dtype, cfg["t_last"])


SWEEP = [(W, P, dt) for W in workloads.SWEEP_W for P in workloads.SWEEP_P
         for dt in workloads.SWEEP_DTYPES]


@pytest.mark.parametrize("W,P,dtype", SWEEP, ids=[f"W{W}-P{P}-{dt}" for W, P, dt in SWEEP])
def test_boundary_sweep(W, P, dtype):
    """1 sequence, 4 query / 2 kv heads, d=128, decode t = P .. 3W+P."""
    s = workloads.sweep_shape(W, P, dtype)
    big = W > 129
    run_sweep(s.Hq, s.Hkv, s.d, P, W, dtype, 3 * W + P, h0=0,
              every_visible=16 if big else 1, every_ring=256 if big else 1,
              every_out=64 if big else 1)


@pytest.mark.parametrize("W,P,h0", [(129, 100, 77), (4096, 1, 4000), (2, 0, 1)])
def test_ring_head_offset_invariance(W, P, h0):
    """The same history gives the same outputs for any initial ring head (up to
    the order of float32 rounding: tiles split at the physical wrap of the ring)."""
    s = workloads.sweep_shape(W, P, "bf16")
    t_last = min(3 * W + P, P + W + 300)
    a, _ = run_sweep(s.Hq, s.Hkv, s.d, P, W, "bf16", t_last, h0=0, every_visible=97,
                     every_ring=997, every_out=53)
    b, _ = run_sweep(s.Hq, s.Hkv, s.d, P, W, "bf16", t_last, h0=h0, every_visible=97,
                     every_ring=997, every_out=53)
    check_close(to_f64(b), to_f64(a), "bf16", f"head offset {h0} vs 0")

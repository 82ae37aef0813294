"""The shared input generator: determinism, independence of coordinates,
rounding and distribution (CPU only)."""
import numpy as np
import torch

import synth
from synth import workloads


def test_rows_are_regenerable_per_position():
    full = synth.rows(0, synth.TID_K, 3, 2, 100, 50, 16, "f32")
    part = synth.rows(0, synth.TID_K, 3, 2, 120, 5, 16, "f32")
    assert np.array_equal(full[20:25], part)
    one = synth.normal(0, synth.TID_K, 3, 1, 130, 7)
    assert np.float32(one) == full[30, 1, 7]


def test_streams_differ():
    a = synth.rows(0, synth.TID_K, 0, 1, 0, 4, 8)
    assert not np.array_equal(a, synth.rows(0, synth.TID_V, 0, 1, 0, 4, 8))
    assert not np.array_equal(a, synth.rows(1, synth.TID_K, 0, 1, 0, 4, 8))
    assert not np.array_equal(a, synth.rows(0, synth.TID_K, 1, 1, 0, 4, 8))


def test_bf16_matches_torch_rounding():
    x = synth.rows(5, synth.TID_Q, 0, 4, 0, 256, 128, "f32")
    bits = synth.rows(5, synth.TID_Q, 0, 4, 0, 256, 128, "bf16")
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    assert np.array_equal(synth.f32_to_bf16(x), ref)
    back = synth.to_f64(bits)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_normal_moments():
    x = synth.rows(0, synth.TID_V, 0, 8, 0, 2048, 128, "f32").astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_chan_scale_lognormal():
    s = synth.chan_scale(0, 8, 128)
    assert s.shape == (8, 128) and (s > 0).all()
    assert abs(np.log(s).std() - 1.0) < 0.15


def test_ragged_draws_in_range():
    seqs = workloads.ragged_draws(0)
    assert len(seqs) == 64
    for s in seqs:
        assert 64 <= s.P <= 512 and s.P <= s.t <= 131072 and 0 <= s.h0 < 4096
    assert seqs == workloads.ragged_draws(0)

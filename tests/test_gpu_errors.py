"""Host-side validation on a live cache: every rejected call returns its status
code, enqueues nothing and leaves the sequence state unchanged."""
import pytest
import torch

from prefix_sliding_window_ring_b200 import PSError, abi, Cache
from tests.helpers import SeqData, ps_dtype, to_torch

pytestmark = pytest.mark.gpu


def code_of(fn, *a, **k):
    with pytest.raises(PSError) as e:
        fn(*a, **k)
    return e.value.code


@pytest.fixture
def cache():
    c = Cache(8, 4, 2, 64, ps_dtype("f32"), 3)
    sd = SeqData(0, 0, 4, 2, 64, "f32")
    c.prefill_prefix(0, to_torch(sd.k(0, 4)), to_torch(sd.v(0, 4)), 4)
    c.append_kv([0], to_torch(sd.k(4, 3)), to_torch(sd.v(4, 3)), 3)
    return c, sd


def state(c, s):
    i = c.seq_info(s)
    return (i.state, i.P, i.next_pos, i.head, i.count)


def test_rejections_leave_state(cache):
    c, sd = cache
    before = state(c, 0)
    k1, v1 = to_torch(sd.k(7, 1)), to_torch(sd.v(7, 1))
    q = to_torch(sd.q(6, 1))
    out = torch.empty_like(q)
    ws = c.decode_workspace(1, 4)
    assert code_of(c.append_kv, [1], k1, v1, 1) == abi.PS_ESTATE        # no prefix yet
    assert code_of(c.append_kv, [0, 0], k1, v1, 1) == abi.PS_EINVAL     # duplicate id
    assert code_of(c.append_kv, [5], k1, v1, 1) == abi.PS_EINVAL        # out of range
    assert code_of(c.append_kv, [0], k1[0, 0, 1:], v1, 1) == abi.PS_EINVAL  # misaligned
    assert code_of(c.attend_decode, q, [0], [5], 4, 0.1, out, ws) == abi.PS_EPOS   # not last
    assert code_of(c.attend_decode, q, [0], [6], 3, 0.1, out, ws) == abi.PS_EINVAL  # Hq % Hkv
    assert code_of(c.attend_decode, q, [0], [6], 6, 0.1, out, ws) == abi.PS_EUNSUPPORTED
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert code_of(abi.ps_attend_decode, c.handle, q, [0], [6], 4, 0.1, out, small, 256) == \
        abi.PS_ENOMEM
    assert code_of(c.prefill_prefix, 0, k1, v1, 1) == abi.PS_ESTATE     # prefix already set
    assert code_of(c.prefill_prefix, 1, k1, v1, 5) == abi.PS_EINVAL     # P_s > P_max
    assert code_of(c.import_window, 0, 10, k1, v1, 1) == abi.PS_EPOS    # n != min(W, 10-4)
    assert code_of(c.import_window, 0, 2, k1, v1, 0) == abi.PS_EPOS     # inside the prefix
    assert code_of(c.import_window, 0, 5, k1, v1, 1, 8) == abi.PS_EINVAL  # head offset >= W
    assert code_of(c.attend_chunk, 0, q, k1, v1, 6, 1, 4, 0.1, out) == abi.PS_EPOS  # t0 != next
    assert code_of(c.seq_reset, 0, -1) == abi.PS_EINVAL
    assert code_of(c.debug_visible, 1, 3) == abi.PS_ESTATE
    assert state(c, 0) == before
    assert c.device_error() == 0
    # the cache still works after the rejections
    c.attend_decode(q, [0], [6], 4, 0.1, out, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()


def test_decode_inside_prefix_rejected():
    c = Cache(8, 4, 1, 64, ps_dtype("f32"), 1)
    sd = SeqData(0, 0, 1, 1, 64, "f32")
    c.prefill_prefix(0, to_torch(sd.k(0, 4)), to_torch(sd.v(0, 4)), 4)
    q = to_torch(sd.q(3, 1))
    assert code_of(c.attend_decode, q, [0], [3], 1, 0.1, torch.empty_like(q)) == abi.PS_EPOS


def test_bounded_wait_times_out_and_reports():
    """A pipeline wait that nothing satisfies gives up after its limit, sets the
    time-out bit of the device error word, and leaves the context usable: a
    decode right after it runs and reports no error."""
    from prefix_sliding_window_ring_b200 import abi
    W, P, Hq, Hkv, d = 8, 2, 2, 1, 64
    c = Cache(W, P, Hkv, d, ps_dtype("f32"), 1)
    sd = SeqData(9, 0, Hq, Hkv, d, "f32")
    c.prefill_prefix(0, to_torch(sd.k(0, P)), to_torch(sd.v(0, P)), P)
    abi.ps_debug_wait_timeout(c.handle, 1 << 20)   # about half a millisecond
    assert c.device_error() == 8                  # the time-out bit, then cleared
    assert c.device_error() == 0
    q = to_torch(sd.q(P, 1))
    out = torch.empty((1, Hq, d), device="cuda")
    c.decode_step(q, to_torch(sd.k(P, 1)), to_torch(sd.v(P, 1)), [0], [P], Hq, 0.125, out)
    assert c.device_error() == 0
    assert torch.isfinite(out).all()
    with pytest.raises(PSError):
        abi.ps_debug_wait_timeout(c.handle, 0)

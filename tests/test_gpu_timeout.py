"""The bounded-wait timeout path of the attention kernel, made to run out on
purpose without faulting or hanging the GPU.

Every wait inside an attention launch gives up after the handle's wait limit
(wm_set_wait_limit).  With a limit of 0 cycles the first wait that is not
already satisfied gives up: the launch finishes the copies and tensor-core
work it started, frees its tensor memory, exits, and wm_sync_status reports
WM_ERR_TIMEOUT.  The handle must then work normally again: the next launch
with the default limit matches the oracle and reports no error.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, TINY, attend_memory
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def _status(kv, wm):
    try:
        kv.sync_status()
        return wm.WM_OK
    except wm.WmError as e:
        return e.code


@pytest.mark.parametrize("L,fused", [
    (TINY, False),
    (TINY, True),
    (Layout(24, 42, 96, 2, 24, heads=4, d=64), True),
    (Layout(5, 7, 9, 2, 9, heads=2, d=128), False),
])
def test_wait_runs_out_then_handle_recovers(wm, L, fused):
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, 1, track_records=False)
    frames = L.W + 3
    for t in range(frames):
        kv.advance(t)
        mem.advance(t)
        _, k, v = si.record_inputs(31, 0, 0, t, 0, L.R, L.heads, L.d)
        kv.write_record(0, t, dev(k), dev(v))
        mem.write_record(0, t, k, v)
    t = frames - 1
    q, k, v = si.record_inputs(31, 0, 0, t, 1, L.R, L.heads, L.d)
    o = torch.zeros(L.R, L.heads, L.d, dtype=torch.bfloat16, device="cuda")
    assert _status(kv, wm) == wm.WM_OK

    # a wait limit of 0: the launch gives up, drains and exits
    kv.set_wait_limit(0)
    if fused:
        kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
    else:
        kv.attend(0, dev(q), o)
    assert _status(kv, wm) == wm.WM_ERR_TIMEOUT
    assert _status(kv, wm) == wm.WM_OK            # the flag was read and cleared

    # the default limit again: same handle, correct results, no error
    kv.set_wait_limit(wm.DEFAULT_WAIT_LIMIT_CYCLES)
    o = torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    if fused:
        # the slot the timed-out launch was writing is undefined: write it again
        kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
        mem.write_record(0, t, k, v)
    else:
        kv.attend(0, dev(q), o)
    assert _status(kv, wm) == wm.WM_OK
    kd, vd = kv.kv_views(0)
    assert np.array_equal(host_bits(kd), mem.K[0]) and np.array_equal(host_bits(vd), mem.V[0])
    assert_attn_close(host_bits(o), attend_memory(mem, 0, q), "after the timeout")
    kv.close()


def test_timeouts_in_a_row_leave_the_device_usable(wm):
    """Several timed-out launches back to back, then a dense call on a fresh
    stream: the context stays usable."""
    L = TINY
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    kv.advance(0)
    q, k, v = si.record_inputs(32, 0, 0, 0, 0, L.R, L.heads, L.d)
    kv.write_record(0, 0, dev(k), dev(v))
    o = torch.zeros(L.R, L.heads, L.d, dtype=torch.bfloat16, device="cuda")
    kv.set_wait_limit(0)
    for _ in range(5):
        kv.attend(0, dev(q), o)
    assert _status(kv, wm) == wm.WM_ERR_TIMEOUT
    kv.set_wait_limit(wm.DEFAULT_WAIT_LIMIT_CYCLES)
    kv.attend(0, dev(q), o)
    assert _status(kv, wm) == wm.WM_OK
    mem = FrameMemory(L, 1, track_records=False)
    mem.advance(0)
    mem.write_record(0, 0, k, v)
    assert_attn_close(host_bits(o), attend_memory(mem, 0, q), "after five timeouts")
    kv.close()

"""GPU parity of the streaming sink (the start image's keys follow the window)
against the oracle: rotation schedule, bit-exact buffers after every advance,
attention within tolerance over the rotated memory."""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, attend_memory, rotation_cos_sin
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, sample_rows, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def theta_for(d, temporal=12):
    th = np.array([10000.0 ** (-2.0 * i / d) for i in range(d // 2)], dtype=np.float32)
    th[temporal:] = 0.0          # pairs outside the temporal band do not turn
    return th


@pytest.mark.parametrize("L,frames,blocks,full_rows", [
    (Layout(2, 3, 2, 1, 3, heads=2, d=64), range(22), 2, True),
    (Layout(3, 5, 2, 2, 5, heads=2, d=128), range(26), 2, True),
    (Layout(24, 42, 96, 2, 24, heads=16, d=64), range(41), 2, False),
])
def test_sink_rollout_matches_oracle(wm, L, frames, blocks, full_rows):
    th = theta_for(L.d)
    kv = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    kv.set_sink(th)
    c, s = wm.wm_sink_cos_sin(kv.h, 4, L.d // 2)
    oc, os_ = rotation_cos_sin(th.astype(np.float64), 4)
    assert np.array_equal(np.array(c, np.float32), oc) and np.array_equal(np.array(s, np.float32), os_)
    mem = FrameMemory(L, blocks, track_records=False)
    mem.sink_theta = th.astype(np.float64)
    rotated_at = []
    for t in frames:
        pos = mem.z0_pos
        kv.advance(t)
        mem.advance(t)
        if mem.z0_pos != pos:
            rotated_at.append(t)
        assert kv.sink_position() == mem.z0_pos
        for b in range(blocks):
            q, k, v = si.record_inputs(41, 0, b, t, 0, L.R, L.heads, L.d)
            o = torch.empty(L.R, L.heads, L.d, dtype=torch.bfloat16, device="cuda")
            kv.write_attend(b, t, dev(q), dev(k), dev(v), o)
            mem.write_record(b, t, k, v)
            rows = None if full_rows else sample_rows(L, t * 7 + b)
            ref = attend_memory(mem, b, q, rows=rows)
            got = host_bits(o) if rows is None else host_bits(o)[rows]
            assert_attn_close(got, ref, f"t={t} block={b}")
        torch.cuda.synchronize()
        for b in range(blocks):
            kd, vd = kv.kv_views(b)
            assert np.array_equal(host_bits(kd), mem.K[b]), f"K differs at t={t}"
            assert np.array_equal(host_bits(vd), mem.V[b]), f"V differs at t={t}"
    expected = [t for t in frames if t >= L.W + 5 and (t - (L.W + 5)) % 4 == 0]
    assert rotated_at == expected and rotated_at
    kv.sync_status()


def test_sink_state_errors(wm):
    L = Layout(2, 3, 2, 1, 3, heads=2, d=64)
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    with pytest.raises(wm.WmError) as e:
        kv.set_sink(theta_for(L.d)[:5])            # wrong number of pairs
    assert e.value.code == wm.WM_ERR_INVALID_ARG
    kv.advance(0)
    with pytest.raises(wm.WmError) as e:
        kv.set_sink(theta_for(L.d))                # after the first advance
    assert e.value.code == wm.WM_ERR_STATE
    assert kv.sink_position() == 0

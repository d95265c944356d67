"""Attention launches whose last wave is split by key range.

A launch of one CTA per (query tile, head) that makes more than one wave of
the SMs plus a remainder of at most half a wave splits the remainder's query
tiles by key range over the SMs that wave would leave idle, and a combine
launch merges the partial results.  On a 148-SM B200 these geometries make
160 (d = 64: 10 query tiles x 16 heads) and 154 (d = 128: 11 x 14) CTAs, so
the last 12 and 6 (query tile, head) pairs -- the last query tiles of the
last head -- are split.  Rows of those tiles and of unsplit ones are checked
against the oracle through the fused and the separate calls, over frames
with one to three key segments, on a bf16 memory and on an FP8 (E4M3) one
(whose V scale the combine launch applies).
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, attend_memory
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu

CASES = [
    # R = 24 * 48 + 48 = 1200 rows (10 query tiles), 16 heads; Y = 0, W = 1
    Layout(24, 48, 48, 0, 1, heads=16, d=64),
    # R = 20 * 60 + 100 = 1300 rows (11 query tiles), 14 heads; Y = 0, W = 1
    Layout(20, 60, 100, 0, 1, heads=14, d=128),
]


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def rows_to_check(L):
    # the last two query tiles (split on a 148-SM part) and the first (not split)
    last = np.arange(L.R - 150, L.R)
    return np.concatenate([np.arange(0, 40), np.arange(L.R // 2, L.R // 2 + 8), last[::3]])


@pytest.mark.parametrize("L", CASES, ids=lambda L: f"d{L.d}-h{L.heads}-R{L.R}")
def test_split_last_wave_matches_oracle(wm, L):
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, 1)
    rows = rows_to_check(L)
    for t in range(4):
        kv.advance(t)
        mem.advance(t)
        q, k, v = si.record_inputs(81, 0, 0, t, 0, L.R, L.heads, L.d)
        o = torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        if t % 2 == 0:
            kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
        else:
            kv.write_record(0, t, dev(k), dev(v))
            kv.attend(0, dev(q), o)
        mem.write_record(0, t, k, v)
        torch.cuda.synchronize()
        ob = host_bits(o)
        nan = ((ob & 0x7F80) == 0x7F80) & ((ob & 0x007F) != 0)
        assert not nan.any(), f"t={t}: {int(nan.sum())} output values were never written"
        assert_attn_close(ob[rows], attend_memory(mem, 0, q, rows=rows), f"t={t} (end {L.end(t)})")
    kd, vd = kv.kv_views(0)
    assert np.array_equal(host_bits(kd), mem.K[0]) and np.array_equal(host_bits(vd), mem.V[0])
    kv.sync_status()
    kv.close()


@pytest.mark.parametrize("L", CASES, ids=lambda L: f"d{L.d}-h{L.heads}-R{L.R}")
def test_split_last_wave_fp8_memory(wm, L):
    # scales that are not powers of two, one per head, for K and for V
    rng = np.random.default_rng(83)
    ks = rng.uniform(1 / 150, 1 / 40, size=(1, L.heads)).astype(np.float32)
    vs = rng.uniform(1 / 150, 1 / 40, size=(1, L.heads)).astype(np.float32)
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W, kv_format="e4m3",
                     k_scale=ks.ravel(), v_scale=vs.ravel())
    mem = FrameMemory(L, 1, kv_format="e4m3", k_scale=ks, v_scale=vs)
    rows = rows_to_check(L)
    for t in range(3):
        kv.advance(t)
        mem.advance(t)
        q, k, v = si.record_inputs(84, 0, 0, t, 0, L.R, L.heads, L.d)
        o = torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        if t % 2 == 0:
            kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
        else:
            kv.write_record(0, t, dev(k), dev(v))
            kv.attend(0, dev(q), o)
        mem.write_record(0, t, k, v)
        torch.cuda.synchronize()
        ob = host_bits(o)
        nan = ((ob & 0x7F80) == 0x7F80) & ((ob & 0x007F) != 0)
        assert not nan.any(), f"t={t}: {int(nan.sum())} output values were never written"
        assert_attn_close(ob[rows], attend_memory(mem, 0, q, rows=rows), f"t={t} (end {L.end(t)})")
    kd, vd = kv.kv_views(0)
    assert np.array_equal(kd.contiguous().cpu().numpy(), mem.K[0])
    assert np.array_equal(vd.contiguous().cpu().numpy(), mem.V[0])
    kv.sync_status()
    kv.close()


def test_split_sessions_on_two_streams(wm):
    """Two sessions of the split geometry (head dimension 64) driven on two
    streams with their calls interleaved, so their attention and combine
    launches may overlap on the device: each handle has its own split scratch."""
    L = CASES[0]
    sessions = [(wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W), FrameMemory(L, 1))
                for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in sessions]
    rows = rows_to_check(L)
    for t in range(3):
        ins = [si.record_inputs(85 + s, 0, 0, t, 0, L.R, L.heads, L.d) for s in range(2)]
        dins = [tuple(dev(x) for x in qkv) for qkv in ins]
        outs = [torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
                for _ in sessions]
        torch.cuda.synchronize()
        for s, (kv, mem) in enumerate(sessions):
            kv.advance(t, streams[s])
            mem.advance(t)
        for s, (kv, mem) in enumerate(sessions):
            qd, kd, vd = dins[s]
            kv.write_attend(0, t, qd, kd, vd, outs[s], streams[s])
            mem.write_record(0, t, ins[s][1], ins[s][2])
        torch.cuda.synchronize()
        for s, (kv, mem) in enumerate(sessions):
            ob = host_bits(outs[s])
            assert_attn_close(ob[rows], attend_memory(mem, 0, ins[s][0], rows=rows),
                              f"session {s} t={t}")
    for kv, _ in sessions:
        kv.sync_status()
        kv.close()

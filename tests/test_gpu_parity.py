"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Buffers (every byte of K and V) must be bit-exact; attention must be within
max-abs 2e-2 and relative L2 5e-3 of the oracle.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, SERVED, TINY, attend, attend_bits, attend_memory
from gpu_util import (assert_attn_close, dev, host_bits, require_gpu, sample_rows,
                      torch)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def nan_like(shape):
    return torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")


def check_buffers(kv, mem, blocks=None):
    torch.cuda.synchronize()
    for b in (range(mem.blocks) if blocks is None else blocks):
        kd, vd = kv.kv_views(b)
        assert np.array_equal(host_bits(kd), mem.K[b]), f"K buffer of block {b} differs at t={mem.t}"
        assert np.array_equal(host_bits(vd), mem.V[b]), f"V buffer of block {b} differs at t={mem.t}"


def roll(wm, L, blocks, frames, steps, config_id, attend_every=True, rows=None):
    """advance / write / attend through the ABI, mirrored by the oracle; checks every call."""
    kv = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, blocks)
    worst = (0.0, 0.0)
    for t in frames:
        kv.advance(t)
        mem.advance(t)
        assert kv.end() == mem.end() == L.end(t)
        check_buffers(kv, mem)
        for step in range(steps):
            for b in range(blocks):
                q, k, v = si.record_inputs(config_id, 0, b, t, step, L.R, L.heads, L.d)
                kv.write_record(b, t, dev(k), dev(v))
                mem.write_record(b, t, k, v)
                check_buffers(kv, mem, [b])
                if attend_every:
                    o = nan_like((L.R, L.heads, L.d))
                    kv.attend(b, dev(q), o)
                    ob = host_bits(o)
                    if rows is None:
                        ref = attend_memory(mem, b, q)
                    else:
                        ob = ob[rows]
                        ref = attend_memory(mem, b, q, rows=rows)
                    e = assert_attn_close(ob, ref, f"t={t} step={step} block={b}")
                    worst = max(worst[0], e[0]), max(worst[1], e[1])
        mem.check_against_records()
    kv.sync_status()
    return kv, mem, worst


def test_tiny_rollout_one_write_per_frame(wm):
    """Tiny config: frames 0..11, one write + attend per frame, all rows."""
    roll(wm, TINY, 1, range(12), 1, config_id=1)


def test_tiny_rollout_four_passes_two_blocks(wm):
    """Three denoising passes plus the clean rewrite per frame, two blocks side by side."""
    roll(wm, TINY, 2, range(12), 4, config_id=11)


@pytest.mark.parametrize("L", [Layout(2, 3, 3, 1, 5, heads=3, d=64), Layout(2, 2, 2, 0, 3, heads=1, d=64),
                               Layout(3, 5, 2, 2, 2, heads=2, d=128), Layout(5, 7, 9, 2, 9, heads=2, d=128)])
def test_small_geometries(wm, L):
    """Y = 0, W = Y (no SUM region) and d = 128 geometries, every call checked."""
    roll(wm, L, 2, range(2 * L.W + 3), 2, config_id=12)


def test_served_default_window_w16(wm):
    """The server's default window W = 16 (C = 5,760 keys): rolled to steady state, all rows of
    one block checked at t = 17..19 through the fused call."""
    L = Layout(24, 42, 96, 2, 16, heads=16, d=64)
    assert L.C == 4 * L.R + 14 * 96 == 5760
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, 1, track_records=False)
    for t in range(20):
        kv.advance(t)
        mem.advance(t)
        q, k, v = si.record_inputs(6, 0, 0, t, 0, L.R, L.heads, L.d)
        o = nan_like((L.R, L.heads, L.d))
        kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
        mem.write_record(0, t, k, v)
        check_buffers(kv, mem)
        if t >= 17:
            assert kv.end() == 5760
            assert_attn_close(host_bits(o), attend_memory(mem, 0, q), f"W=16 t={t}")
    kv.sync_status()


def test_served_single_block_steady_state(wm):
    """Served shape, one block rolled write-only to t=31; attend with all 1104 queries over 6,528 keys."""
    L = SERVED
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, 1, track_records=False)
    for t in range(32):
        kv.advance(t)
        mem.advance(t)
        _, k, v = si.record_inputs(2, 0, 0, t, 0, L.R, L.heads, L.d)
        kv.write_record(0, t, dev(k), dev(v))
        mem.write_record(0, t, k, v)
        check_buffers(kv, mem)
    assert kv.end() == 6528
    q, _, _ = si.record_inputs(2, 0, 0, 31, 1, L.R, L.heads, L.d)
    o = nan_like((L.R, L.heads, L.d))
    kv.attend(0, dev(q), o)
    kv.sync_status()
    assert_attn_close(host_bits(o), attend_memory(mem, 0, q), "served t=31")


# ------------------------------------------------------------------ dense entry point

DENSE_CASES = [(1, 1, 1, 64), (5, 3, 2, 64), (128, 128, 2, 64), (129, 300, 3, 64),
               (200, 129, 2, 64), (64, 1000, 1, 64), (300, 1000, 2, 128), (257, 129, 4, 128),
               (33, 1, 2, 128), (1104, 6528, 2, 64),
               # the page's full-resolution comparison point: 1008 raw queries x 26,208 keys
               (1008, 26208, 2, 64),
               # key counts just below, at and above multiples of the 128-key tiles,
               # and around 96 (a partly filled first tile)
               (130, 96, 2, 64), (130, 97, 2, 64), (130, 127, 1, 64), (130, 256, 1, 64),
               (130, 257, 2, 64), (130, 289, 2, 64)]


def dense_inputs(lq, lk, heads, d, tag):
    q = si.normal_bf16(si.seed_for(90, tag, lq, lk, heads * 1000 + d, si.T_Q), (lq, heads, d))
    k = si.normal_bf16(si.seed_for(90, tag, lq, lk, heads * 1000 + d, si.T_K), (lk, heads, d))
    v = si.normal_bf16(si.seed_for(90, tag, lq, lk, heads * 1000 + d, si.T_V), (lk, heads, d))
    return q, k, v


def run_dense(wm, q, k, v):
    lq, heads, d = q.shape
    lk = k.shape[0]
    o = nan_like((lq, heads, d))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    wm.wm_attend_dense(dev(q), dev(k), dev(v), o, lq, lk, heads, d, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return host_bits(o)


@pytest.mark.parametrize("lq,lk,heads,d", DENSE_CASES)
def test_dense_against_oracle(wm, lq, lk, heads, d):
    """Ragged query and key tails, several tiles, one key, both head dims."""
    q, k, v = dense_inputs(lq, lk, heads, d, 0)
    assert_attn_close(run_dense(wm, q, k, v), attend_bits(q, k, v), f"dense {lq}x{lk}x{heads}x{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_constant_values_give_ones(wm, d):
    q, k, _ = dense_inputs(300, 777, 2, d, 1)
    v = np.full(k.shape, si.f32_to_bf16_bits(np.array([1.0], np.float32))[0], np.uint16)
    o = si.bf16_bits_to_f64(run_dense(wm, q, k, v))
    assert np.abs(o - 1.0).max() <= 2.0 ** -8


@pytest.mark.parametrize("d", [64, 128])
def test_single_key_returns_value_exactly(wm, d):
    q, k, v = dense_inputs(77, 1, 3, d, 2)
    o = run_dense(wm, q, k, v)
    assert np.array_equal(o, np.broadcast_to(v, o.shape))


def test_zero_query_gives_mean(wm):
    _, k, v = dense_inputs(130, 500, 2, 64, 3)
    q = np.zeros((130, 2, 64), np.uint16)
    o = run_dense(wm, q, k, v)
    ref = np.broadcast_to(si.bf16_bits_to_f64(v).mean(axis=0), (130, 2, 64))
    assert_attn_close(o, ref, "zero query")


def test_permuted_keys_same_output(wm):
    q, k, v = dense_inputs(256, 900, 2, 64, 4)
    perm = np.random.default_rng(7).permutation(900)
    o1 = run_dense(wm, q, k, v)
    o2 = run_dense(wm, q, k[perm], v[perm])
    ref = attend_bits(q, k, v)
    assert_attn_close(o1, ref, "original order")
    assert_attn_close(o2, ref, "permuted order")


@pytest.mark.parametrize("d", [64, 128])
def test_wide_score_range_exercises_rescaling(wm, d):
    """K rows scaled by up to 8x: the running max moves often and O is rescaled in TMEM."""
    q, k, v = dense_inputs(256, 1500, 2, d, 5)
    kf = si.bf16_bits_to_f32(k) * np.linspace(0.25, 8.0, 1500, dtype=np.float32)[:, None, None]
    k2 = si.f32_to_bf16_bits(kf)
    assert_attn_close(run_dense(wm, q, k2, v), attend_bits(q, k2, v), "wide range")


def test_sampled_rows_helper_is_in_range():
    rows = sample_rows(SERVED, 0)
    assert rows.min() == 0 and rows.max() == SERVED.R - 1 and len(rows) >= 60


# ------------------------------------------------------------ fused write + attend

@pytest.mark.parametrize("L,frames", [
    (TINY, range(12)),
    (Layout(24, 42, 96, 2, 24, heads=4, d=64), range(30)),
    (Layout(3, 5, 2, 0, 4, heads=2, d=64), range(9)),
    (Layout(5, 7, 9, 2, 9, heads=2, d=128), range(14)),
    # record and summary lengths multiples of 8: each of the three key segments
    # ends in a partly filled tile whose missing rows are masked
    (Layout(4, 4, 8, 2, 6, heads=2, d=64), range(12)),
    (Layout(8, 10, 16, 1, 7, heads=2, d=64), range(14)),
])
def test_write_attend_equals_write_then_attend(wm, L, frames):
    """One launch (keys: buffer before/after the slot + the record from the caller) gives
    the same buffer bytes as write_record followed by attend, and the same attention."""
    blocks = 2
    a = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    b = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, blocks, track_records=False)
    for t in frames:
        a.advance(t)
        b.advance(t)
        mem.advance(t)
        for step in range(2):
            for blk in range(blocks):
                q, k, v = si.record_inputs(21, 0, blk, t, step, L.R, L.heads, L.d)
                qd, kd, vd = dev(q), dev(k), dev(v)
                oa, ob = nan_like((L.R, L.heads, L.d)), nan_like((L.R, L.heads, L.d))
                a.write_record(blk, t, kd, vd)
                a.attend(blk, qd, oa)
                b.write_attend(blk, t, qd, kd, vd, ob)
                mem.write_record(blk, t, k, v)
                ref = attend_memory(mem, blk, q)
                assert_attn_close(host_bits(oa), ref, f"separate t={t}")
                assert_attn_close(host_bits(ob), ref, f"fused t={t}")
        torch.cuda.synchronize()
        for blk in range(blocks):
            ka, va = a.kv_views(blk)
            kb, vb = b.kv_views(blk)
            assert torch.equal(ka, kb) and torch.equal(va, vb), f"buffers differ at t={t}"
            assert np.array_equal(host_bits(kb), mem.K[blk]) and np.array_equal(host_bits(vb), mem.V[blk])
    a.sync_status()
    b.sync_status()


def test_write_attend_state_errors(wm):
    L = TINY
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    q = torch.zeros(L.R, L.heads, L.d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wm.WmError) as e:
        kv.write_attend(0, 0, q, q, q, q)          # before advance(0)
    assert e.value.code == wm.WM_ERR_STATE
    kv.advance(0)
    with pytest.raises(wm.WmError) as e:
        kv.write_attend(0, 1, q, q, q, q)          # wrong frame
    assert e.value.code == wm.WM_ERR_STATE
    with pytest.raises(wm.WmError) as e:
        kv.write_attend(1, 0, q, q, q, q)          # no such block
    assert e.value.code == wm.WM_ERR_INVALID_ARG
    kv.write_attend(0, 0, q, q, q, q)
    kv.sync_status()

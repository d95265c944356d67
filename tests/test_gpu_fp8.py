"""GPU parity of the FP8 (E4M3) frame memory against the oracle (reading R7).

Stored codes must be bit-exact after every call (the quantisation divides in
float32 and rounds to nearest even with saturation on both sides); attention
must be within max-abs 2e-2 and relative L2 5e-3 of the oracle's fp64
attention over the dequantised prefix -- the same tolerance as the bf16
buffer, since the codes are widened exactly and the scales are applied in
float32.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import (FrameMemory, Layout, SERVED, TINY, attend, attend_memory, dequantize_e4m3,
                    e4m3_encode)
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, sample_rows, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def make_scales(blocks, heads, seed, saturate_head=True):
    """Scales that are not powers of two (so the float32 division rounds); with
    N(0,1) values, 1/40 .. 1/150 keeps most codes normal, and one head at 1/200
    pushes values beyond 2.24 into saturation."""
    rng = np.random.default_rng(seed)
    ks = rng.uniform(1 / 150, 1 / 40, size=(blocks, heads)).astype(np.float32)
    vs = rng.uniform(1 / 150, 1 / 40, size=(blocks, heads)).astype(np.float32)
    if saturate_head:
        ks[:, 0] = np.float32(1 / 200)
    return ks, vs


def pair(wm, L, blocks, ks, vs):
    kv = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W, kv_format="e4m3",
                     k_scale=ks.ravel(), v_scale=vs.ravel())
    mem = FrameMemory(L, blocks, kv_format="e4m3", k_scale=ks, v_scale=vs)
    assert wm.wm_kv_format(kv.h) == wm.WM_KV_E4M3
    return kv, mem


def codes(t):
    return t.contiguous().cpu().numpy()


def check_codes(kv, mem, blocks=None):
    torch.cuda.synchronize()
    for b in (range(mem.blocks) if blocks is None else blocks):
        kd, vd = kv.kv_views(b)
        assert np.array_equal(codes(kd), mem.K[b]), f"K codes of block {b} differ at t={mem.t}"
        assert np.array_equal(codes(vd), mem.V[b]), f"V codes of block {b} differ at t={mem.t}"


def nan_out(L):
    return torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")


@pytest.mark.parametrize("L,fused", [
    (TINY, False), (TINY, True),
    (Layout(2, 2, 2, 0, 3, heads=1, d=64), True),
    (Layout(3, 5, 2, 2, 2, heads=2, d=128), False),
    (Layout(5, 7, 9, 2, 9, heads=2, d=128), True),
])
def test_fp8_rollout_every_call(wm, L, fused):
    blocks = 2
    ks, vs = make_scales(blocks, L.heads, 1)
    kv, mem = pair(wm, L, blocks, ks, vs)
    for t in range(2 * L.W + 3):
        kv.advance(t)
        mem.advance(t)
        check_codes(kv, mem)
        for step in range(2):
            for b in range(blocks):
                q, k, v = si.record_inputs(50, 0, b, t, step, L.R, L.heads, L.d)
                o = nan_out(L)
                if fused:
                    kv.write_attend(b, t, dev(q), dev(k), dev(v), o)
                else:
                    kv.write_record(b, t, dev(k), dev(v))
                    kv.attend(b, dev(q), o)
                mem.write_record(b, t, k, v)
                check_codes(kv, mem, [b])
                assert_attn_close(host_bits(o), attend_memory(mem, b, q), f"t={t} step={step} b={b}")
        mem.check_against_records()
    kv.sync_status()
    kv.close()


def test_fp8_served_single_block_steady_state(wm):
    """Served shape (16 x 64, 1104 queries over 6,528 keys), rolled to t = 31, all rows."""
    L = SERVED
    ks, vs = make_scales(1, L.heads, 2)
    kv, mem = pair(wm, L, 1, ks, vs)
    for t in range(32):
        kv.advance(t)
        mem.advance(t)
        _, k, v = si.record_inputs(51, 0, 0, t, 0, L.R, L.heads, L.d)
        kv.write_record(0, t, dev(k), dev(v))
        mem.write_record(0, t, k, v)
    check_codes(kv, mem)
    sat = (mem.K[0, :, 0] & 0x7F) == 0x7E                   # +-448: saturated codes of head 0
    assert sat.sum() > 1000                                 # saturation is exercised
    q, _, _ = si.record_inputs(51, 0, 0, 31, 1, L.R, L.heads, L.d)
    o = nan_out(L)
    kv.attend(0, dev(q), o)
    kv.sync_status()
    assert_attn_close(host_bits(o), attend_memory(mem, 0, q), "fp8 served t=31")
    kv.close()


def test_fp8_batch_workload_scaled_keys_sampled_rows(wm):
    """Served shape with K rows scaled per token by U(0.5, 2), three blocks in steady state,
    sampled rows of every attend, fused calls."""
    L = Layout(24, 42, 96, 2, 24, heads=16, d=64)
    blocks = 3
    ks, vs = make_scales(blocks, L.heads, 3, saturate_head=False)
    kv, mem = pair(wm, L, blocks, ks, vs)
    rows = sample_rows(L, 5)
    for t in range(34):
        kv.advance(t)
        mem.advance(t)
        for b in range(blocks):
            q, k, v = si.record_inputs(4, 2, b, t, 0, L.R, L.heads, L.d, k_row_scale=True)
            o = nan_out(L)
            kv.write_attend(b, t, dev(q), dev(k), dev(v), o)
            mem.write_record(b, t, k, v)
            if t >= 31:
                assert_attn_close(host_bits(o)[rows], attend_memory(mem, b, q, rows=rows), f"t={t} b={b}")
    check_codes(kv, mem)
    kv.sync_status()
    kv.close()


DENSE = [(1, 1, 1, 64), (129, 300, 3, 64), (200, 129, 2, 64), (1104, 6528, 2, 64), (300, 1000, 2, 128),
         (33, 1, 2, 128), (257, 4000, 4, 128)]


@pytest.mark.parametrize("lq,lk,heads,d", DENSE)
def test_fp8_dense_against_oracle(wm, lq, lk, heads, d):
    rng = np.random.default_rng(lq * 7 + lk)
    q = si.normal_bf16(si.seed_for(91, 0, lq, lk, heads * 1000 + d, si.T_Q), (lq, heads, d))
    kf = rng.standard_normal((lk, heads, d)).astype(np.float32) * 2
    vf = rng.standard_normal((lk, heads, d)).astype(np.float32)
    ks = rng.uniform(1 / 100, 1 / 20, heads).astype(np.float32)
    vs = rng.uniform(1 / 100, 1 / 20, heads).astype(np.float32)
    k8 = e4m3_encode(kf / ks[None, :, None])
    v8 = e4m3_encode(vf / vs[None, :, None])
    o = torch.full((lq, heads, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    nbytes = wm.wm_attend_dense_fp8_scratch_bytes(lk, heads, d)
    scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    wm.wm_attend_dense_fp8(dev(q), torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda(),
                           torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), o, lq, lk, heads,
                           d, scratch, nbytes, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = attend(si.bf16_bits_to_f64(q), dequantize_e4m3(k8, ks), dequantize_e4m3(v8, vs))
    assert_attn_close(host_bits(o), ref, f"dense fp8 {lq}x{lk}x{heads}x{d}")


def test_fp8_rejects_sink_and_small_scratch(wm):
    L = TINY
    ks, vs = make_scales(1, L.heads, 4)
    kv, _ = pair(wm, L, 1, ks, vs)
    with pytest.raises(wm.WmError) as e:
        kv.set_sink([0.1] * (L.d // 2))
    assert e.value.code == wm.WM_ERR_UNSUPPORTED
    kv.close()
    x = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(wm.WmError) as e:
        wm.wm_attend_dense_fp8(x, x, x, x, x, x, 1, 100, 1, 64, x, 100 * 64 * 4 - 16)
    assert e.value.code == wm.WM_ERR_INVALID_ARG

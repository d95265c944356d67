"""GPU parity over seeded random geometries: for each, a short rollout
through the C ABI (advance, fused write+attend on even frames, write then
attend on odd ones), with every byte of every buffer compared against the
oracle after each frame and every attention output within the oracle
tolerance (max-abs 2e-2, relative L2 5e-3).  Geometries: head dimension 64
or 128, 1..4 heads, grids of 1..6 x 1..7, X = 1..12, Y = 0..3, W = Y..Y+5
(tiny records, one-row and ragged 128-row tiles, W = Y); two of them on the
FP8 (E4M3) memory."""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, attend_memory
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu

BLOCKS = 2


def geometries(n=12, seed=777):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        y = int(rng.integers(0, 4))
        d = 64 if i % 3 else 128
        out.append(Layout(int(rng.integers(1, 7)), int(rng.integers(1, 8)), int(rng.integers(1, 13)), y,
                          y + int(rng.integers(0, 6)), heads=int(rng.integers(1, 5)), d=d))
    return out


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def _rollout(wm, L, fmt, seed):
    if fmt == "e4m3":
        rng = np.random.default_rng(seed)
        ks = rng.uniform(1 / 150, 1 / 40, size=(BLOCKS, L.heads)).astype(np.float32)
        vs = rng.uniform(1 / 150, 1 / 40, size=(BLOCKS, L.heads)).astype(np.float32)
        kv = wm.KVMemory(BLOCKS, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W, kv_format="e4m3",
                         k_scale=ks.ravel(), v_scale=vs.ravel())
        mem = FrameMemory(L, BLOCKS, kv_format="e4m3", k_scale=ks, v_scale=vs)
        to_host = lambda x: x.contiguous().cpu().numpy()
    else:
        kv = wm.KVMemory(BLOCKS, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
        mem = FrameMemory(L, BLOCKS)
        to_host = host_bits
    for t in range(L.W + 4):
        kv.advance(t)
        mem.advance(t)
        for b in range(BLOCKS):
            q, k, v = si.record_inputs(seed, 0, b, t, 0, L.R, L.heads, L.d)
            o = torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
            if t % 2 == 0:
                kv.write_attend(b, t, dev(q), dev(k), dev(v), o)
            else:
                kv.write_record(b, t, dev(k), dev(v))
                kv.attend(b, dev(q), o)
            mem.write_record(b, t, k, v)
            torch.cuda.synchronize()
            assert_attn_close(host_bits(o), attend_memory(mem, b, q), f"t={t} block={b}")
        for b in range(BLOCKS):
            kd, vd = kv.kv_views(b)
            assert np.array_equal(to_host(kd), mem.K[b]), f"K buffer of block {b} at t={t}"
            assert np.array_equal(to_host(vd), mem.V[b]), f"V buffer of block {b} at t={t}"
    kv.sync_status()
    kv.close()


@pytest.mark.parametrize("i,L", list(enumerate(geometries())),
                         ids=lambda x: x if isinstance(x, int) else
                         f"{x.grid_h}x{x.grid_w}-X{x.X}-Y{x.Y}-W{x.W}-h{x.heads}-d{x.d}")
def test_random_geometry_rollout(wm, i, L):
    _rollout(wm, L, "e4m3" if i in (1, 5) else "bf16", 900 + i)

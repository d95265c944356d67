"""Head-dimension-128 attention through a handle: one O shared by the two
softmax warpgroups, with one exponent reference per row fixed from their
first key tiles, and an exact recomputation of any (query tile, head) whose
row max later outgrows that reference's headroom.

The case that needs the recomputation: two keys aligned with one query row,
at 6x and 9x that query, in two different late tiles (the caller's record,
the last key segment of the fused write+attend), so that two tiles overflow
the fixed reference by different amounts.  Clamping each tile to the
headroom would weigh them alike; the exact result follows the larger one.
Rows of every frame are checked against the fp64 oracle, through the fused
and the separate calls.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, attend_memory
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu

L = Layout(8, 16, 16, 1, 2, heads=2, d=128)   # R = 144, capacity 448 keys


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def scaled_bits(bits, c):
    """bf16 bit array -> the bf16 bits of c times its values (round to nearest even)."""
    x = (bits.astype(np.uint32) << 16).view(np.float32) * np.float32(c)
    b = x.view(np.uint32).astype(np.uint64)
    return (((b + 0x7FFF + ((b >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


@pytest.mark.parametrize("fused", [True, False])
def test_keys_far_above_the_first_tiles(wm, fused):
    kv = wm.KVMemory(1, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, 1)
    row = 3
    for t in range(5):
        kv.advance(t)
        mem.advance(t)
        q, k, v = si.record_inputs(91, 0, 0, t, 0, L.R, L.heads, L.d)
        if t >= 3:
            k = k.copy()
            k[0, 0] = scaled_bits(q[row, 0], 6.0)            # record tile 0
            k[L.R - 2, 0] = scaled_bits(q[row, 0], 9.0)      # record tile 1
        o = torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        if fused:
            kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
        else:
            kv.write_record(0, t, dev(k), dev(v))
            kv.attend(0, dev(q), o)
        mem.write_record(0, t, k, v)
        torch.cuda.synchronize()
        ob = host_bits(o)
        assert_attn_close(ob, attend_memory(mem, 0, q), f"t={t} fused={fused}")
    kv.sync_status()
    kv.close()

"""Head-dimension-128 attention: one O shared by the two softmax warpgroups,
with one exponent reference per row fixed from their first key tiles, and an
exact recomputation, by the CTA itself before it exits, of the rows of any
CTA in which a later tile's row max outgrew that reference's headroom.

The case that needs the recomputation: two keys aligned with one query row,
at 6x and 9x that query, in two different late tiles, so that two tiles
overflow the fixed reference by different amounts.  Clamping each tile to
the headroom would weigh them alike; the exact result follows the larger
one.  Checked against the fp64 oracle through the fused and the separate
calls of a handle (the keys in the record, the fused call's last segment),
through the dense call, and on a geometry whose last wave is split by key
range (the recomputation then writes a piece's partial result).
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, attend_bits, attend_memory
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


def test_dense_call_keys_far_above_the_first_tiles(wm):
    lq, lk, heads, d = 200, 700, 3, 128
    q = si.normal_bf16(931, (lq, heads, d))
    k = si.normal_bf16(932, (lk, heads, d)).copy()
    v = si.normal_bf16(933, (lk, heads, d))
    row = 150                                        # query tile 1
    k[300, 1] = scaled_bits(q[row, 1], 6.0)          # key tile 2
    k[650, 1] = scaled_bits(q[row, 1], 9.0)          # key tile 5
    o = torch.full((lq, heads, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    wm.wm_attend_dense(dev(q), dev(k), dev(v), o, lq, lk, heads, d, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_attn_close(host_bits(o), attend_bits(q, k, v), "dense d=128")


def test_split_piece_keys_far_above_the_first_tiles(wm):
    # 11 query tiles x 14 heads = 154 CTAs on a 148-SM part: the last six
    # (query tile, head) items are split by key range, 4 key tiles a piece.
    # At frame 8 the buffer holds 10,500 keys and the record sits at rows
    # 1,300-2,599 (head dimension 128 attends over the buffer in one segment
    # once the record is stored); record rows 1,050 and 1,200 are buffer rows
    # 2,350 and 2,500, key tiles 18 and 19: the third and fourth tiles of the
    # piece of tiles 16-19, so that piece must recompute its partial result
    # (one overflowing tile per piece would be harmless after the merge)
    Ls = Layout(20, 60, 100, 6, 7, heads=14, d=128)
    kv = wm.KVMemory(1, Ls.heads, Ls.d, Ls.grid_h, Ls.grid_w, Ls.X, Ls.Y, Ls.W)
    mem = FrameMemory(Ls, 1)
    row = Ls.R - 5                                   # the last query tile
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(Ls.R - 128, Ls.R, 2), [row]]))
    for t in range(9):
        kv.advance(t)
        mem.advance(t)
        q, k, v = si.record_inputs(94, 0, 0, t, 0, Ls.R, Ls.heads, Ls.d)
        if t == 8:
            k = k.copy()
            k[1050, 13] = scaled_bits(q[row, 13], 6.0)
            k[1200, 13] = scaled_bits(q[row, 13], 9.0)
        o = torch.full((Ls.R, Ls.heads, Ls.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        kv.write_attend(0, t, dev(q), dev(k), dev(v), o)
        mem.write_record(0, t, k, v)
        if t >= 7:
            torch.cuda.synchronize()
            ob = host_bits(o)
            assert_attn_close(ob[rows], attend_memory(mem, 0, q, rows=rows), f"t={t} split")
    kv.sync_status()
    kv.close()

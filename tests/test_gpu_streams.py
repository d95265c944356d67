"""Sessions on separate CUDA streams: three handles (two bf16, one FP8) driven
frame by frame on three non-default streams with their calls interleaved on
the host, so their kernels may overlap on the device.  Each handle keeps its
own buffers, status word and (FP8) widening scratch, and programmatic
dependent launch orders each stream's own kernels only; the outputs and
every buffer byte must match each session's oracle."""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, Layout, attend_memory
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu

L = Layout(4, 6, 5, 1, 4, heads=2, d=64)
BLOCKS = 3


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def test_three_sessions_on_three_streams(wm):
    rng = np.random.default_rng(71)
    ks = rng.uniform(1 / 150, 1 / 40, size=(BLOCKS, L.heads)).astype(np.float32)
    vs = rng.uniform(1 / 150, 1 / 40, size=(BLOCKS, L.heads)).astype(np.float32)
    sessions = [
        (wm.KVMemory(BLOCKS, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W), FrameMemory(L, BLOCKS),
         host_bits),
        (wm.KVMemory(BLOCKS, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W), FrameMemory(L, BLOCKS),
         host_bits),
        (wm.KVMemory(BLOCKS, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W, kv_format="e4m3",
                     k_scale=ks.ravel(), v_scale=vs.ravel()),
         FrameMemory(L, BLOCKS, kv_format="e4m3", k_scale=ks, v_scale=vs),
         lambda x: x.contiguous().cpu().numpy()),
    ]
    streams = [torch.cuda.Stream() for _ in sessions]
    for t in range(2 * L.W + 3):
        # this frame's inputs, on the device before any session stream uses them
        ins = {}
        for s in range(len(sessions)):
            for b in range(BLOCKS):
                q, k, v = si.record_inputs(72 + s, 0, b, t, 0, L.R, L.heads, L.d)
                ins[s, b] = (q, k, v, dev(q), dev(k), dev(v))
        outs = {(s, b): torch.full((L.R, L.heads, L.d), float("nan"), dtype=torch.bfloat16,
                                   device="cuda") for s in range(len(sessions)) for b in range(BLOCKS)}
        torch.cuda.synchronize()
        for s, (kv, mem, _) in enumerate(sessions):
            kv.advance(t, streams[s])
            mem.advance(t)
        for b in range(BLOCKS):
            for s, (kv, mem, _) in enumerate(sessions):
                q, k, v, qd, kd, vd = ins[s, b]
                if (t + s) % 2 == 0:
                    kv.write_attend(b, t, qd, kd, vd, outs[s, b], streams[s])
                else:
                    kv.write_record(b, t, kd, vd, streams[s])
                    kv.attend(b, qd, outs[s, b], streams[s])
                mem.write_record(b, t, k, v)
        torch.cuda.synchronize()
        for s, (kv, mem, to_host) in enumerate(sessions):
            for b in range(BLOCKS):
                q = ins[s, b][0]
                assert_attn_close(host_bits(outs[s, b]), attend_memory(mem, b, q),
                                  f"session {s} t={t} block={b}")
                kb, vb = kv.kv_views(b)
                assert np.array_equal(to_host(kb), mem.K[b]), f"session {s} K block {b} t={t}"
                assert np.array_equal(to_host(vb), mem.V[b]), f"session {s} V block {b} t={t}"
    for kv, _, _ in sessions:
        kv.sync_status()
        kv.close()

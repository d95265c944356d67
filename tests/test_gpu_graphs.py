"""Frame-steps captured as CUDA graphs through the C ABI replay exactly.

The bench's graph measurement captures one frame-step per graph for one
period of the slot pattern and replays the graphs in order; this checks, on
the tiny layout (period lcm(Y+1, W-Y) = 12), that a replayed rollout leaves
every byte of K and V and every output equal to the same calls made eagerly,
and that those buffers are the oracle's.
"""
import math

import numpy as np
import pytest

import seeded_inputs as si
from oracle import FrameMemory, TINY, attend_memory
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager_and_oracle():
    require_gpu()
    import kv_memory_attention_b200 as wm
    L, blocks = TINY, 2
    period = math.lcm(L.Y + 1, L.W - L.Y)
    t0 = L.W + 1                                   # steady state
    eager = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    graphed = wm.KVMemory(blocks, L.heads, L.d, L.grid_h, L.grid_w, L.X, L.Y, L.W)
    mem = FrameMemory(L, blocks)
    inputs = {b: [dev(x) for x in si.record_inputs(21, 0, b, 0, 0, L.R, L.heads, L.d)]
              for b in range(blocks)}
    for t in range(t0):
        for kv in (eager, graphed):
            kv.advance(t)
        mem.advance(t)
        for b in range(blocks):
            q, k, v = inputs[b]
            for kv in (eager, graphed):
                kv.write_record(b, t, k, v)
            mem.write_record(b, t, host_bits(k), host_bits(v))
    o_eager = {b: torch.empty(L.R, L.heads, L.d, dtype=torch.bfloat16, device="cuda")
               for b in range(blocks)}
    o_graph = {b: torch.empty_like(o_eager[b]) for b in range(blocks)}

    def step(kv, t, outs, stream=None):
        kv.advance(t, stream)
        for b in range(blocks):
            q, k, v = inputs[b]
            kv.write_attend(b, t, q, k, v, outs[b], stream)

    cap = torch.cuda.Stream()
    graphs = []
    torch.cuda.synchronize()
    for i in range(period):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(graphed, t0 + i, o_graph, torch.cuda.current_stream())
        graphs.append(g)
    # two cycles: the second replays frames t0+period.. (same slots)
    for cycle in range(2):
        for i, g in enumerate(graphs):
            t = t0 + cycle * period + i
            g.replay()
            step(eager, t, o_eager)
            mem.advance(t)
            for b in range(blocks):
                q, k, v = inputs[b]
                mem.write_record(b, t, host_bits(k), host_bits(v))
            torch.cuda.synchronize()
            for b in range(blocks):
                assert np.array_equal(host_bits(o_graph[b]), host_bits(o_eager[b])), (t, b)
    torch.cuda.synchronize()
    eager.sync_status()
    graphed.sync_status()
    for b in range(blocks):
        ke, ve = eager.kv_views(b)
        kg, vg = graphed.kv_views(b)
        assert np.array_equal(host_bits(kg), host_bits(ke))
        assert np.array_equal(host_bits(vg), host_bits(ve))
        assert np.array_equal(host_bits(ke), mem.K[b])
        assert np.array_equal(host_bits(ve), mem.V[b])
        assert_attn_close(host_bits(o_graph[b]), attend_memory(mem, b, host_bits(inputs[b][0])),
                          f"graph replay, block {b}")
    del graphs

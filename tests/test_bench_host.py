"""Host-side facts bench.py relies on, checked against the oracle's layout.

The CUDA-graph measurement replays one captured frame-step per frame for
GRAPH_PERIOD frames, in order, again and again; that continues the rollout
exactly only if every slot a frame-step touches repeats with that period.
"""
import os
import sys

from oracle import SERVED

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _touched(L, t):
    """What frame-step t touches: the record's rows, the evicted frame's
    source and destination rows, and the filled prefix."""
    ev = L.evicted_frame(t)
    evict = None if ev is None else (L.raw_slot(ev), L.sum_slot(ev))
    return (tuple(L.record_rows(t)), evict, L.end(t))


def test_graph_period_is_the_served_slot_period():
    L = SERVED
    P = bench.GRAPH_PERIOD
    assert (bench.Y, bench.W, bench.X, bench.GH, bench.GW) == (L.Y, L.W, L.X, L.grid_h, L.grid_w)
    steady = range(bench.T_STEADY, bench.T_STEADY + 3 * P)
    for t in steady:
        assert _touched(L, t) == _touched(L, t + P), t
    # and it is the smallest such period
    for q in range(1, P):
        assert any(_touched(L, t) != _touched(L, t + q) for t in steady), q


def test_copy_byte_counts():
    L = SERVED
    row = bench.HEADS * bench.D * 2
    assert bench.EVICT_BYTES == 2 * 2 * L.X * row * bench.BLOCKS
    assert bench.WRITE_BYTES == 2 * 2 * L.R * row

"""Host layout arithmetic of the C ABI against the oracle over seeded random
geometries (no kernel is launched): capacity, the filled prefix end(t), the
record's first row and the RAW / SUM slots, for t = 0 .. 3 (W + 2), over
grids of 1..40 x 1..50, X = 1..128, Y = 0..6 and W = Y..Y+30 (W = Y, no SUM
region, included)."""
import numpy as np
import pytest

from oracle import Layout


def geometries(n=60, seed=20240):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        y = int(rng.integers(0, 7))
        out.append(Layout(int(rng.integers(1, 41)), int(rng.integers(1, 51)), int(rng.integers(1, 129)),
                          y, y + int(rng.integers(0, 31))))
    return out


@pytest.fixture(scope="module")
def wm():
    import kv_memory_attention_b200 as wm
    return wm


@pytest.mark.parametrize("L", geometries(), ids=lambda L: f"{L.grid_h}x{L.grid_w}-X{L.X}-Y{L.Y}-W{L.W}")
def test_random_geometry_layout(wm, L):
    gh, gw, X, Y, W = L.grid_h, L.grid_w, L.X, L.Y, L.W
    assert wm.wm_layout_capacity(gh, gw, X, Y, W) == L.C
    for t in range(0, 3 * (W + 2) + 1):
        assert wm.wm_layout_end(gh, gw, X, Y, W, t) == L.end(t), t
        assert wm.wm_layout_record_row(gh, gw, X, Y, t) == L.record_rows(t)[0], t
        if t >= 1:
            assert wm.wm_layout_raw_slot(Y, t) == L.raw_slot(t)
            assert wm.wm_layout_sum_slot(Y, W, t) == (L.sum_slot(t) if W > Y else -1)
    # from frame W + 1 on (SUM full) the filled prefix is the whole buffer
    assert wm.wm_layout_end(gh, gw, X, Y, W, W + 1) == L.C
    assert wm.wm_layout_end(gh, gw, X, Y, W, W) < L.C or W == Y

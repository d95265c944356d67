"""The attention kernel's polynomial exponential (3 of every 8 exponentials at
head dimension 64) against 2^x computed in float64 on the host, on the
device, through wm_selftest_exp2: relative error within the 1.7e-3 the
polynomial was fitted to, over the arguments the softmax can produce (the
lazy rescale keeps them at most 8) and the whole range where the bit
arithmetic is valid ([-125, 127]); 2^-125 below it."""
import numpy as np
import pytest

from gpu_util import require_gpu, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def run(wm, x):
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    wm.wm_selftest_exp2(xd, yd, x.size)
    torch.cuda.synchronize()
    return yd.cpu().numpy()


def test_relative_error_over_the_softmax_range(wm):
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-125.0, 127.0, 2_000_000), rng.uniform(-20.0, 8.0, 2_000_000),
                        np.arange(-125, 128, dtype=np.float64) + 0.5,      # reduction boundaries
                        np.arange(-125, 128, dtype=np.float64)]).astype(np.float32)
    x = x[: x.size // 2 * 2]
    y = run(wm, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert np.isfinite(y).all() and (y > 0).all()
    assert rel.max() <= 1.75e-3, rel.max()
    # a minimax fit's error equioscillates over the reduced interval, so its mean
    # magnitude is about 2/pi of the maximum (1.08e-3 for 1.7e-3), not far above
    assert rel.mean() <= 0.7 * 1.75e-3


def test_below_range_clamps_and_zero_is_one(wm):
    x = np.array([-126.0, -500.0, -np.inf, 0.0], np.float32)
    y = run(wm, x)
    assert np.all(y[:3] == np.float32(2.0 ** -125) * np.float32(y[3]))
    assert abs(float(y[3]) - 1.0) <= 1.75e-3

"""Helpers shared by the GPU parity tests (device transfers, tolerance checks).

Attention tolerance against the fp64 oracle: max-abs 2e-2 and relative L2
5e-3 over the compared outputs.  Buffer contents and slot indexing must be
bit-exact.
"""
import numpy as np
import pytest

import seeded_inputs as si

MAX_ABS = 2e-2
REL_L2 = 5e-3

torch = pytest.importorskip("torch")


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def dev(bits: np.ndarray):
    """bf16 bit array (uint16) -> CUDA bf16 tensor of the same shape."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit array."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def attn_errors(o_bits: np.ndarray, ref: np.ndarray):
    o = si.bf16_bits_to_f64(o_bits)
    assert o.shape == ref.shape
    assert np.isfinite(o).all()
    diff = o - ref
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel


def assert_attn_close(o_bits, ref, what=""):
    max_abs, rel = attn_errors(o_bits, ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


class DevicePool:
    """The seeded generator's sample pool, resident on the device.

    ``normal(seed, shape)`` returns exactly the bytes of
    ``seeded_inputs.pool_normal_bf16(seed, shape)`` without a host->device
    copy per tensor (the window arithmetic mirrors the generator's).
    """

    def __init__(self):
        pool = si._pool()["bf16"]
        self.size = pool.shape[0]
        self.t = dev(pool)

    def normal(self, seed: int, shape):
        n = int(np.prod(shape))
        start = seed % self.size
        if start + n <= self.size:
            out = self.t[start:start + n].clone()
        else:
            out = torch.cat([self.t[start:], self.t[:n - (self.size - start)]])
        return out.view(*shape)


def sample_rows(layout, seed: int, n_random: int = 60):
    """Rows 0, HW-1, HW, R-1 plus seeded random rows of a record."""
    rng = np.random.default_rng(seed)
    fixed = [0, layout.HW - 1, layout.HW, layout.R - 1]
    extra = rng.choice(layout.R, size=n_random, replace=False)
    return np.unique(np.concatenate([fixed, extra]))

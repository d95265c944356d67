"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no arithmetic of the method: it only draws numbers and
converts between float32 and bfloat16 bit patterns.  Both the CUDA path (via
the tests and ``bench.py``) and the fp64 oracle consume what it produces, so a
mismatch between them can never come from the inputs.

Every tensor is identified by a tuple
``(config, session, block, frame, step, tensor)`` that is packed into 64 bits
and mixed with SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) into the key of a Philox-4x64
counter-based generator (Salmon et al., "Parallel random numbers: as easy as
1, 2, 3", SC 2011).  The same tuple always gives the same tensor, in any
order of generation.

Distributions (the workloads the model card describes carry K, V, Q rows of
``heads x head_dim`` bfloat16 values; the synthetic stand-in is):
  * Q, K, V: N(0, 1) float32, rounded to nearest-even bfloat16;
  * K row scale (batch-of-sessions workload): one U(0.5, 2) float32 per token
    row, shared by all heads and channels, applied in float32 before rounding.

Record-sized tensors (``record_inputs``) are windows of one shared pool of
2^25 N(0,1) float32 samples drawn once from Philox with the base seed; the
window start is the tensor's 64-bit key modulo the pool size (wrapping
around).  Each tensor is still N(0,1) and fixed by its tuple, and a
28-block, 41-frame rollout needs seconds instead of minutes to generate.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 0x5EED

# tensor ids of the seed tuple
T_Q, T_K, T_V, T_KSCALE = 0, 1, 2, 3

_MASK64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One SplitMix64 output step applied to ``x`` (64-bit wrap-around)."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def seed_for(config: int, session: int, block: int, frame: int, step: int,
             tensor: int, base: int = BASE_SEED) -> int:
    """64-bit key for one tensor, from its identifying tuple."""
    fields = (config, session, block, frame, step, tensor)
    h = base & _MASK64
    for v in fields:
        h = splitmix64(h ^ (int(v) & _MASK64))
    return h


def _gen(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=seed))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); returns uint16 bits.

    Inputs are finite and far below the float32 maximum (normal samples), so
    the 32-bit sum below cannot carry out of the word and NaN handling is not
    needed.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return bf16_bits_to_f32(b).astype(np.float64)


def normal_bf16(seed: int, shape) -> np.ndarray:
    """N(0,1) float32 samples rounded to bfloat16, as uint16 bits of ``shape``."""
    n = int(np.prod(shape))
    z = _gen(seed).standard_normal(n, dtype=np.float32)
    return f32_to_bf16_bits(z).reshape(shape)


def uniform_f32(seed: int, n: int, lo: float, hi: float) -> np.ndarray:
    """``n`` float32 samples of U(lo, hi)."""
    u = _gen(seed).random(n, dtype=np.float32)
    return (np.float32(lo) + (np.float32(hi) - np.float32(lo)) * u).astype(np.float32)


def scaled_rows_bf16(seed: int, scale_seed: int, rows: int, heads: int, d: int,
                     lo: float = 0.5, hi: float = 2.0) -> np.ndarray:
    """N(0,1) rows, each multiplied in float32 by its own U(lo, hi) scale, then rounded."""
    z = _gen(seed).standard_normal(rows * heads * d, dtype=np.float32).reshape(rows, heads, d)
    s = uniform_f32(scale_seed, rows, lo, hi)
    return f32_to_bf16_bits(z * s[:, None, None])


POOL_LOG2 = 25
_POOL = {}


def _pool():
    if "f32" not in _POOL:
        z = _gen(splitmix64(BASE_SEED ^ 0x9001)).standard_normal(1 << POOL_LOG2, dtype=np.float32)
        _POOL["f32"] = z
        _POOL["bf16"] = f32_to_bf16_bits(z)
    return _POOL


def _window(arr: np.ndarray, seed: int, n: int) -> np.ndarray:
    size = arr.shape[0]
    assert n <= size
    start = seed % size
    if start + n <= size:
        return arr[start:start + n].copy()
    return np.concatenate([arr[start:], arr[:n - (size - start)]])


def pool_normal_bf16(seed: int, shape) -> np.ndarray:
    """N(0,1) bf16 bits of ``shape``: the pool window selected by ``seed``."""
    n = int(np.prod(shape))
    return _window(_pool()["bf16"], seed, n).reshape(shape)


def pool_scaled_rows_bf16(seed: int, scale_seed: int, rows: int, heads: int, d: int,
                          lo: float = 0.5, hi: float = 2.0) -> np.ndarray:
    """Pool window as float32 rows, each times its own U(lo, hi), then rounded to bf16."""
    z = _window(_pool()["f32"], seed, rows * heads * d).reshape(rows, heads, d)
    s = uniform_f32(scale_seed, rows, lo, hi)
    return f32_to_bf16_bits(z * s[:, None, None])


def record_inputs(config: int, session: int, block: int, frame: int, step: int,
                  rows: int, heads: int, d: int, k_row_scale: bool = False):
    """(Q, K, V) bf16 bit arrays ``[rows, heads, d]`` for one write+attend step."""
    shape = (rows, heads, d)
    sq = seed_for(config, session, block, frame, step, T_Q)
    sk = seed_for(config, session, block, frame, step, T_K)
    sv = seed_for(config, session, block, frame, step, T_V)
    q = pool_normal_bf16(sq, shape)
    if k_row_scale:
        ss = seed_for(config, session, block, frame, step, T_KSCALE)
        k = pool_scaled_rows_bf16(sk, ss, rows, heads, d)
    else:
        k = pool_normal_bf16(sk, shape)
    v = pool_normal_bf16(sv, shape)
    return q, k, v

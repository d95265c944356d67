"""Pins for the oracle's FP8 (E4M3) K/V buffer (reading R7 of the oracle).

The page of another system ("commaai/worldmodel-4B", README) says only that
its checkpoint keeps FP8 KV caches; the oracle reads that as OCP FP8 E4M3
codes with one float32 scale per (block, head) for K and for V.  Nothing here
compares the oracle with itself:
  * the codec against PyTorch's own float8_e4m3fn conversions (an
    independent implementation of the same format) and the constants the
    format fixes (largest finite 448, smallest normal 2^-6, smallest
    subnormal 2^-9, the NaN codes);
  * the quantisation against its error bound (half a unit in the last place);
  * the buffer against the bf16 oracle on values every step represents
    exactly, with different scales per block, head and tensor, so that a
    dropped, swapped or misplaced scale fails.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import (E4M3_MAX, E4M3_NAN, FrameMemory, Layout, TINY, attend_memory, dequantize_e4m3,
                    e4m3_decode, e4m3_encode, quantize_e4m3)

torch = pytest.importorskip("torch")


def torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def torch_encode(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_every_code_like_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours, ref = e4m3_decode(codes), torch_decode(codes).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])


def test_format_constants():
    assert e4m3_decode(np.array([0x7E]))[0] == E4M3_MAX == 448.0
    assert e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6          # smallest normal
    assert e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9          # smallest subnormal
    assert e4m3_decode(np.array([0x38]))[0] == 1.0                # exponent field 7 = bias
    assert e4m3_decode(np.array([0x80]))[0] == 0.0 and np.signbit(e4m3_decode(np.array([0x80]))[0])
    finite = e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = finite[np.isfinite(finite)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert len(np.unique(finite)) == 253                          # 254 finite codes, +0 and -0 equal


def test_encode_like_torch_dense_and_ties():
    x = np.linspace(-448.0, 448.0, 1_000_001).astype(np.float32)
    assert np.array_equal(e4m3_encode(x), torch_encode(x))
    # every exact midpoint between neighbouring representable values: ties go to the even code
    vals = np.unique(e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)   # exact in float32
    for m in (mids, -mids):
        got = e4m3_encode(m)
        assert np.array_equal(got, torch_encode(m))
        assert np.all((got & 1) == 0)                             # the even neighbour
    # the subnormal range and a spread of magnitudes, both signs
    rng = np.random.default_rng(11)
    y = np.concatenate([rng.uniform(-2 ** -6, 2 ** -6, 100_000),
                        np.exp2(rng.uniform(-12, 8.8, 100_000)) * rng.choice([-1, 1], 100_000)])
    y = np.clip(y, -447.9, 447.9).astype(np.float32)
    assert np.array_equal(e4m3_encode(y), torch_encode(y))


def test_saturation_and_nan():
    big = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e30, np.inf], np.float32)
    assert np.array_equal(e4m3_encode(big), np.full(7, 0x7E, np.uint8))
    assert np.array_equal(e4m3_encode(-big), np.full(7, 0xFE, np.uint8))
    assert e4m3_encode(np.array([np.nan], np.float32))[0] == E4M3_NAN
    assert e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80


def test_quantisation_error_within_half_ulp():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal(200_000) * 3).astype(np.float32)
    back = e4m3_decode(e4m3_encode(x))
    ax = np.abs(x.astype(np.float64))
    normal = (ax >= 2 ** -6) & (ax <= 448)
    assert np.all(np.abs(back - x)[normal] <= ax[normal] * 2.0 ** -4)
    assert np.all(np.abs(back - x)[ax < 2 ** -6] <= 2.0 ** -10)


def test_quantize_divides_by_the_head_scale_in_float32():
    """Per-head scales: the code of x is e4m3(float32(x) / scale); quantities that are
    code values times their head's scale come back exactly."""
    heads, d = 3, 8
    scale = np.array([0.5, 3.0, 1.0 / 64], np.float32)
    codes = np.random.default_rng(13).integers(0, 0x7F, size=(5, heads, d)).astype(np.uint8)
    codes[codes == 0x7F] = 0x7E
    codes |= np.uint8(0x80) * (np.arange(5 * heads * d).reshape(5, heads, d) % 2).astype(np.uint8)
    vals = e4m3_decode(codes) * scale.astype(np.float64)[None, :, None]
    bits = si.f32_to_bf16_bits(vals.astype(np.float32))
    exact = si.bf16_bits_to_f64(bits) == vals                     # those bf16 holds exactly
    q = quantize_e4m3(bits, scale)
    assert exact.mean() > 0.5
    assert np.array_equal(q[exact], codes[exact])
    np.testing.assert_array_equal(dequantize_e4m3(q, scale)[exact], vals[exact])
    # a scale applied to the wrong head changes codes
    assert not np.array_equal(quantize_e4m3(bits, scale[::-1]), q)


def _representable_record(rng, L, k_scale, v_scale):
    """K, V rows whose values are E4M3 codes times the head's scale and fit bf16 exactly."""
    def one(scale):
        c = rng.integers(0x20, 0x50, size=(L.R, L.heads, L.d)).astype(np.uint8)  # 2^-3 .. 2^3
        c |= (rng.integers(0, 2, size=c.shape) * 0x80).astype(np.uint8)
        v = e4m3_decode(c) * np.asarray(scale, np.float64)[None, :, None]
        b = si.f32_to_bf16_bits(v.astype(np.float32))
        assert np.array_equal(si.bf16_bits_to_f64(b), v)
        return b
    return one(k_scale), one(v_scale)


@pytest.mark.parametrize("L", [TINY, Layout(3, 4, 2, 1, 5, heads=3, d=16)])
def test_fp8_buffer_equals_bf16_buffer_on_representable_values(L):
    blocks = 2
    rng = np.random.default_rng(14)
    # powers of two keep value * scale exact in bf16; different per block, head and tensor
    ks = np.exp2(rng.integers(-3, 3, size=(blocks, L.heads))).astype(np.float32)
    vs = np.exp2(rng.integers(-3, 3, size=(blocks, L.heads))).astype(np.float32)
    assert not np.array_equal(ks, vs)
    m8 = FrameMemory(L, blocks, kv_format="e4m3", k_scale=ks, v_scale=vs)
    m16 = FrameMemory(L, blocks)
    for t in range(2 * L.W + 3):
        m8.advance(t)
        m16.advance(t)
        for b in range(blocks):
            k, v = _representable_record(rng, L, ks[b], vs[b])
            m8.write_record(b, t, k, v)
            m16.write_record(b, t, k, v)
            q = si.normal_bf16(si.seed_for(40, 0, b, t, 0, si.T_Q), (L.R, L.heads, L.d))
            np.testing.assert_allclose(attend_memory(m8, b, q), attend_memory(m16, b, q),
                                       rtol=0, atol=1e-12)
        m8.check_against_records()
        # the stored codes are the quantised records; unfilled rows stay zero
        for b in range(blocks):
            kp8, vp8 = m8.prefix(b)
            kp16, vp16 = m16.prefix(b)
            assert np.array_equal(kp8, kp16) and np.array_equal(vp8, vp16)


def test_fp8_buffer_quantisation_error_against_bf16():
    """Random N(0,1) records: the FP8 buffer's attention differs from the bf16
    buffer's by about the quantisation error (a few percent), not more."""
    L = TINY
    ks = np.full((1, L.heads), 1.0 / 64, np.float32)
    m8 = FrameMemory(L, 1, kv_format="e4m3", k_scale=ks, v_scale=ks)
    m16 = FrameMemory(L, 1)
    for t in range(10):
        m8.advance(t)
        m16.advance(t)
        q, k, v = si.record_inputs(41, 0, 0, t, 0, L.R, L.heads, L.d)
        m8.write_record(0, t, k, v)
        m16.write_record(0, t, k, v)
    a, b = attend_memory(m8, 0, q), attend_memory(m16, 0, q)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-3 < rel < 0.1


def test_fp8_buffer_rejects_the_sink():
    L = TINY
    m8 = FrameMemory(L, 1, kv_format="e4m3", k_scale=np.ones((1, L.heads)), v_scale=np.ones((1, L.heads)))
    m8.sink_theta = np.ones(L.d // 2)
    with pytest.raises(ValueError):
        m8.advance(0)

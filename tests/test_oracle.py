"""Pins for the fp64 oracle: facts the model card prints, closed forms and invariants.

None of these compare the oracle with itself.  Each pin comes from outside it:
a number printed on the page (tests/golden/page_facts.json), a closed form of
softmax attention, or an invariant the page states (what a frame attends to,
no mask).  They are chosen so that a dropped term, a wrong sign or index, a
transposed operand or an off-by-one slot fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import seeded_inputs as si
from oracle import (FrameMemory, Layout, SERVED, SERVED_W16, SCALED, TINY, attend, attend_bits,
                    attend_memory, masked_history_attend, softmax_weights, visible_history_mask)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


@pytest.fixture(scope="module")
def facts():
    with open(GOLDEN) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


# ---------------------------------------------------------------- layout pins

def test_served_constants_match_page(facts):
    gh, gw = facts["served_grid"]
    assert SERVED.HW == gh * gw == facts["raw_tokens_per_frame"]
    assert SERVED.X == facts["summary_tokens_X"]
    assert SERVED.Y == facts["frames_kept_whole_Y"]
    assert SERVED.W == facts["window_W_trained"]
    assert SERVED_W16.W == facts["window_W_served_default"]


def test_served_key_count_is_6528(facts):
    # Z0 + 3 records + 22 summaries of 96 rows
    assert SERVED.C == 1104 + 3 * 1104 + 22 * 96 == facts["keys_in_buffer_served"]
    for t in range(SERVED.W + 1, SERVED.W + 200):
        assert SERVED.end(t) == facts["keys_in_buffer_served"]


def test_full_resolution_span_is_26208(facts):
    # the same span (start image + current frame + W window frames) kept at full resolution
    span_frames = SERVED.W + 2
    assert span_frames * SERVED.HW == facts["keys_full_resolution_same_span"]


def test_end_sequence_served_and_tiny():
    served = [SERVED.end(t) for t in range(8)]
    assert served == [1104, 2208, 3312, 4416, 4512, 4608, 4704, 4800]
    assert SERVED.end(24) == 6432 and SERVED.end(25) == 6528
    tiny = [TINY.end(t) for t in range(12)]
    assert tiny == [28, 56, 84, 112, 116, 120, 124, 128, 128, 128, 128, 128]
    assert TINY.C == 128
    assert SCALED.R == 3856 and SCALED.C == 27200


def test_page_overwrite_example(facts):
    ex = facts["overwrite_example"]
    L = SERVED
    assert L.raw_slot(ex["current_frame"]) == L.raw_slot(ex["raw_slot_of"])
    assert L.sum_slot(ex["summary_of"]) == L.sum_slot(ex["summary_overwrites"])
    assert L.evicted_frame(ex["current_frame"]) == ex["summary_of"]


def _small(layout, heads=1, d=8):
    return Layout(layout.grid_h, layout.grid_w, layout.X, layout.Y, layout.W, heads=heads, d=d)


def test_served_rotation_reproduces_page_example(facts):
    """Roll the served geometry to frame 31 and watch which slots get overwritten."""
    ex = facts["overwrite_example"]
    L = _small(SERVED)
    mem = FrameMemory(L, blocks=1)
    rng = np.random.default_rng(0)
    for t in range(ex["current_frame"] + 1):
        if t == ex["current_frame"]:
            f = L.evicted_frame(t)
            u = L.sum_slot(f)
            assert mem.sum_tag[u] == ex["summary_overwrites"]      # frame 6's summary is there
            s = L.raw_slot(t)
            assert mem.raw_tag[s] == ex["raw_slot_of"]             # frame 28's record is there
        mem.advance(t)
        k = rng.integers(0, 2**16, size=(L.R, 1, 8), dtype=np.uint16)
        mem.write_record(0, t, k, k ^ 0x5555)
    u = L.sum_slot(ex["summary_of"])
    assert mem.sum_tag[u] == ex["summary_of"]
    assert mem.raw_tag[L.raw_slot(ex["current_frame"])] == ex["current_frame"]
    mem.check_against_records()


@pytest.mark.parametrize("layout", [TINY, SERVED, SERVED_W16, SCALED,
                                    Layout(3, 5, 2, 0, 4), Layout(3, 5, 2, 3, 3)])
def test_kept_frames_invariant(layout):
    """RAW holds frames max(1,t-Y)..t; SUM holds frames max(1,t-W)..t-Y-1; end counts them."""
    L = _small(layout)
    mem = FrameMemory(L, blocks=1)
    z = np.zeros((L.R, 1, 8), dtype=np.uint16)
    for t in range(0, 3 * L.W + 10):
        mem.advance(t)
        mem.write_record(0, t, z + t, z + t)
        raw, summ = mem.kept_frames()
        assert raw == list(range(max(1, t - L.Y), t + 1))
        assert summ == list(range(max(1, t - L.W), max(1, t - L.Y)))
        assert L.end(t) == L.R * (1 + len(raw)) + L.X * len(summ)
        assert visible_history_mask(L, t).sum() == L.end(t)
        assert L.end(t) <= L.C


def test_buffer_bytes_match_records_every_call():
    L = TINY
    mem = FrameMemory(L, blocks=2)
    for t in range(12):
        mem.advance(t)
        mem.check_against_records()
        for step in range(4):
            for b in range(2):
                _, k, v = si.record_inputs(1, 0, b, t, step, L.R, L.heads, L.d)
                mem.write_record(b, t, k, v)
                mem.check_against_records()


def test_state_errors():
    mem = FrameMemory(TINY, blocks=1)
    with pytest.raises(ValueError):
        mem.advance(1)
    mem.advance(0)
    z = np.zeros((TINY.R, TINY.heads, TINY.d), np.uint16)
    with pytest.raises(ValueError):
        mem.write_record(0, 1, z, z)


# ------------------------------------------------- attention = masked history

@pytest.mark.parametrize("layout", [TINY, Layout(2, 3, 3, 1, 5, heads=2, d=16),
                                    Layout(2, 2, 2, 0, 3, heads=1, d=8)])
def test_buffer_attention_equals_masked_full_history(layout):
    """Section 'One buffer, no mask': the buffer alone decides visibility."""
    L = layout
    mem = FrameMemory(L, blocks=1)
    hist_k, hist_v = {}, {}
    for t in range(2 * L.W + 2):
        mem.advance(t)
        for step in range(4):                       # three denoising passes + clean rewrite
            q, k, v = si.record_inputs(99, 0, 0, t, step, L.R, L.heads, L.d)
            mem.write_record(0, t, k, v)
            hist_k[t], hist_v[t] = k, v
            o_buf = attend_memory(mem, 0, q)
            o_ref = masked_history_attend(L, hist_k, hist_v, q, t)
            np.testing.assert_allclose(o_buf, o_ref, rtol=0, atol=1e-12)


def test_masked_history_differs_if_mask_is_wrong():
    """Sanity of the pin itself: dropping the summary-only rule changes the answer."""
    L = TINY
    t = 9
    hist_k, hist_v = {}, {}
    for f in range(t + 1):
        _, hist_k[f], hist_v[f] = si.record_inputs(5, 0, 0, f, 0, L.R, L.heads, L.d)
    q, _, _ = si.record_inputs(5, 0, 0, t, 1, L.R, L.heads, L.d)
    good = masked_history_attend(L, hist_k, hist_v, q, t)
    k = np.concatenate([si.bf16_bits_to_f64(hist_k[f]) for f in range(t + 1)])
    v = np.concatenate([si.bf16_bits_to_f64(hist_v[f]) for f in range(t + 1)])
    everything = attend(si.bf16_bits_to_f64(q), k, v)
    assert np.abs(good - everything).max() > 1e-3


# ------------------------------------------------------ softmax closed forms

def test_permutation_invariance():
    rng = np.random.default_rng(1)
    q, k, v = (rng.standard_normal((n, 3, 16)) for n in (7, 50, 50))
    perm = rng.permutation(50)
    np.testing.assert_allclose(attend(q, k, v), attend(q, k[perm], v[perm]), rtol=0, atol=1e-12)


def test_weights_sum_to_one():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((9, 2, 32)) * 3, rng.standard_normal((70, 2, 32)) * 3
    w = softmax_weights(q, k)
    np.testing.assert_allclose(w.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    assert (w >= 0).all()


def test_weights_two_keys_logistic():
    """softmax_weights of two keys: logistic((s0 - s1) / sqrt(d)); pins its scale."""
    d = 64
    q = np.zeros((1, 1, d)); q[0, 0, 3] = 2.0
    k = np.zeros((2, 1, d)); k[0, 0, 3] = 5.0; k[1, 0, 3] = -3.0
    w = softmax_weights(q, k)
    w0 = 1.0 / (1.0 + np.exp(-(2.0 * 5.0 - 2.0 * -3.0) / 8.0))
    np.testing.assert_allclose(w[0, 0], [w0, 1.0 - w0], rtol=0, atol=1e-15)


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((5, 2, 16)), rng.standard_normal((40, 2, 16))
    v = np.ones((40, 2, 16))
    np.testing.assert_allclose(attend(q, k, v), 1.0, rtol=0, atol=1e-12)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(4)
    q, k, v = rng.standard_normal((6, 3, 8)), rng.standard_normal((1, 3, 8)), rng.standard_normal((1, 3, 8))
    o = attend(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-12)


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(5)
    k, v = rng.standard_normal((33, 2, 8)), rng.standard_normal((33, 2, 8))
    q = np.zeros((4, 2, 8))
    o = attend(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), rtol=0, atol=1e-12)


def test_two_keys_logistic_closed_form():
    """With two keys the weight of key 0 is the logistic function of (s0 - s1)/sqrt(d)."""
    d = 16
    q = np.zeros((1, 1, d)); q[0, 0, 0] = 1.0
    k = np.zeros((2, 1, d)); k[0, 0, 0] = 3.0; k[1, 0, 0] = -1.0
    v = np.zeros((2, 1, d)); v[0, 0, :] = 1.0; v[1, 0, :] = -2.0
    w0 = 1.0 / (1.0 + np.exp(-(3.0 - (-1.0)) / 4.0))      # sqrt(16) = 4
    expect = w0 * 1.0 + (1 - w0) * (-2.0)
    np.testing.assert_allclose(attend(q, k, v)[0, 0], expect, rtol=0, atol=1e-14)


def test_one_hot_selection_per_head():
    """Each query of each head picks out a different key: catches transposes and head mix-ups."""
    d, heads, n = 16, 3, 16
    rng = np.random.default_rng(6)
    basis = [rng.permutation(d) for _ in range(heads)]     # each head its own key directions
    k = np.zeros((n, heads, d))
    for h in range(heads):
        for j in range(n):
            k[j, h, basis[h][j]] = 1.0
    v = np.arange(n * heads * d, dtype=np.float64).reshape(n, heads, d)
    lq = 5
    q = np.zeros((lq, heads, d))
    sel = np.zeros((lq, heads), dtype=int)
    for i in range(lq):
        for h in range(heads):
            sel[i, h] = (3 * i + 5 * h + 1) % n
            q[i, h, basis[h][sel[i, h]]] = 400.0   # score 100 after 1/sqrt(16)
    o = attend(q, k, v)
    for i in range(lq):
        for h in range(heads):
            np.testing.assert_allclose(o[i, h], v[sel[i, h], h], rtol=1e-12, atol=1e-9)


def test_attend_bits_widen_exactly():
    bits = si.f32_to_bf16_bits(np.array([1.0, -2.5, 0.15625, 3.0e-3], np.float32))
    back = si.bf16_bits_to_f64(bits)
    assert back[0] == 1.0 and back[1] == -2.5 and back[2] == 0.15625
    assert abs(back[3] - 3.0e-3) <= 3.0e-3 * 2.0 ** -8
    q = bits.reshape(1, 1, 4)
    o = attend_bits(q, q, q)
    np.testing.assert_allclose(o[0, 0], back, rtol=0, atol=1e-15)


# ------------------------------------------------------- generator sanity

def test_generator_is_deterministic_and_normal():
    a = si.normal_bf16(si.seed_for(2, 0, 3, 31, 0, si.T_Q), (1104, 16, 64))
    b = si.normal_bf16(si.seed_for(2, 0, 3, 31, 0, si.T_Q), (1104, 16, 64))
    c = si.normal_bf16(si.seed_for(2, 0, 3, 31, 1, si.T_Q), (1104, 16, 64))
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    x = si.bf16_bits_to_f64(a)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to even (1.0)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)
    out = si.bf16_bits_to_f64(si.f32_to_bf16_bits(x))
    assert out[0] == 1.0 and out[1] == 1.0 + 2.0 ** -6 and out[2] == -1.0


# ---------------------------------------------------- streaming sink (start image keys)

from oracle import rotate_keys_bf16, rotate_pairs_f64, rotation_cos_sin, sink_shift

THETA = np.array([1.0e-4 * 10000.0 ** (-i / 16) for i in range(32)])   # 32 pairs of d = 64
THETA[12:] = 0.0                                                        # 12 temporal pairs


def test_rotation_composes_as_the_page_states():
    """rotation(id + T) = rotation(id) * rotation(T)."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 3, 64))
    th = rng.uniform(0, 2, 32)
    two = rotate_pairs_f64(rotate_pairs_f64(x, th, 7.0), th, 13.0)
    np.testing.assert_allclose(two, rotate_pairs_f64(x, th, 20.0), rtol=0, atol=1e-12)


def test_joint_rotation_keeps_scores_and_only_relative_shift_matters():
    rng = np.random.default_rng(12)
    q, k = rng.standard_normal((4, 64)), rng.standard_normal((9, 64))
    th = rng.uniform(0, 1, 32)
    s0 = q @ k.T
    np.testing.assert_allclose(rotate_pairs_f64(q, th, 5.0) @ rotate_pairs_f64(k, th, 5.0).T, s0,
                               rtol=0, atol=1e-12)
    a = rotate_pairs_f64(q, th, 11.0) @ rotate_pairs_f64(k, th, 4.0).T
    b = rotate_pairs_f64(q, th, 7.0) @ k.T
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    # and it is not the identity: a shift of the keys alone changes the scores
    assert np.abs(q @ rotate_pairs_f64(k, th, 3.0).T - s0).max() > 1e-3


def test_rotation_keeps_pair_norms_and_quarter_turn():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((6, 64))
    th = rng.uniform(0, 3, 32)
    y = rotate_pairs_f64(x, th, 2.0)
    np.testing.assert_allclose(x[:, 0::2] ** 2 + x[:, 1::2] ** 2, y[:, 0::2] ** 2 + y[:, 1::2] ** 2,
                               rtol=1e-12)
    q = rotate_pairs_f64(x, np.full(32, np.pi / 2), 1.0)           # (a, b) -> (-b, a)
    np.testing.assert_allclose(q[:, 0::2], -x[:, 1::2], atol=1e-12)
    np.testing.assert_allclose(q[:, 1::2], x[:, 0::2], atol=1e-12)


def test_stored_rotation_identity_cases_and_rounding():
    k = si.normal_bf16(99, (7, 2, 64))
    assert np.array_equal(rotate_keys_bf16(k, THETA, 0), k)          # shift 0: cos 1, sin 0
    out = rotate_keys_bf16(k, THETA, 9)
    assert np.array_equal(out[..., 24:], k[..., 24:])                 # non-temporal pairs untouched
    exact = rotate_pairs_f64(si.bf16_bits_to_f64(k), THETA, 9.0)
    got = si.bf16_bits_to_f64(out)
    assert np.all(np.abs(got - exact) <= 2.0 ** -8 * np.abs(exact) + 1e-30 + 2.0 ** -120)
    c, s = rotation_cos_sin(THETA, 9)
    assert c.dtype == np.float32 and np.all(c[12:] == 1) and np.all(s[12:] == 0)


@pytest.mark.parametrize("layout", [SERVED, TINY, SERVED_W16])
def test_sink_schedule_keeps_gap_between_one_and_four(layout):
    """Rotations fire when the gap hits the trigger (5) and leave a gap of 1."""
    z0, rotations = 0, []
    for t in range(0, 200):
        shift = sink_shift(layout, t, z0)
        oldest = max(1, t - layout.W) if t >= 1 else None
        if shift:
            assert oldest - z0 == 5 and shift == 4
            rotations.append(t)
            z0 += shift
        if t >= 1:
            assert 1 <= oldest - z0 <= 4
    first = layout.W + 5
    assert rotations[0] == first and all(b - a == 4 for a, b in zip(rotations, rotations[1:]))


def test_memory_rotates_only_start_image_keys():
    L = Layout(2, 3, 2, 1, 3, heads=2, d=64)
    mem = FrameMemory(L, blocks=2)
    mem.sink_theta = THETA
    prev_pos = 0
    for t in range(12):
        before = mem.K.copy(), mem.V.copy()
        mem.advance(t)
        shift_happened = mem.z0_pos != prev_pos
        if shift_happened:
            assert not np.array_equal(mem.K[:, :L.R], before[0][:, :L.R])
        else:
            assert np.array_equal(mem.K[:, :L.R], before[0][:, :L.R])
        assert np.array_equal(mem.V[:, :L.R], before[1][:, :L.R])        # values untouched
        prev_pos = mem.z0_pos
        for b in range(2):
            _, k, v = si.record_inputs(31, 0, b, t, 0, L.R, L.heads, L.d)
            mem.write_record(b, t, k, v)
        mem.check_against_records()
    assert mem.z0_pos == 4              # one rotation, at t = W + 5 = 8 (the next would be t = 12)

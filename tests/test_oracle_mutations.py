"""The oracle's pins catch plausible mistakes: each test plants one mistake in
the oracle (on the CPU, through monkeypatching) and checks that at least one
pin fails.  The pins here are the same kinds as in test_oracle.py: numbers the
model card prints, closed forms of softmax attention, and the page's
visibility rule checked by brute force."""
import json
import os

import numpy as np
import pytest

import seeded_inputs as si
import oracle.kvmemory as kvm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


def pin_page_example():
    L = kvm.SERVED
    assert L.raw_slot(31) == L.raw_slot(28) and L.sum_slot(28) == L.sum_slot(6)
    assert L.evicted_frame(31) == 28


def pin_key_counts():
    f = _facts()
    L = kvm.SERVED
    assert [L.end(t) for t in range(5)] == [1104, 2208, 3312, 4416, 4512]
    assert L.end(31) == f["keys_in_buffer_served"] == 6528


def pin_rollout_against_history():
    """Tiny memory, frames 0..11: kept frames, record bytes, and buffer attention
    against masked full-history attention (the page's visibility rule)."""
    L = kvm.TINY
    mem = kvm.FrameMemory(L, 1)
    hk, hv = [], []
    for t in range(12):
        mem.advance(t)
        q, k, v = si.record_inputs(7, 0, 0, t, 0, L.R, L.heads, L.d)
        mem.write_record(0, t, k, v)
        hk.append(k)
        hv.append(v)
        mem.check_against_records()
        raw, summ = mem.kept_frames()
        assert raw == [f for f in range(max(1, t - L.Y), t + 1)]
        assert summ == [f for f in range(max(1, t - L.W), t - L.Y)]
        a = kvm.attend_memory(mem, 0, q)
        b = kvm.masked_history_attend(L, hk, hv, q, t)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def pin_softmax_closed_forms():
    d = 16
    q = np.zeros((1, 1, d)); q[0, 0, 0] = 1.0
    k = np.zeros((2, 1, d)); k[0, 0, 0] = 3.0; k[1, 0, 0] = -1.0
    v = np.zeros((2, 1, d)); v[0, 0, :] = 1.0; v[1, 0, :] = -2.0
    w0 = 1.0 / (1.0 + np.exp(-4.0 / 4.0))
    np.testing.assert_allclose(kvm.attend(q, k, v)[0, 0], w0 - 2.0 * (1 - w0), rtol=0, atol=1e-14)
    rng = np.random.default_rng(3)
    qq, kk = rng.standard_normal((5, 2, 16)), rng.standard_normal((40, 2, 16))
    np.testing.assert_allclose(kvm.attend(qq, kk, np.ones((40, 2, 16))), 1.0, rtol=0, atol=1e-12)


def pin_one_hot_heads():
    d, heads, n = 16, 3, 16
    rng = np.random.default_rng(6)
    basis = [rng.permutation(d) for _ in range(heads)]
    k = np.zeros((n, heads, d))
    for h in range(heads):
        for j in range(n):
            k[j, h, basis[h][j]] = 1.0
    v = np.arange(n * heads * d, dtype=np.float64).reshape(n, heads, d)
    q = np.zeros((2, heads, d))
    for h in range(heads):
        q[0, h, basis[h][h + 1]] = 400.0
        q[1, h, basis[h][2 * h + 3]] = 400.0
    o = kvm.attend(q, k, v)
    for h in range(heads):
        np.testing.assert_allclose(o[0, h], v[h + 1, h], rtol=1e-12, atol=1e-9)
        np.testing.assert_allclose(o[1, h], v[2 * h + 3, h], rtol=1e-12, atol=1e-9)


def pin_fp8_exact_values():
    """E4M3 buffer on values that are code values times the head's scale equals the bf16 buffer."""
    L = kvm.TINY
    ks = np.array([[0.5, 2.0]], np.float32)
    vs = np.array([[4.0, 0.25]], np.float32)
    m8 = kvm.FrameMemory(L, 1, kv_format="e4m3", k_scale=ks, v_scale=vs)
    m16 = kvm.FrameMemory(L, 1)
    rng = np.random.default_rng(9)
    for t in range(3):
        m8.advance(t)
        m16.advance(t)
        rec = []
        for sc in (ks[0], vs[0]):
            c = rng.integers(0x20, 0x50, size=(L.R, L.heads, L.d)).astype(np.uint8)
            rec.append(si.f32_to_bf16_bits((kvm.e4m3_decode(c) * sc.astype(np.float64)[None, :, None])
                                           .astype(np.float32)))
        m8.write_record(0, t, *rec)
        m16.write_record(0, t, *rec)
        q = si.normal_bf16(si.seed_for(8, 0, 0, t, 0, si.T_Q), (L.R, L.heads, L.d))
        np.testing.assert_allclose(kvm.attend_memory(m8, 0, q), kvm.attend_memory(m16, 0, q),
                                   rtol=0, atol=1e-12)


PINS = [pin_page_example, pin_key_counts, pin_rollout_against_history, pin_softmax_closed_forms,
        pin_one_hot_heads, pin_fp8_exact_values]


def failing_pins():
    out = []
    for p in PINS:
        try:
            p()
        except (AssertionError, ValueError, IndexError, KeyError):
            out.append(p.__name__)
    return out


def test_pins_pass_on_the_oracle_as_written():
    assert failing_pins() == []


def _attend_variant(kind):
    orig = kvm.attend

    def mutated(q, k, v, scale=None):
        q = np.asarray(q, np.float64)
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        d = q.shape[-1]
        sc = (1.0 / d if kind == "scale" else 1.0 / np.sqrt(d)) if scale is None else scale
        out = np.empty(q.shape)
        for h in range(q.shape[1]):
            kh = k[:, 0, :] if kind == "head" else k[:, h, :]
            s = (q[:, h, :] @ kh.T) * sc
            p = np.exp(s - s.max(axis=1, keepdims=True))
            out[:, h, :] = p @ v[:, h, :] if kind == "norm" else (p @ v[:, h, :]) / p.sum(axis=1, keepdims=True)
        return out
    return orig, mutated


def _evict_from_slot_start(self, t):
    """advance() with the summary rows read from the start of the RAW slot."""
    L = self.layout
    f = L.evicted_frame(t)
    if f is not None and L.W > L.Y:
        r0, r1 = L.raw_rows(L.raw_slot(f))
        d0, d1 = L.sum_rows(L.sum_slot(f))
        self.K[:, d0:d1] = self.K[:, r0:r0 + L.X]
        self.V[:, d0:d1] = self.V[:, r0:r0 + L.X]
        self.sum_tag[L.sum_slot(f)] = f
    self.t = t
    self.written = set()


MUTATIONS = {
    "raw slot base t mod (Y+1)": lambda mp: mp.setattr(kvm.Layout, "raw_slot", lambda self, t: t % (self.Y + 1)),
    "sum slot base f mod (W-Y)": lambda mp: mp.setattr(kvm.Layout, "sum_slot", lambda self, f: f % (self.W - self.Y)),
    "evicted frame t-Y": lambda mp: mp.setattr(kvm.Layout, "evicted_frame",
                                               lambda self, t: (t - self.Y) if t - self.Y >= 1 else None),
    "end one row short": lambda mp: mp.setattr(kvm.Layout, "end", lambda self, t: self.R * (1 + min(t, self.Y + 1))
                                               + self.X * min(max(t - self.Y - 1, 0), self.W - self.Y) - 1),
    "eviction source rows": lambda mp: mp.setattr(kvm.FrameMemory, "advance", _evict_from_slot_start),
    "scale 1/d": lambda mp: mp.setattr(kvm, "attend", _attend_variant("scale")[1]),
    "no normalisation": lambda mp: mp.setattr(kvm, "attend", _attend_variant("norm")[1]),
    "K head index": lambda mp: mp.setattr(kvm, "attend", _attend_variant("head")[1]),
    "fp8 scale multiplies": lambda mp: mp.setattr(
        kvm, "quantize_e4m3", lambda bits, scale: kvm.e4m3_encode(
            si.bf16_bits_to_f32(bits) * np.asarray(scale, np.float32).reshape(1, -1, 1))),
    "fp8 decode ignores scale": lambda mp: mp.setattr(kvm, "dequantize_e4m3", lambda c, s: kvm.e4m3_decode(c)),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_each_planted_mistake_fails_a_pin(name, monkeypatch):
    MUTATIONS[name](monkeypatch)
    assert failing_pins(), f"no pin caught: {name}"

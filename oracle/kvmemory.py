"""fp64 CPU oracle for the Summaryformer frame memory and the attention that reads it.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package;
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` (plus its ``--impl reference`` arm) may call it.  It shares no
code with the CUDA library: the only module both sides use is
``seeded_inputs``, which draws the inputs and holds none of the method.

Source: the model card "GTA world model: weights and inference code"
(lucidml/gta).  Section names below refer to that page.

What the page fixes, restated:
  * "A frame is a record": record(t) = the frame's H*W raw tokens followed by
    its X summary tokens (raw first).
  * "What a frame attends to": the keys visible to frame t's tokens are its
    own record, the full records of frames t-Y..t-1, only the X summary rows
    of the frames older than those but still inside the window W, and the
    start image (frame 0) in full, which is never evicted.
  * "One buffer, no mask": one preallocated K/V buffer per block with regions
    | Z0: record(0) | RAW: (Y+1) rotating records | SUM: (W-Y) x X rotating
    summary rows |; reading is buffer[0:end], the filled prefix, one dense
    unmasked attention.  A frame that drops out of the raw window keeps only
    its X summary rows (K and V), moved from RAW into SUM; the next frame then
    reuses its RAW slot.  Served-shape example: frame 31 takes frame 28's RAW
    slot and frame 28's summary takes the SUM slot of frame 6's.  Served
    numbers: 6,528 buffered keys, against 26,208 for the same span at full
    resolution.
  * "The rest of the model", Sampling: a frame is produced by three
    denoising passes, after which a clean pass writes the frame's final
    record over the same slot.

Readings where the page leaves a step open (each is also listed in the design
notes of the repository):
  R1 slot base: frame t >= 1 goes to RAW slot (t-1) mod (Y+1); the summary of
     frame f >= 1 goes to SUM slot (f-1) mod (W-Y).  Both agree with the worked
     example (31 = 28 mod 3, 28 = 6 mod 22); only this base keeps the filled
     part of the buffer a contiguous prefix while the buffer fills.
  R2 eviction happens at the start of frame t (advance), before any write of
     frame t, and moves frame t-Y-1 (t >= Y+2) in every block.
  R3 frame 0 is written into Z0 and attends to [0:R) (itself).
  R4 the frame being generated is in its own read set ("itself").
  R5 attention uses scale 1/sqrt(d) and an ordinary softmax (the page names
     the attention kernels, FlexAttention and flash_attn_with_kvcache, whose
     default is this scale).
  R6 (section "Running for a long time: the start image follows the window")
     the oldest frame in memory while frame t is generated is max(1, t - W);
     the gap is that frame's id minus the start image's temporal position,
     which starts at 0.  When the gap reaches 5 at the start of a frame, the
     start image's keys (Z0 rows of K, every block) are rotated forward by
     gap - 1 frames, in place; values are untouched.  The rotation acts on
     adjacent dimension pairs (2i, 2i+1) of each head as on complex numbers,
     pair i turning by theta_i * shift (theta_i = 0: not a temporal pair),
     computed in float32 as a' = a*c - b*s, b' = a*s + b*c (each product and
     sum rounded to float32, c and s the float32 cosine and sine) and rounded
     to bfloat16: the page gives neither the frequencies nor the precision,
     so the frequencies are a parameter and the precision is the kernel's.
  R7 (FP8 buffer; the page of another system, "commaai/worldmodel-4B", README,
     says only that its checkpoint keeps FP8 KV caches) the buffer may store
     K and V as OCP FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3
     mantissa bits, subnormals, no infinities, S.1111.111 = NaN, largest
     finite value 448).  Each (block, head) has one float32 scale for K and
     one for V, fixed when the buffer is created.  A stored code is the
     float32 quotient x / scale rounded to nearest, ties to even, and
     saturated to +-448 (NaN stays NaN); a code means code_value * scale.
     Eviction moves codes.  Attention is the same softmax over the dequantised
     values.  The streaming sink is not defined for this format.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import seeded_inputs as si


# ---------------------------------------------------------------------------
# Layout: section "One buffer, no mask" plus readings R1/R2
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Layout:
    """Geometry of one block's buffer; rows are token rows of ``heads x d``."""
    grid_h: int
    grid_w: int
    X: int          # summary tokens per record
    Y: int          # frames kept whole besides the current one
    W: int          # memory window in frames
    heads: int = 1
    d: int = 64

    @property
    def HW(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def R(self) -> int:
        """Rows of one record: H*W raw tokens then X summary tokens."""
        return self.HW + self.X

    @property
    def n_raw_slots(self) -> int:
        return self.Y + 1

    @property
    def n_sum_slots(self) -> int:
        return self.W - self.Y

    @property
    def C(self) -> int:
        """Buffer capacity in rows: Z0 + (Y+1) records + (W-Y)*X summary rows."""
        return self.R * (self.Y + 2) + self.X * (self.W - self.Y)

    # region starts --------------------------------------------------------
    def z0_rows(self):
        return 0, self.R

    def raw_rows(self, s: int):
        assert 0 <= s <= self.Y
        return self.R * (1 + s), self.R * (2 + s)

    def sum_rows(self, u: int):
        assert 0 <= u < self.W - self.Y
        base = self.R * (self.Y + 2)
        return base + self.X * u, base + self.X * (u + 1)

    # slot arithmetic ------------------------------------------------------
    def raw_slot(self, t: int) -> int:
        """RAW slot of frame t >= 1 (reading R1)."""
        assert t >= 1
        return (t - 1) % (self.Y + 1)

    def sum_slot(self, f: int) -> int:
        """SUM slot of frame f >= 1's summary (reading R1)."""
        assert f >= 1 and self.W > self.Y
        return (f - 1) % (self.W - self.Y)

    def evicted_frame(self, t: int):
        """Frame whose summary moves RAW -> SUM at the start of frame t, or None."""
        f = t - self.Y - 1
        return f if f >= 1 else None

    def record_rows(self, t: int):
        """Rows the record of frame t occupies."""
        return self.z0_rows() if t == 0 else self.raw_rows(self.raw_slot(t))

    def end(self, t: int) -> int:
        """Filled prefix while frame t is generated, counted from the regions.

        Z0 always; RAW holds frames 1..t up to Y+1 of them; SUM holds the
        summaries of frames 1..t-Y-1 up to W-Y of them.
        """
        n_raw = min(t, self.Y + 1)
        n_sum = min(max(t - self.Y - 1, 0), self.W - self.Y)
        return self.R * (1 + n_raw) + self.X * n_sum


# ---------------------------------------------------------------------------
# Streaming sink: section "Running for a long time" (reading R6)
# ---------------------------------------------------------------------------

def rotation_cos_sin(theta, shift: int):
    """float32 cosine and sine of theta_i * shift (double precision, then rounded)."""
    ang = np.asarray(theta, dtype=np.float64) * float(shift)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rotate_pairs_f64(x: np.ndarray, theta, shift: float) -> np.ndarray:
    """Exact-arithmetic reference: adjacent pairs of the last axis turned by theta_i * shift."""
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(theta, dtype=np.float64) * shift
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * np.cos(ang) - b * np.sin(ang)
    out[..., 1::2] = a * np.sin(ang) + b * np.cos(ang)
    return out


def rotate_keys_bf16(k_bits: np.ndarray, theta, shift: int) -> np.ndarray:
    """The in-place key rotation as stored: float32 arithmetic in a fixed order, then bf16.

    Pairs with theta_i == 0 are left untouched (bit for bit).
    """
    c, s = rotation_cos_sin(theta, shift)
    x = si.bf16_bits_to_f32(k_bits)
    a, b = x[..., 0::2], x[..., 1::2]
    na = np.subtract(np.multiply(a, c, dtype=np.float32), np.multiply(b, s, dtype=np.float32),
                     dtype=np.float32)
    nb = np.add(np.multiply(a, s, dtype=np.float32), np.multiply(b, c, dtype=np.float32),
                dtype=np.float32)
    out = np.array(k_bits, dtype=np.uint16, copy=True)
    rot = np.asarray(theta) != 0
    ra, rb = si.f32_to_bf16_bits(na), si.f32_to_bf16_bits(nb)
    out[..., 0::2] = np.where(rot, ra, out[..., 0::2])
    out[..., 1::2] = np.where(rot, rb, out[..., 1::2])
    return out


def sink_shift(layout: "Layout", t: int, z0_pos: int, trigger: int = 5, target: int = 1) -> int:
    """Frames to move the start image forward at the start of frame t (0: no rotation)."""
    if t < 1:
        return 0
    oldest = max(1, t - layout.W)
    gap = oldest - z0_pos
    return gap - target if gap >= trigger else 0


# ---------------------------------------------------------------------------
# FP8 E4M3 codes (reading R7)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0          # 1.75 * 2^8, the largest finite E4M3 value
E4M3_NAN = 0x7F           # the code a NaN input gets


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code as float64: sign, 4-bit exponent (bias 7) and
    3-bit mantissa; exponent field 0 holds the subnormals m/8 * 2^-6; the
    all-ones exponent with all-ones mantissa is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * mag
    return np.where((e == 15) & ((c & 7) == 7), np.nan, val)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code of each value: nearest representable value, ties to the even
    mantissa; magnitudes of 448 and above saturate to 448; NaN -> E4M3_NAN."""
    v = np.asarray(x, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    # subnormal range, a < 2^-6: units of 2^-9 (the value 8 * 2^-9 is the
    # smallest normal, code 0x08, which the same formula produces)
    sub = np.rint(np.where(a < 2.0 ** -6, a, 0.0) / 2.0 ** -9)
    # normal range: a = (1 + f) * 2^e with f in [0, 1)
    mant, ex = np.frexp(np.where((a > 0) & (a < E4M3_MAX), a, 1.0))   # a = mant * 2^ex
    e = ex - 1
    m = np.rint((mant * 2.0 - 1.0) * 8.0)               # 3-bit mantissa, half to even
    carry = m == 8
    e = np.where(carry, e + 1, e)
    m = np.where(carry, 0, m)
    normal = ((e + 7) << 3) | m.astype(np.int64)
    code = np.where(a < 2.0 ** -6, sub.astype(np.int64), normal)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = code | np.where(neg, 0x80, 0)
    code = np.where(nan, E4M3_NAN, code)
    return code.astype(np.uint8)


def quantize_e4m3(bits: np.ndarray, scale) -> np.ndarray:
    """bf16 bit patterns ``[rows, heads, d]`` -> E4M3 codes with one float32
    scale per head: code = e4m3(float32(x) / scale), the division in float32."""
    x = si.bf16_bits_to_f32(bits)
    s = np.asarray(scale, dtype=np.float32).reshape(1, -1, 1)
    return e4m3_encode(np.divide(x, s, dtype=np.float32))


def dequantize_e4m3(codes: np.ndarray, scale) -> np.ndarray:
    """E4M3 codes ``[rows, heads, d]`` -> code value * scale (per head), float64 (exact)."""
    s = np.asarray(scale, dtype=np.float32).astype(np.float64).reshape(1, -1, 1)
    return e4m3_decode(codes) * s


# ---------------------------------------------------------------------------
# The memory: a host mirror updated by the page's rules
# ---------------------------------------------------------------------------

@dataclass
class FrameMemory:
    """Mirror of all blocks' K/V buffers (bf16 bit patterns) of one session.

    Besides the mirror it keeps, independently, the latest record written for
    every (block, frame) and a frame-id tag per slot, so that every byte of
    the mirror can be checked against the record it logically came from.
    """
    layout: Layout
    blocks: int
    track_records: bool = True   # keep every record for check_against_records (small runs)
    t: int = -1
    K: np.ndarray = field(init=False)
    V: np.ndarray = field(init=False)
    records: dict = field(init=False)       # (block, frame) -> (K rows, V rows)
    sink_theta: object = None                # per-pair temporal frequencies (None: no sink)
    z0_pos: int = 0                          # temporal position of the start image
    raw_tag: list = field(init=False)        # frame id held by each RAW slot
    sum_tag: list = field(init=False)        # frame id whose summary each SUM slot holds
    written: set = field(init=False)         # blocks written at the current t
    kv_format: str = "bf16"                  # "bf16" bit patterns or "e4m3" codes (R7)
    k_scale: object = None                   # e4m3: float32 [blocks, heads]
    v_scale: object = None

    def __post_init__(self):
        L = self.layout
        shape = (self.blocks, L.C, L.heads, L.d)
        if self.kv_format not in ("bf16", "e4m3"):
            raise ValueError(self.kv_format)
        store = np.uint8 if self.kv_format == "e4m3" else np.uint16
        if self.kv_format == "e4m3":
            self.k_scale = np.asarray(self.k_scale, np.float32).reshape(self.blocks, L.heads)
            self.v_scale = np.asarray(self.v_scale, np.float32).reshape(self.blocks, L.heads)
        self.K = np.zeros(shape, dtype=store)
        self.V = np.zeros(shape, dtype=store)
        self.records = {}
        self.raw_tag = [None] * (L.Y + 1)
        self.sum_tag = [None] * max(L.W - L.Y, 0)
        self.written = set()

    def end(self) -> int:
        return self.layout.end(self.t)

    def advance(self, t: int) -> None:
        """Start frame t; move frame t-Y-1's X summary rows RAW -> SUM in every block."""
        if t != self.t + 1:
            raise ValueError(f"advance({t}) after frame {self.t}")
        L = self.layout
        f = L.evicted_frame(t)
        if f is not None and L.W > L.Y:
            s = L.raw_slot(f)
            if self.raw_tag[s] != f:
                raise ValueError(f"frame {f} leaves the raw window but was never written")
            r0, r1 = L.raw_rows(s)
            src0 = r0 + L.HW                       # summary tokens follow the raw ones
            u = L.sum_slot(f)
            d0, d1 = L.sum_rows(u)
            assert d1 - d0 == r1 - src0 == L.X
            self.K[:, d0:d1] = self.K[:, src0:r1]
            self.V[:, d0:d1] = self.V[:, src0:r1]
            self.sum_tag[u] = f
        if self.sink_theta is not None:
            if self.kv_format != "bf16":
                raise ValueError("the streaming sink is defined for bf16 buffers only")
            shift = sink_shift(L, t, self.z0_pos)
            if shift:
                self.K[:, :L.R] = rotate_keys_bf16(self.K[:, :L.R], self.sink_theta, shift)
                if self.track_records:
                    for (b, f), (kf, vf) in list(self.records.items()):
                        if f == 0:
                            self.records[(b, 0)] = (self.K[b, :L.R].copy(), vf)
                self.z0_pos += shift
        self.t = t
        self.written = set()

    def write_record(self, block: int, t: int, k: np.ndarray, v: np.ndarray) -> None:
        """Store frame t's record (``[R, heads, d]`` bf16 bits) in Z0 or its RAW slot."""
        L = self.layout
        if t != self.t:
            raise ValueError(f"write_record at t={t}, current frame {self.t}")
        assert k.shape == v.shape == (L.R, L.heads, L.d)
        if self.kv_format == "e4m3":
            k = quantize_e4m3(k, self.k_scale[block])
            v = quantize_e4m3(v, self.v_scale[block])
        r0, r1 = L.record_rows(t)
        self.K[block, r0:r1] = k
        self.V[block, r0:r1] = v
        if t >= 1:
            self.raw_tag[L.raw_slot(t)] = t
        if self.track_records:
            self.records[(block, t)] = (k.copy(), v.copy())
        self.written.add(block)

    def prefix(self, block: int):
        """K, V of buffer[0:end] as fp64 arrays ``[end, heads, d]`` (dequantised for e4m3)."""
        e = self.end()
        if self.kv_format == "e4m3":
            return (dequantize_e4m3(self.K[block, :e], self.k_scale[block]),
                    dequantize_e4m3(self.V[block, :e], self.v_scale[block]))
        return si.bf16_bits_to_f64(self.K[block, :e]), si.bf16_bits_to_f64(self.V[block, :e])

    def check_against_records(self) -> None:
        """Every filled row equals the row it came from; unfilled rows are zero."""
        assert self.track_records, "records are not kept for this memory"
        L = self.layout
        t = self.t
        for b in range(self.blocks):
            if (b, 0) in self.records:
                k0, v0 = self.records[(b, 0)]
                assert np.array_equal(self.K[b, :L.R], k0) and np.array_equal(self.V[b, :L.R], v0)
            for s, f in enumerate(self.raw_tag):
                if f is None or (b, f) not in self.records:
                    continue
                kf, vf = self.records[(b, f)]
                r0, r1 = L.raw_rows(s)
                assert np.array_equal(self.K[b, r0:r1], kf) and np.array_equal(self.V[b, r0:r1], vf)
            for u, f in enumerate(self.sum_tag):
                if f is None:
                    continue
                kf, vf = self.records[(b, f)]
                d0, d1 = L.sum_rows(u)
                assert np.array_equal(self.K[b, d0:d1], kf[L.HW:])
                assert np.array_equal(self.V[b, d0:d1], vf[L.HW:])
            e = L.end(t)
            assert not self.K[b, e:].any() and not self.V[b, e:].any()

    def kept_frames(self):
        """(frames held whole in RAW, frames held as summaries in SUM), sorted."""
        raw = sorted(f for f in self.raw_tag if f is not None)
        summ = sorted(f for f in self.sum_tag if f is not None)
        return raw, summ


# ---------------------------------------------------------------------------
# Attention: section "One buffer, no mask" (one dense unmasked read of the prefix)
# ---------------------------------------------------------------------------

def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None) -> np.ndarray:
    """O[i,h] = sum_j softmax_j(q[i,h].k[j,h] * scale) v[j,h], all keys j, fp64.

    ``q``: [Lq, heads, d]; ``k``, ``v``: [Lk, heads, d]; any real dtype (widened
    to fp64).  Returns fp64 ``[Lq, heads, d]``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty(q.shape, dtype=np.float64)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) * scale          # [Lq, Lk]
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        out[:, h, :] = (p @ v[:, h, :]) / p.sum(axis=1, keepdims=True)
    return out


def softmax_weights(q: np.ndarray, k: np.ndarray, scale: float | None = None) -> np.ndarray:
    """The attention weights p/sum(p) as fp64 ``[heads, Lq, Lk]`` (for normalisation pins)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    w = np.empty((q.shape[1], q.shape[0], k.shape[0]))
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        w[h] = p / p.sum(axis=1, keepdims=True)
    return w


def attend_bits(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                scale: float | None = None) -> np.ndarray:
    """``attend`` on bf16 bit patterns (exact widening first)."""
    return attend(si.bf16_bits_to_f64(q_bits), si.bf16_bits_to_f64(k_bits),
                  si.bf16_bits_to_f64(v_bits), scale)


def attend_memory(mem: FrameMemory, block: int, q_bits: np.ndarray, rows=None,
                  scale: float | None = None) -> np.ndarray:
    """Frame t's queries of ``block`` against buffer[0:end]; optionally a subset of query rows."""
    k, v = mem.prefix(block)
    q = si.bf16_bits_to_f64(q_bits)
    if rows is not None:
        q = q[np.asarray(rows)]
    return attend(q, k, v, scale)


# ---------------------------------------------------------------------------
# Brute force: masked attention over the full, unrotated history
# (section "What a frame attends to", items 1-4)
# ---------------------------------------------------------------------------

def visible_history_mask(layout: Layout, t: int) -> np.ndarray:
    """Boolean mask over the concatenation record(0) ++ record(1) ++ ... ++ record(t).

    Kept: frame 0 whole; frames t-Y .. t whole; the X summary rows of frames
    t-W .. t-Y-1 (frames >= 1).  Everything else is masked out.
    """
    L = layout
    keep = []
    for f in range(t + 1):
        whole = f == 0 or f >= t - L.Y
        summary_only = (not whole) and f >= max(t - L.W, 1)
        row = np.zeros(L.R, dtype=bool)
        if whole:
            row[:] = True
        elif summary_only:
            row[L.HW:] = True
        keep.append(row)
    return np.concatenate(keep)


def masked_history_attend(layout: Layout, history_k: list, history_v: list, q_bits: np.ndarray,
                          t: int, scale: float | None = None) -> np.ndarray:
    """Attention of frame t's queries over the full history with the visibility mask.

    ``history_k[f]``/``history_v[f]``: the latest record written for frame f
    (bf16 bits ``[R, heads, d]``), f = 0..t.
    """
    k = np.concatenate([si.bf16_bits_to_f64(history_k[f]) for f in range(t + 1)])
    v = np.concatenate([si.bf16_bits_to_f64(history_v[f]) for f in range(t + 1)])
    mask = visible_history_mask(layout, t)
    return attend(si.bf16_bits_to_f64(q_bits), k[mask], v[mask], scale)


# ---------------------------------------------------------------------------
# Named workloads (shapes from the model card's served numbers plus synthetic variants)
# ---------------------------------------------------------------------------

TINY = Layout(grid_h=4, grid_w=6, X=4, Y=2, W=6, heads=2, d=64)
SERVED = Layout(grid_h=24, grid_w=42, X=96, Y=2, W=24, heads=16, d=64)
SERVED_W16 = Layout(grid_h=24, grid_w=42, X=96, Y=2, W=16, heads=16, d=64)
SCALED = Layout(grid_h=45, grid_w=80, X=256, Y=2, W=48, heads=24, d=128)

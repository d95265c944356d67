"""ctypes binding of ``libwmkv.so`` (the C ABI declared in ``include/wmkv.h``).

Argument marshalling only: every step of the frame memory and its attention
runs in the library's CUDA kernels.  Tensors are passed as device pointers
(``tensor.data_ptr()``); PyTorch is used by callers for device memory and
streams.  There is no fallback: if the library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwmkv.so")

WM_OK = 0
WM_ERR_INVALID_ARG = -1
WM_ERR_STATE = -2
WM_ERR_UNSUPPORTED = -3
WM_ERR_OOM = -4
WM_ERR_CUDA = -5
WM_ERR_TIMEOUT = -6

_c_int, _c_i64, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p

# name -> (restype, argtypes), in the order of include/wmkv.h
SIGNATURES = {
    "wm_kvbuf_create": (_c_int, [ctypes.POINTER(_vp), _c_int, _c_int, _c_int, _c_int, _c_int,
                                 _c_int, _c_int, _c_int]),
    "wm_kvbuf_create_fp8": (_c_int, [ctypes.POINTER(_vp), _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_int, _c_int, _c_int, ctypes.POINTER(ctypes.c_float),
                                     ctypes.POINTER(ctypes.c_float)]),
    "wm_kv_format": (_c_int, [_vp]),
    "wm_kvbuf_destroy": (_c_int, [_vp]),
    "wm_advance": (_c_int, [_vp, _c_i64, _vp]),
    "wm_write_record": (_c_int, [_vp, _c_int, _c_i64, _vp, _vp, _vp]),
    "wm_attend": (_c_int, [_vp, _c_int, _vp, _vp, _vp]),
    "wm_write_attend": (_c_int, [_vp, _c_int, _c_i64, _vp, _vp, _vp, _vp, _vp]),
    "wm_set_sink": (_c_int, [_vp, ctypes.POINTER(ctypes.c_float), _c_int, _c_int, _c_int]),
    "wm_sink_position": (_c_i64, [_vp]),
    "wm_sink_cos_sin": (_c_int, [_vp, _c_i64, ctypes.POINTER(ctypes.c_float),
                                 ctypes.POINTER(ctypes.c_float)]),
    "wm_end": (_c_i64, [_vp]),
    "wm_capacity": (_c_i64, [_vp]),
    "wm_current_frame": (_c_i64, [_vp]),
    "wm_raw_slot": (_c_int, [_vp, _c_i64]),
    "wm_sum_slot": (_c_int, [_vp, _c_i64]),
    "wm_kv_ptrs": (_c_int, [_vp, _c_int, ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "wm_sync_status": (_c_int, [_vp]),
    "wm_set_wait_limit": (_c_int, [_vp, ctypes.c_uint64]),
    "wm_strerror": (ctypes.c_char_p, [_c_int]),
    "wm_last_cuda_error": (ctypes.c_char_p, []),
    "wm_selftest_exp2": (_c_int, [_vp, _vp, _c_i64, _vp]),
    "wm_layout_capacity": (_c_i64, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "wm_layout_end": (_c_i64, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_i64]),
    "wm_layout_raw_slot": (_c_int, [_c_int, _c_i64]),
    "wm_layout_sum_slot": (_c_int, [_c_int, _c_int, _c_i64]),
    "wm_layout_record_row": (_c_i64, [_c_int, _c_int, _c_int, _c_int, _c_i64]),
    "wm_attend_dense": (_c_int, [_vp, _vp, _vp, _vp, _c_i64, _c_i64, _c_int, _c_int, _vp, _vp]),
    "wm_attend_dense_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_i64, _c_i64, _c_int, _c_int,
                                     _vp, _c_i64, _vp, _vp]),
    "wm_attend_dense_fp8_scratch_bytes": (_c_i64, [_c_i64, _c_int, _c_int]),
    "wm_attend_dense_fp8_static": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_i64, _c_i64, _c_int,
                                            _c_int, _vp, _vp]),
}

WM_FP8_STATIC_SCRATCH_BYTES = 32 << 20

WM_KV_BF16 = 0
WM_KV_E4M3 = 1


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libwmkv.so not built at {LIB_PATH}; run python -m kv_memory_attention_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


class WmError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = LIB.wm_strerror(code).decode()
        if code == WM_ERR_CUDA:
            msg += f" ({LIB.wm_last_cuda_error().decode()})"
        super().__init__(f"{where}: {msg} [{code}]")
        self.code = code


def _check(code: int, where: str) -> int:
    if code != WM_OK:
        raise WmError(code, where)
    return code


def _ptr(x) -> int | None:
    """Device pointer of a tensor, or an int address as is; None stays NULL."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    """A torch.cuda.Stream, a raw cudaStream_t int, or None (torch's current stream)."""
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------- ABI wrappers

def wm_kvbuf_create(blocks: int, heads: int, d: int, grid_h: int, grid_w: int, X: int, Y: int,
                    W: int) -> int:
    h = _vp()
    _check(LIB.wm_kvbuf_create(ctypes.byref(h), blocks, heads, d, grid_h, grid_w, X, Y, W),
           "wm_kvbuf_create")
    return h.value


def wm_kvbuf_create_fp8(blocks: int, heads: int, d: int, grid_h: int, grid_w: int, X: int, Y: int,
                        W: int, k_scale, v_scale) -> int:
    """k_scale / v_scale: blocks * heads floats each (block-major)."""
    n = blocks * heads
    if len(k_scale) != n or len(v_scale) != n:
        raise ValueError(f"expected {n} scales per tensor")
    ks = (ctypes.c_float * n)(*[float(x) for x in k_scale])
    vs = (ctypes.c_float * n)(*[float(x) for x in v_scale])
    h = _vp()
    _check(LIB.wm_kvbuf_create_fp8(ctypes.byref(h), blocks, heads, d, grid_h, grid_w, X, Y, W, ks, vs),
           "wm_kvbuf_create_fp8")
    return h.value


def wm_kv_format(h: int) -> int:
    return LIB.wm_kv_format(h)


def wm_kvbuf_destroy(h: int) -> None:
    _check(LIB.wm_kvbuf_destroy(h), "wm_kvbuf_destroy")


def wm_advance(h: int, t: int, stream=None) -> None:
    _check(LIB.wm_advance(h, t, _stream(stream)), "wm_advance")


def wm_write_record(h: int, block: int, t: int, K, V, stream=None) -> None:
    _check(LIB.wm_write_record(h, block, t, _ptr(K), _ptr(V), _stream(stream)), "wm_write_record")


def wm_attend(h: int, block: int, Q, O, stream=None) -> None:
    _check(LIB.wm_attend(h, block, _ptr(Q), _ptr(O), _stream(stream)), "wm_attend")


def wm_write_attend(h: int, block: int, t: int, Q, K, V, O, stream=None) -> None:
    _check(LIB.wm_write_attend(h, block, t, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _stream(stream)),
           "wm_write_attend")


def wm_set_sink(h: int, theta, gap_trigger: int = 5, gap_target: int = 1) -> None:
    arr = (ctypes.c_float * len(theta))(*[float(x) for x in theta])
    _check(LIB.wm_set_sink(h, arr, len(theta), gap_trigger, gap_target), "wm_set_sink")


def wm_sink_position(h: int) -> int:
    return LIB.wm_sink_position(h)


def wm_sink_cos_sin(h: int, shift: int, n_pairs: int):
    c = (ctypes.c_float * n_pairs)()
    s = (ctypes.c_float * n_pairs)()
    _check(LIB.wm_sink_cos_sin(h, shift, c, s), "wm_sink_cos_sin")
    return list(c), list(s)


def wm_end(h: int) -> int:
    return LIB.wm_end(h)


def wm_capacity(h: int) -> int:
    return LIB.wm_capacity(h)


def wm_current_frame(h: int) -> int:
    return LIB.wm_current_frame(h)


def wm_raw_slot(h: int, t: int) -> int:
    return LIB.wm_raw_slot(h, t)


def wm_sum_slot(h: int, f: int) -> int:
    return LIB.wm_sum_slot(h, f)


def wm_kv_ptrs(h: int, block: int) -> tuple[int, int]:
    k, v = _vp(), _vp()
    _check(LIB.wm_kv_ptrs(h, block, ctypes.byref(k), ctypes.byref(v)), "wm_kv_ptrs")
    return k.value, v.value


def wm_sync_status(h: int) -> None:
    _check(LIB.wm_sync_status(h), "wm_sync_status")


def wm_set_wait_limit(h: int, cycles: int) -> None:
    _check(LIB.wm_set_wait_limit(h, cycles), "wm_set_wait_limit")


DEFAULT_WAIT_LIMIT_CYCLES = 4_000_000_000


def wm_strerror(code: int) -> str:
    return LIB.wm_strerror(code).decode()


def wm_attend_dense(Q, K, V, O, Lq: int, Lk: int, heads: int, d: int, dev_status=None,
                    stream=None) -> None:
    _check(LIB.wm_attend_dense(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), Lq, Lk, heads, d,
                               _ptr(dev_status), _stream(stream)), "wm_attend_dense")


def wm_attend_dense_fp8_scratch_bytes(Lk: int, heads: int, d: int) -> int:
    return LIB.wm_attend_dense_fp8_scratch_bytes(Lk, heads, d)


def wm_attend_dense_fp8(Q, K8, V8, k_scale, v_scale, O, Lq: int, Lk: int, heads: int, d: int,
                        scratch, scratch_bytes: int, dev_status=None, stream=None) -> None:
    _check(LIB.wm_attend_dense_fp8(_ptr(Q), _ptr(K8), _ptr(V8), _ptr(k_scale), _ptr(v_scale), _ptr(O),
                                   Lq, Lk, heads, d, _ptr(scratch), scratch_bytes, _ptr(dev_status),
                                   _stream(stream)), "wm_attend_dense_fp8")


def wm_attend_dense_fp8_static(Q, K8, V8, k_scale, v_scale, O, Lq: int, Lk: int, heads: int, d: int,
                               dev_status=None, stream=None) -> None:
    """wm_attend_dense_fp8 with the library's fixed device scratch (no allocation)."""
    _check(LIB.wm_attend_dense_fp8_static(_ptr(Q), _ptr(K8), _ptr(V8), _ptr(k_scale), _ptr(v_scale),
                                          _ptr(O), Lq, Lk, heads, d, _ptr(dev_status), _stream(stream)),
           "wm_attend_dense_fp8_static")


def wm_selftest_exp2(x, y, n: int, stream=None) -> None:
    _check(LIB.wm_selftest_exp2(_ptr(x), _ptr(y), n, _stream(stream)), "wm_selftest_exp2")


def wm_layout_capacity(grid_h, grid_w, X, Y, W) -> int:
    return LIB.wm_layout_capacity(grid_h, grid_w, X, Y, W)


def wm_layout_end(grid_h, grid_w, X, Y, W, t) -> int:
    return LIB.wm_layout_end(grid_h, grid_w, X, Y, W, t)


def wm_layout_raw_slot(Y, t) -> int:
    return LIB.wm_layout_raw_slot(Y, t)


def wm_layout_sum_slot(Y, W, f) -> int:
    return LIB.wm_layout_sum_slot(Y, W, f)


def wm_layout_record_row(grid_h, grid_w, X, Y, t) -> int:
    return LIB.wm_layout_record_row(grid_h, grid_w, X, Y, t)


# ---------------------------------------------------------------- convenience

class KVMemory:
    """One session's frame memory: owns a ``wm_kvbuf`` handle.

    ``kv_views(block)`` returns torch views of the block's K and V buffers,
    ``[C, heads, d]`` bf16 (read them only after the stream has reached the
    calls that wrote them).
    """

    def __init__(self, blocks, heads, d, grid_h, grid_w, X, Y, W, kv_format="bf16",
                 k_scale=None, v_scale=None):
        self.blocks, self.heads, self.d = blocks, heads, d
        self.grid_h, self.grid_w, self.X, self.Y, self.W = grid_h, grid_w, X, Y, W
        self.HW = grid_h * grid_w
        self.R = self.HW + X
        self.kv_format = kv_format
        self.h = None
        if kv_format == "bf16":
            self.h = wm_kvbuf_create(blocks, heads, d, grid_h, grid_w, X, Y, W)
        elif kv_format == "e4m3":
            self.h = wm_kvbuf_create_fp8(blocks, heads, d, grid_h, grid_w, X, Y, W,
                                         list(k_scale), list(v_scale))
        else:
            raise ValueError(kv_format)
        self.C = wm_capacity(self.h)

    def close(self):
        if self.h:
            wm_kvbuf_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def advance(self, t, stream=None):
        wm_advance(self.h, t, stream)

    def write_record(self, block, t, K, V, stream=None):
        wm_write_record(self.h, block, t, K, V, stream)

    def attend(self, block, Q, O, stream=None):
        wm_attend(self.h, block, Q, O, stream)

    def write_attend(self, block, t, Q, K, V, O, stream=None):
        wm_write_attend(self.h, block, t, Q, K, V, O, stream)

    def end(self):
        return wm_end(self.h)

    def set_sink(self, theta, gap_trigger=5, gap_target=1):
        wm_set_sink(self.h, theta, gap_trigger, gap_target)

    def sink_position(self):
        return wm_sink_position(self.h)

    def sync_status(self):
        wm_sync_status(self.h)

    def set_wait_limit(self, cycles):
        wm_set_wait_limit(self.h, cycles)

    def kv_views(self, block):
        """Torch views of the block's buffers: bf16, or uint8 E4M3 codes."""
        import torch
        kp, vp = wm_kv_ptrs(self.h, block)
        n = self.C * self.heads * self.d
        dt = torch.uint8 if self.kv_format == "e4m3" else torch.bfloat16
        return (_device_view(kp, n, dt).view(self.C, self.heads, self.d),
                _device_view(vp, n, dt).view(self.C, self.heads, self.d))


def _device_view(ptr: int, numel: int, dtype):
    """A torch tensor aliasing library-owned device memory (no copy, no ownership)."""
    import torch
    one_byte = dtype == torch.uint8

    class _Holder:
        def __init__(self, p, n):
            self.__cuda_array_interface__ = {
                "shape": (n,), "typestr": "|u1" if one_byte else "<i2", "data": (p, False),
                "version": 3, "strides": None}

    t = torch.as_tensor(_Holder(ptr, numel), device="cuda")
    return t if one_byte else t.view(dtype)

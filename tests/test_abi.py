"""CPU tests of the C ABI: the library loads, exports what include/wmkv.h
declares, and its host-side layout arithmetic and argument checks agree with
the oracle.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

from oracle import SCALED, SERVED, SERVED_W16, TINY, Layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wmkv.h")


@pytest.fixture(scope="module")
def wm():
    import kv_memory_attention_b200 as wm
    return wm


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^WM_API\s+[\w\s\*]+?\b(wm_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("wm_kvbuf_create", "wm_write_record", "wm_advance", "wm_attend",
                     "wm_attend_dense", "wm_sync_status", "wm_kv_ptrs"):
        assert required in names


def test_library_exports_every_declared_symbol(wm):
    lib = ctypes.CDLL(wm.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(wm.SIGNATURES)


LAYOUTS = [TINY, SERVED, SERVED_W16, SCALED, Layout(3, 5, 2, 0, 4), Layout(3, 5, 2, 3, 3),
           Layout(1, 1, 1, 0, 0), Layout(7, 9, 13, 5, 31)]


@pytest.mark.parametrize("L", LAYOUTS)
def test_layout_arithmetic_matches_oracle(wm, L):
    assert wm.wm_layout_capacity(L.grid_h, L.grid_w, L.X, L.Y, L.W) == L.C
    for t in range(0, 201):
        assert wm.wm_layout_end(L.grid_h, L.grid_w, L.X, L.Y, L.W, t) == L.end(t)
        assert wm.wm_layout_record_row(L.grid_h, L.grid_w, L.X, L.Y, t) == L.record_rows(t)[0]
        if t >= 1:
            assert wm.wm_layout_raw_slot(L.Y, t) == L.raw_slot(t)
            if L.W > L.Y:
                assert wm.wm_layout_sum_slot(L.Y, L.W, t) == L.sum_slot(t)
            else:
                assert wm.wm_layout_sum_slot(L.Y, L.W, t) == -1
    assert wm.wm_layout_end(L.grid_h, L.grid_w, L.X, L.Y, L.W, -1) == -1
    assert wm.wm_layout_raw_slot(L.Y, 0) == -1


def test_layout_rejects_bad_geometry(wm):
    assert wm.wm_layout_capacity(0, 5, 2, 1, 4) == -1
    assert wm.wm_layout_capacity(3, 5, 0, 1, 4) == -1
    assert wm.wm_layout_capacity(3, 5, 2, 5, 4) == -1       # W < Y
    assert wm.wm_layout_end(3, 5, 2, -1, 4, 3) == -1


@pytest.mark.parametrize("args,code", [
    ((0, 16, 64, 24, 42, 96, 2, 24), -1),     # blocks
    ((1, 0, 64, 24, 42, 96, 2, 24), -1),      # heads
    ((1, 16, 64, 0, 42, 96, 2, 24), -1),      # grid_h
    ((1, 16, 64, 24, 42, 0, 2, 24), -1),      # X
    ((1, 16, 64, 24, 42, 96, -1, 24), -1),    # Y
    ((1, 16, 64, 24, 42, 96, 5, 4), -1),      # W < Y
    ((1, 16, 32, 24, 42, 96, 2, 24), -3),     # d unsupported
    ((1, 16, 96, 24, 42, 96, 2, 24), -3),
])
def test_create_rejects_bad_arguments_before_the_device(wm, args, code):
    with pytest.raises(wm.WmError) as e:
        wm.wm_kvbuf_create(*args)
    assert e.value.code == code


def test_null_handle_and_pointer_errors(wm):
    lib = wm.LIB
    assert lib.wm_advance(None, 0, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_write_record(None, 0, 0, 16, 16, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_attend(None, 0, 16, 16, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_sync_status(None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_set_wait_limit(None, 5) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_selftest_exp2(None, 16, 2, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_selftest_exp2(16, 16, 3, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_selftest_exp2(12, 16, 2, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_kvbuf_destroy(None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_end(None) == -1
    # dense: misaligned / null pointers and bad sizes never reach the device
    assert lib.wm_attend_dense(None, 16, 16, 16, 1, 1, 1, 64, None, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_attend_dense(24, 16, 16, 16, 1, 1, 1, 64, None, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_attend_dense(16, 16, 16, 16, 0, 1, 1, 64, None, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_attend_dense(16, 16, 16, 16, 1, 0, 1, 64, None, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_attend_dense(16, 16, 16, 16, 1, 1, 65536, 64, None, None) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_attend_dense(16, 16, 16, 16, 1, 1, 1, 96, None, None) == wm.WM_ERR_UNSUPPORTED
    assert lib.wm_attend_dense(16, 16, 16, 16, 1, 1, 1, 80, None, None) == wm.WM_ERR_UNSUPPORTED


def test_fp8_argument_checks(wm):
    lib = wm.LIB
    h = ctypes.c_void_p()
    ones = (ctypes.c_float * 4)(1.0, 1.0, 1.0, 1.0)
    bad = (ctypes.c_float * 4)(1.0, 0.0, 1.0, 1.0)
    nan = (ctypes.c_float * 4)(1.0, float("nan"), 1.0, 1.0)
    args = (2, 2, 64, 4, 6, 4, 2, 6)
    assert lib.wm_kvbuf_create_fp8(ctypes.byref(h), *args, None, ones) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_kvbuf_create_fp8(ctypes.byref(h), *args, ones, bad) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_kvbuf_create_fp8(ctypes.byref(h), *args, nan, ones) == wm.WM_ERR_INVALID_ARG
    assert lib.wm_kvbuf_create_fp8(ctypes.byref(h), 2, 2, 96, 4, 6, 4, 2, 6, ones, ones) == \
        wm.WM_ERR_UNSUPPORTED
    assert lib.wm_kv_format(None) == wm.WM_ERR_INVALID_ARG
    assert wm.wm_attend_dense_fp8_scratch_bytes(1000, 3, 64) == 2 * 1000 * 3 * 64 * 2
    assert wm.wm_attend_dense_fp8_scratch_bytes(0, 3, 64) == -1
    assert wm.wm_attend_dense_fp8_scratch_bytes(10, 3, 80) == -1
    f = lib.wm_attend_dense_fp8
    assert f(16, 16, 16, None, 16, 16, 1, 1, 1, 64, 16, 256, None, None) == wm.WM_ERR_INVALID_ARG
    assert f(16, 16, 24, 16, 16, 16, 1, 1, 1, 64, 16, 256, None, None) == wm.WM_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, 16, 1, 1, 1, 64, 16, 255, None, None) == wm.WM_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, 16, 1, 0, 1, 64, 16, 256, None, None) == wm.WM_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, 16, 1, 1, 1, 96, 16, 1 << 20, None, None) == wm.WM_ERR_UNSUPPORTED


def test_strerror_covers_codes(wm):
    for c in range(0, -7, -1):
        assert wm.wm_strerror(c) and wm.wm_strerror(c) != "unknown error"
    assert wm.wm_strerror(-99) == "unknown error"

"""wm_attend_dense_fp8_static: the dense FP8 attention for callers that
cannot allocate device memory (a plug-in handed only one call's tensors, a
framework whose pool owns every allocation, a server that must not grow its
footprint once running).  It widens the keys and values into a fixed device
array inside the library instead of caller-provided scratch.

The test calls it twice in a row through the C ABI, on different inputs and
sizes (so the second call runs over what the first left in the shared array),
and compares each output with wm_attend_dense_fp8 on the same inputs with
caller-owned scratch, within the tolerance the other attention tests use.  It
also checks that a call too large for the array is refused.  It runs the same
alone in a fresh process or after the other tests (the array's address is
looked up on the first call, whenever that comes).  This file is named so
that pytest collects it last.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import e4m3_encode
from gpu_util import assert_attn_close, dev, host_bits, require_gpu, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wm():
    require_gpu()
    import kv_memory_attention_b200 as wm
    return wm


def fp8_inputs(lq, lk, heads, d, seed):
    rng = np.random.default_rng(seed)
    q = si.normal_bf16(si.seed_for(92, seed, lq, lk, heads * 1000 + d, si.T_Q), (lq, heads, d))
    ks = rng.uniform(1 / 100, 1 / 20, heads).astype(np.float32)
    vs = rng.uniform(1 / 100, 1 / 20, heads).astype(np.float32)
    k8 = e4m3_encode(rng.standard_normal((lk, heads, d)).astype(np.float32) * 2 / ks[None, :, None])
    v8 = e4m3_encode(rng.standard_normal((lk, heads, d)).astype(np.float32) / vs[None, :, None])
    return (dev(q), torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda(),
            torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda())


def test_static_scratch_matches_caller_scratch_twice(wm):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # served-size first (6,528 keys x 16 heads x 64: 26.7 MB of the 32 MiB array), then a
    # smaller, differently shaped call that reuses the array's first bytes
    for lq, lk, heads, d, seed in ((1104, 6528, 16, 64, 1), (300, 1000, 3, 128, 2)):
        q, k8, v8, ks, vs = fp8_inputs(lq, lk, heads, d, seed)
        nbytes = wm.wm_attend_dense_fp8_scratch_bytes(lk, heads, d)
        scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o_ref = torch.full((lq, heads, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        wm.wm_attend_dense_fp8(q, k8, v8, ks, vs, o_ref, lq, lk, heads, d, scratch, nbytes, status)
        o = torch.full((lq, heads, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        wm.wm_attend_dense_fp8_static(q, k8, v8, ks, vs, o, lq, lk, heads, d, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = host_bits(o_ref)
        assert np.isfinite(si.bf16_bits_to_f64(ref)).all()
        assert_attn_close(host_bits(o), si.bf16_bits_to_f64(ref), f"static vs caller scratch {lq}x{lk}")


def test_static_scratch_refuses_calls_beyond_its_size(wm):
    x = torch.zeros(64, dtype=torch.uint8, device="cuda")
    lk = wm.WM_FP8_STATIC_SCRATCH_BYTES // (2 * 16 * 64 * 2) + 1      # one key too many
    assert wm.wm_attend_dense_fp8_scratch_bytes(lk, 16, 64) > wm.WM_FP8_STATIC_SCRATCH_BYTES
    with pytest.raises(wm.WmError) as e:
        wm.wm_attend_dense_fp8_static(x, x, x, x, x, x, 1, lk, 16, 64)
    assert e.value.code == wm.WM_ERR_INVALID_ARG

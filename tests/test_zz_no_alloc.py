"""qknorm_layerwise_noalloc: layerwise QK-Norm for callers that cannot
allocate GPU memory when they call in (a runtime with its own fixed memory
pool, an application that forbids allocations on its hot path).  The entry
point keeps its intermediate per-token sums in a static array inside the
library, so the caller passes only its own buffer and weights.

The test calls it through the C ABI twice in a row, on two different inputs,
and compares each result with the float64 oracle and with the existing
qknorm_layerwise entry point on the same input, within the parity
tolerances of the other GPU tests.  The second call runs over the array the
first one filled, so a result that depended on leftovers would show.  The
device counter of in-kernel waits that gave up must not move.  This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import attention_qk_norm_b200 as qkn
from attention_qk_norm_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

DTYPE_CODE = {synth.BF16: 0, synth.FP32: 1, synth.FP16: 2, synth.FP8: 3}


def _entry():
    f = qkn.load_library().qknorm_layerwise_noalloc
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    f.argtypes = [vp, i32, i64, i32, i32, i32, i64, vp, vp, f32, vp]
    f.restype = i32
    return f


def _call(f, buf, c, gq, gk):
    return f(ctypes.c_void_p(buf.data_ptr()), DTYPE_CODE[c.dtype], c.T, c.Hq, c.Hk, c.D,
             c.row_stride, ctypes.c_void_p(gq.data_ptr()),
             ctypes.c_void_p(gk.data_ptr()) if gk is not None else None, c.eps,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_layerwise_two_calls_in_a_row():
    f = _entry()
    cases = [
        synth.make_case(1000, 32, 8, 128, seed=301, layerwise=True, scale="lognormal"),
        synth.make_case(257, 64, 8, 64, dtype=synth.FP32, seed=302, layerwise=True,
                        scale="stress", zero_frac=0.02, outlier_frac=0.02),
    ]
    torch.cuda.synchronize()
    timeouts_before = qkn.wait_timeouts()
    for c in cases:
        mine, gq, gk = gu.to_device(c)
        ref = mine.clone()
        assert _call(f, mine, c, gq, gk) == 0
        qkn.qknorm_layerwise(ref, c.Hq, c.Hk, c.D, gq, gk, c.eps, nshards=1)
        torch.cuda.synchronize()
        got, want = gu.stored_bits(mine), gu.stored_bits(ref)
        qk = (c.Hq + c.Hk) * c.D
        oracle_want = gu.oracle_out(c, "layerwise", c.qkv, c.T)
        gu.check(got, oracle_want, c.qkv, c.dtype, qk, "noalloc vs oracle T=%d" % c.T)
        gu.check(got, gu.as_f64(want, c.dtype), c.qkv, c.dtype, qk, "noalloc T=%d" % c.T)
    assert qkn.wait_timeouts() == timeouts_before


def test_noalloc_rejects_tokens_beyond_its_scratch():
    f = _entry()
    c = synth.make_case(65537, 1, 0, 64, seed=303, layerwise=True)
    buf, gq, _ = gu.to_device(c)
    before = buf.clone()
    assert _call(f, buf, c, gq, None) == -8
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), before.view(torch.int16))

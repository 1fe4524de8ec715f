"""attn_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plugin inside a framework that owns
all device memory, a latency-critical path).  attn_bwd_noalloc takes no
workspace; it uses a fixed scratch array inside the library.  This file is
collected last so that a failure here leaves every other test already run.
The check: the cases run small, large, small (each case twice in a row)
through the C ABI, so the shared scratch array is reused after a smaller and
after a larger problem; every call is compared against attn_bwd with a
caller-allocated workspace (dK/dV bit-identical, dQ within the backward
tolerance: it differs only by the order of fp32 reduce-adds) and against
the float64 oracle with the tolerance of the other backward tests.
"""

import oracle

import ctypes

import numpy as np
import pytest

from synth import make_shape_inputs
from tests._util import check_grad, to_dev, to_f64

SCRATCH_BYTES = 32 << 20


@pytest.fixture(scope="module")
def ta():
    import tiled_exact_attention_02_b200 as ta
    f = ta.lib.attn_bwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp] * 9 + [i] * 6 + [ctypes.c_float, i, i, vp]
    f.restype = i
    return ta


def _noalloc(ta, q, k, v, o, lse, do, dq, dk, dv, causal, window, scale):
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    import torch
    return ta.lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq, Lk, d,
                                   scale, int(causal), window, torch.cuda.current_stream().cuda_stream)


def test_noalloc_rejects_problems_beyond_its_scratch(ta):
    # Validation happens before anything is launched.
    rows = SCRATCH_BYTES // (129 * 4) + 1024
    P = 1 << 20
    assert ta.lib.attn_bwd_noalloc(*([P] * 9), 1, 1, 1, rows, 128, 128, 0.1, 1, 0, None) == ta.ATTN_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_matches_attn_bwd_twice(ta):
    import torch
    small = (2, 2, 2, 333, 333, 64, True, 40)
    large = (1, 4, 2, 1000, 1000, 128, True, 0)
    for B, Hq, Hkv, Lq, Lk, d, causal, window in (small, large, small):
        x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq + d, with_do=True)
        q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
        scale = d ** -0.5
        o, lse = ta.attention(q, k, v, causal, window, scale)
        ref = ta.attention_backward(q, k, v, o, lse, do, causal, window, scale)
        rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window)
        for _ in range(2):
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            st = _noalloc(ta, q, k, v, o, lse, do, dq, dk, dv, causal, window, scale)
            assert st == ta.ATTN_OK, ta.status_string(st)
            assert ta.device_error()[0] == ta.ATTN_OK
            for name, got, want, orc in (("dQ", dq, ref[0], rq), ("dK", dk, ref[1], rk), ("dV", dv, ref[2], rv)):
                check_grad(to_f64(got), to_f64(want), name + " vs attn_bwd")
                check_grad(to_f64(got), orc, name + " vs oracle")
            assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])

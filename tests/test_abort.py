"""The backward kernel's abort path, exercised without a GPU fault.

attn_selftest_bwd_abort runs the real backward with one barrier arrival
withheld (a wait that nothing completes), and a short wait limit.  The
bounded wait runs out; every role of the CTA then lets what it started
finish (TMA copies, MMAs, the dQ reduce-adds), tensor memory is freed and the
kernel exits.  The test checks that the timeout is reported, that the call
ends promptly, that guard bytes around every output and the workspace are
untouched, and that the context computes correct results afterwards.
"""

import time

import numpy as np
import pytest

import oracle
from synth import make_shape_inputs
from tests._util import check_grad, to_dev, to_f64


@pytest.fixture(scope="module")
def ta():
    import tiled_exact_attention_02_b200 as ta
    return ta


@pytest.mark.gpu
@pytest.mark.parametrize("d,stall_step", [(128, 3), (128, 0), (64, 2)])
def test_backward_abort_reports_timeout_and_leaves_context_usable(ta, d, stall_step):
    import torch
    from tests.test_canaries import Guarded
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    B, Hq, Hkv, L = 1, 4, 2, 1000
    x = make_shape_inputs(B, Hq, Hkv, L, L, d, seed=77 + d, with_do=True)
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    scale = d ** -0.5
    o, lse = ta.attention(q, k, v, True, 0, scale)
    assert ta.device_error()[0] == ta.ATTN_OK
    dq = Guarded(tuple(q.shape), torch.bfloat16, seed=1)
    dk = Guarded(tuple(k.shape), torch.bfloat16, seed=2)
    dv = Guarded(tuple(v.shape), torch.bfloat16, seed=3)
    ws = Guarded((ta.bwd_workspace_size(B, Hq, Hkv, L, L, d),), torch.uint8, seed=4)
    sp = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    st = ta.lib.attn_selftest_bwd_abort(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                        do.data_ptr(), dq.t.data_ptr(), dk.t.data_ptr(), dv.t.data_ptr(),
                                        B, Hq, Hkv, L, L, d, scale, 1, 0, stall_step, 20_000_000,
                                        ws.t.data_ptr(), ws.nbytes, sp)
    assert st == ta.ATTN_OK, ta.status_string(st)
    status, site = ta.device_error()
    elapsed = time.perf_counter() - t0
    assert status == ta.ATTN_ERR_TIMEOUT, (status, site)
    assert site >= 100  # a wait site of the backward kernel
    assert elapsed < 10.0
    for name, g in (("dQ", dq), ("dK", dk), ("dV", dv), ("workspace", ws)):
        assert g.intact(), f"the aborted backward wrote outside {name}"
    assert ta.device_error()[0] == ta.ATTN_OK  # the word was cleared
    # The same context then computes the right gradients.
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, True, 0)
    gq, gk, gv = ta.attention_backward(q, k, v, o, lse, do, True, 0, scale)
    assert ta.device_error()[0] == ta.ATTN_OK
    check_grad(to_f64(gq), rq, "dQ")
    check_grad(to_f64(gk), rk, "dK")
    check_grad(to_f64(gv), rv, "dV")


def test_abort_selftest_rejects_bad_arguments(ta):
    # Validation returns before anything is launched (runs on the CPU).
    P = 1 << 20
    args = [P] * 9 + [1, 2, 1, 64, 64, 128, 0.1, 1, 0]
    assert ta.lib.attn_selftest_bwd_abort(*args, -1, 1000, P, 1 << 20, None) == ta.ATTN_ERR_INVALID_ARG
    assert ta.lib.attn_selftest_bwd_abort(*args, 0, 0, P, 1 << 20, None) == ta.ATTN_ERR_INVALID_ARG
    assert ta.lib.attn_selftest_bwd_abort(*args, 0, 20_000_000_000, P, 1 << 20, None) == ta.ATTN_ERR_INVALID_ARG

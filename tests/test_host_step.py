"""attn_step_host (host buffers, chunked copies overlapped with the kernels)
against the device entry points on the whole problem and against the oracle.

O, LSE, dK and dV come from the same kernels with the same per-row and
per-key arithmetic order, so they must match the device path bit for bit.
dQ is summed over key tiles by fp32 reduce-adds whose order depends on CTA
timing, so it is compared with the backward tolerance instead (and against
the oracle on the small case).
"""

import numpy as np
import pytest

import oracle
from synth import make_shape_inputs
from tests._util import check_grad, check_lse, check_o, rel_fro, row_errors, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_exact_attention_02_b200 as ta
    return ta


def _host(bits, pinned):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


def _run_host(ta, x, causal, window, scale, backward, pinned):
    import torch
    q, k, v = (_host(x[n], pinned) for n in "qkv")
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    alloc = (lambda shape, dt: torch.empty(shape, dtype=dt, pin_memory=True)) if pinned else \
        (lambda shape, dt: torch.empty(shape, dtype=dt))
    o = alloc(q.shape, torch.bfloat16)
    lse = alloc((B, Hq, Lq), torch.float32)
    extra = {}
    if backward:
        extra = dict(do=_host(x["do"], pinned), dq=alloc(q.shape, torch.bfloat16), dk=alloc(k.shape, torch.bfloat16),
                     dv=alloc(v.shape, torch.bfloat16))
    buf = torch.empty(ta.step_host_buffer_size(B, Hq, Hkv, Lq, Lk, d, backward), dtype=torch.uint8, device="cuda")
    ta.step_host(q, k, v, o, lse, buf, causal=causal, window=window, scale=scale, **extra)
    torch.cuda.current_stream().synchronize()
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    return o, lse, extra


# (B, Hq, Hkv, Lq, Lk, d, causal, window): several chunks per sequence, GQA, masks, ragged tiles
CASES = [
    (2, 8, 2, 300, 300, 128, 1, 0),
    (3, 4, 4, 257, 500, 64, 2, 64),
    (1, 16, 2, 200, 200, 128, 0, 50),
    (2, 32, 8, 16, 1000, 128, 2, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window", CASES)
@pytest.mark.parametrize("pinned", [True, False])
def test_step_host_matches_device_path(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, pinned):
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=B * 7 + Hq + Lq + Lk + d, with_do=True)
    scale = d ** -0.5
    o_h, lse_h, g = _run_host(ta, x, causal, window, scale, True, pinned)

    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = ta.attention(q, k, v, causal, window, scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ta.bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d), dtype=torch.uint8, device="cuda")
    ta.bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal, window, scale)
    torch.cuda.synchronize()

    assert torch.equal(o_h, o.cpu()), "O differs from attn_fwd"
    assert torch.equal(lse_h, lse.cpu()), "LSE differs from attn_fwd"
    assert torch.equal(g["dk"], dk.cpu()), "dK differs from attn_bwd"
    assert torch.equal(g["dv"], dv.cpu()), "dV differs from attn_bwd"
    assert rel_fro(to_f64(g["dq"]), to_f64(dq)) <= 1e-3, "dQ differs from attn_bwd"
    assert np.max(row_errors(to_f64(g["dq"]), to_f64(dq)), initial=0.0) <= 1e-2, "a dQ row differs from attn_bwd"


def test_step_host_forward_only_against_oracle(ta):
    B, Hq, Hkv, Lq, Lk, d, causal, window = 2, 6, 3, 130, 270, 128, 2, 0
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=123)
    scale = d ** -0.5
    o_h, lse_h, _ = _run_host(ta, x, causal, window, scale, False, True)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window)
    check_o(to_f64(o_h), ro, "O")
    check_lse(to_f64(lse_h), rl, "LSE")


def test_step_host_backward_against_oracle(ta):
    B, Hq, Hkv, Lq, Lk, d, causal, window = 1, 4, 2, 200, 200, 64, 1, 0
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=321, with_do=True)
    scale = d ** -0.5
    _, _, g = _run_host(ta, x, causal, window, scale, True, True)
    rdq, rdk, rdv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window)
    for name, got, ref in (("dQ", g["dq"], rdq), ("dK", g["dk"], rdk), ("dV", g["dv"], rdv)):
        check_grad(to_f64(got), ref, name)


def test_step_host_error_after_queued_chunks_leaves_buffers_quiet(ta):
    """A failure at a late chunk (made on the host by the self-test hook) is
    returned only after the chunks already queued have finished: host outputs
    overwritten right after the call are not touched by a late copy."""
    import torch
    B, Hq, Hkv, Lq, Lk, d = 2, 8, 8, 512, 512, 128  # 16 kv groups -> 8 chunks
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=99, with_do=True)
    q, k, v, do = (_host(x[n], True) for n in ("q", "k", "v", "do"))
    pin = lambda t: torch.zeros(t.shape, dtype=t.dtype, pin_memory=True)
    o, dq, dk, dv = pin(q), pin(q), pin(k), pin(v)
    lse = torch.zeros((B, Hq, Lq), dtype=torch.float32, pin_memory=True)
    buf = torch.empty(ta.step_host_buffer_size(B, Hq, Hkv, Lq, Lk, d, True), dtype=torch.uint8, device="cuda")
    assert ta.lib.attn_selftest_step_host_fail_at(6) == ta.ATTN_OK
    with pytest.raises(ta.AttnError) as ei:
        ta.step_host(q, k, v, o, lse, buf, do=do, dq=dq, dk=dk, dv=dv, causal=True, scale=d ** -0.5)
    assert ei.value.status == ta.ATTN_ERR_CUDA and "self-test" in str(ei.value)
    marker = torch.tensor(-7.0, dtype=torch.bfloat16)
    for t in (o, dq, dk, dv):
        t.fill_(marker)
    lse.fill_(-7.0)
    torch.cuda.synchronize()
    for t in (o, dq, dk, dv):
        assert bool((t == marker).all())
    assert bool((lse == -7.0).all())
    # The hook fires once: the next call runs normally.
    ta.step_host(q, k, v, o, lse, buf, do=do, dq=dq, dk=dk, dv=dv, causal=True, scale=d ** -0.5)
    torch.cuda.synchronize()
    assert ta.device_error()[0] == ta.ATTN_OK
    assert not bool((o == marker).any())

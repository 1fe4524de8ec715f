"""Backward parity: dQ, dK, dV from the CUDA path against the float64 oracle.

The forward outputs O and LSE fed to the backward pass come from the CUDA
forward (as in training); the oracle recomputes everything from Q, K, V, dO
in float64.  Tolerance: relative Frobenius error <= 2e-2 for each gradient.
"""

import numpy as np
import pytest

import oracle
from synth import WORKLOADS, make_inputs, make_shape_inputs
from tests._util import check_grad, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_exact_attention_02_b200 as ta
    return ta


def run_fwd_bwd(ta, x, causal, window, scale):
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = ta.attention(q, k, v, causal, window, scale)
    dq, dk, dv = ta.attention_backward(q, k, v, o, lse, do, causal, window, scale)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    return to_f64(dq), to_f64(dk), to_f64(dv)


EDGE = [
    (1, 1, 1, 128, 128, 128, False, 0),
    (1, 2, 2, 7, 7, 128, True, 0),
    (1, 2, 1, 129, 129, 128, True, 0),
    (2, 4, 2, 200, 200, 128, True, 0),
    (1, 2, 2, 100, 333, 128, False, 0),
    (1, 2, 2, 333, 100, 128, False, 0),
    (1, 4, 4, 257, 257, 128, True, 1),
    (1, 2, 2, 384, 384, 128, True, 1000),
    (1, 8, 1, 256, 256, 128, True, 0),
    (1, 6, 2, 300, 300, 128, True, 64),
    (1, 2, 2, 300, 100, 128, True, 50),
    (1, 1, 1, 128, 128, 64, False, 0),
    (1, 2, 1, 200, 200, 64, True, 0),
    (2, 4, 2, 333, 333, 64, True, 77),
    (1, 2, 2, 1000, 1000, 128, True, 0),
    # two-sided window (no causal mask): |i - j| < w
    (1, 2, 2, 257, 257, 128, False, 1),
    (1, 4, 2, 700, 700, 128, False, 100),
    (1, 2, 1, 300, 500, 64, False, 130),
    (1, 2, 2, 500, 300, 128, False, 64),
    # bottom-right causal (causal = 2): query i at key position i + Lk - Lq
    (1, 2, 2, 100, 333, 128, 2, 0),
    (1, 4, 2, 1, 1000, 128, 2, 0),
    (2, 2, 1, 333, 100, 64, 2, 0),
    (1, 2, 2, 200, 700, 128, 2, 64),
    (1, 4, 4, 129, 129, 128, 2, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window", EDGE)
def test_bwd_edge_shapes(ta, B, Hq, Hkv, Lq, Lk, d, causal, window):
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 3 + Lk + d + 1, with_do=True)
    scale = d ** -0.5
    dq, dk, dv = run_fwd_bwd(ta, x, causal, window, scale)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window)
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")


VARLEN = [
    (3, 4, 2, 300, 300, 128, 1, 0, [300, 129, 0], [300, 129, 0]),
    (3, 2, 2, 257, 400, 128, 2, 0, [1, 100, 257], [400, 37, 256]),
    (2, 4, 4, 200, 200, 64, 0, 0, [200, 77], [150, 200]),
    (2, 2, 1, 500, 500, 128, 1, 64, [500, 333], [500, 333]),
    (2, 2, 2, 300, 300, 128, 0, 50, [300, 128], [10, 300]),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,lq,lk", VARLEN)
def test_bwd_varlen(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, lq, lk):
    """Per-sequence lengths: gradients against the oracle, zeros in the padding."""
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 13 + Lk + d + 9, with_do=True)
    scale = d ** -0.5
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    tq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    tk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    o, lse = ta.attention(q, k, v, causal, window, scale, seqlens_q=tq, seqlens_k=tk)
    dq, dk, dv = ta.attention_backward(q, k, v, o, lse, do, causal, window, scale, seqlens_q=tq, seqlens_k=tk)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window, seqlens_q=lq, seqlens_k=lk)
    check_grad(to_f64(dq), rq, "dQ")
    check_grad(to_f64(dk), rk, "dK")
    check_grad(to_f64(dv), rv, "dV")
    for b in range(B):
        assert np.all(to_f64(dq)[b, :, lq[b]:] == 0)
        assert np.all(to_f64(dk)[b, :, lk[b]:] == 0) and np.all(to_f64(dv)[b, :, lk[b]:] == 0)


GLOBAL = [
    (1, 2, 2, 700, 700, 128, 0, 64, 1, 1),
    (1, 4, 2, 1000, 1000, 128, 1, 128, 4, 0),
    (2, 2, 1, 300, 500, 64, 2, 50, 130, 20),
    (1, 2, 2, 257, 257, 128, 0, 8, 0, 3),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,gh,gt", GLOBAL)
def test_bwd_global_tokens(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, gh, gt):
    """Gradients with global head/tail key positions, against the oracle."""
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 19 + Lk + d + gh + 5 * gt, with_do=True)
    scale = d ** -0.5
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = ta.attention(q, k, v, causal, window, scale, global_head=gh, global_tail=gt)
    dq, dk, dv = ta.attention_backward(q, k, v, o, lse, do, causal, window, scale, global_head=gh, global_tail=gt)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window, global_head=gh,
                                 global_tail=gt)
    check_grad(to_f64(dq), rq, "dQ")
    check_grad(to_f64(dk), rk, "dK")
    check_grad(to_f64(dv), rv, "dV")


# Block-sparse mask ("大模型高效注意力机制全解析" §4.1.2), block size b, alone and under
# causal / window masks, blocks smaller and larger than a tile, Lq != Lk.
# (B, Hq, Hkv, Lq, Lk, d, causal, window, b)
SPARSE = [
    (1, 2, 2, 700, 700, 128, 0, 0, 64),
    (1, 4, 2, 1000, 1000, 128, 1, 0, 128),
    (2, 2, 1, 300, 500, 64, 2, 0, 50),
    (1, 2, 2, 513, 513, 128, 0, 100, 200),
    (1, 4, 4, 257, 257, 64, 1, 64, 1),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,b", SPARSE)
def test_bwd_sparse_block(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, b):
    """Gradients under the block-sparse mask, against the oracle."""
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 23 + Lk + d + b, with_do=True)
    scale = d ** -0.5
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = ta.attention(q, k, v, causal, window, scale, sparse_block=b)
    dq, dk, dv = ta.attention_backward(q, k, v, o, lse, do, causal, window, scale, sparse_block=b)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window, sparse_block=b)
    check_grad(to_f64(dq), rq, "dQ")
    check_grad(to_f64(dk), rk, "dK")
    check_grad(to_f64(dv), rv, "dV")


def test_bwd_gqa_window_2048(ta):
    x = make_shape_inputs(1, 8, 2, 2048, 2048, 128, seed=17, with_do=True)
    dq, dk, dv = run_fwd_bwd(ta, x, True, 300, 128 ** -0.5)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], 128 ** -0.5, True, 300)
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")


def test_bwd_full_size_sampled_heads(ta):
    """The fwd+bwd workload at full size (benchmark launch configuration);
    whole K/V heads (independent units) from both sequences compared against
    the oracle, row by row."""
    w = WORKLOADS["mha_causal_fwdbwd"]
    x = make_inputs(w)
    dq, dk, dv = run_fwd_bwd(ta, x, w.causal, w.window, w.scale)
    heads = [(0, 0), (0, 17), (1, 5), (1, 31)]
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, w.window, heads=heads)
    for b, h in heads:
        check_grad(dq[b, h], rq[b, h], f"dQ[{b},{h}]")
        check_grad(dk[b, h], rk[b, h], f"dK[{b},{h}]")
        check_grad(dv[b, h], rv[b, h], f"dV[{b},{h}]")
    assert np.all(np.isfinite(dq)) and np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


@pytest.mark.parametrize("name,heads", [("gqa_causal_8192", [(0, 0), (3, 7)]), ("gqa_window_32768", [(0, 5)])])
def test_bwd_gqa_full_size_sampled_heads(ta, name, heads):
    """Backward of the full-size GQA workloads (causal with Q x 2, and the
    32768-token causal window of 4096) with a dO drawn after Q, K, V: whole
    K/V heads, i.e. the kv head's dK/dV summed over its 4 query heads and
    those heads' dQ, against the oracle row by row."""
    import dataclasses
    import torch
    w = dataclasses.replace(WORKLOADS[name], backward=True)
    x = make_inputs(w)
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    o, lse = ta.attention(q, k, v, w.causal, w.window, w.scale)
    dq, dk, dv = ta.attention_backward(q, k, v, o, lse, do, w.causal, w.window, w.scale)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())
    del q, k, v, o, lse, do
    G = w.Hq // w.Hkv
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, w.window, heads=heads)
    for b, g in heads:
        check_grad(to_f64(dk[b, g]), rk[b, g], f"dK[{b},{g}]")
        check_grad(to_f64(dv[b, g]), rv[b, g], f"dV[{b},{g}]")
        for h in range(g * G, (g + 1) * G):
            check_grad(to_f64(dq[b, h]), rq[b, h], f"dQ[{b},{h}]")


def test_autograd_wrapper(ta):
    import torch
    x = make_shape_inputs(1, 2, 1, 300, 300, 128, seed=3, with_do=True)
    q, k, v, do = (to_dev(x[n]).requires_grad_(n != "do") for n in ("q", "k", "v", "do"))
    o = ta.tiled_attention(q, k, v, True, 0, None)
    o.backward(do)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], 128 ** -0.5, True, 0)
    check_grad(to_f64(q.grad), rq, "dQ")
    check_grad(to_f64(k.grad), rk, "dK")
    check_grad(to_f64(v.grad), rv, "dV")


def test_bwd_repeated_calls_identical_up_to_atomics(ta):
    """Two backward calls on the same inputs agree (dQ differs only by the
    order of fp32 atomic adds)."""
    x = make_shape_inputs(1, 2, 2, 512, 512, 128, seed=8, with_do=True)
    a = run_fwd_bwd(ta, x, True, 0, 128 ** -0.5)
    b = run_fwd_bwd(ta, x, True, 0, 128 ** -0.5)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
    assert np.max(np.abs(a[0] - b[0])) <= 2 ** -6 * max(1.0, np.max(np.abs(a[0])))

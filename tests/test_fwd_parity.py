"""Forward parity: the CUDA path (through the C ABI) against the float64 oracle.

Same seeded bf16 inputs on both sides.  Tolerances: O max-abs 1e-2 and
relative Frobenius 5e-3; LSE 1e-5 relative (absolute below |LSE| = 1).
"""

import ctypes

import numpy as np
import pytest

import oracle
from synth import WORKLOADS, make_inputs, make_shape_inputs
from tests._util import check_lse, check_o, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_exact_attention_02_b200 as ta
    return ta


def run_fwd(ta, x, causal, window, scale, sparse_block=0):
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o, lse = ta.attention(q, k, v, causal, window, scale, sparse_block=sparse_block)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    return to_f64(o), to_f64(lse)


# (B, Hq, Hkv, Lq, Lk, d, causal, window): tails, partial tiles, masks, groups
EDGE = [
    (1, 1, 1, 1, 1, 64, False, 0),
    (1, 2, 2, 7, 7, 128, True, 0),
    (1, 2, 1, 129, 129, 64, True, 0),
    (2, 4, 2, 200, 200, 128, True, 0),
    (1, 2, 2, 100, 333, 128, False, 0),
    (1, 2, 2, 333, 100, 64, False, 0),
    (1, 4, 4, 257, 257, 64, True, 1),
    (1, 2, 2, 384, 384, 128, True, 1000),
    (1, 8, 1, 256, 256, 128, True, 0),
    (1, 6, 2, 300, 300, 128, True, 64),
    (1, 3, 3, 640, 640, 128, True, 130),
    (1, 2, 2, 300, 100, 128, True, 50),
    (2, 2, 2, 513, 513, 64, False, 0),
    (1, 4, 2, 1000, 1000, 128, True, 0),
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
def test_fwd_edge_shapes(ta, B, Hq, Hkv, Lq, Lk, d, causal, window):
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 7 + Lk + d)
    scale = d ** -0.5
    o, lse = run_fwd(ta, x, causal, window, scale)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window)
    check_o(o, ro, "O")
    check_lse(lse, rl, "LSE")


# Short queries with a GQA group (G > 1, Lq < 128): the G heads of a kv group
# share the tile rows (row r = query r % Lq of head r / Lq), one tile or two,
# tiles inside one head and across heads, the group's last tile ragged.
# (B, Hq, Hkv, Lq, Lk, d, causal, window)
PACKED = [
    (2, 8, 2, 16, 1000, 128, 2, 0),
    (1, 12, 2, 40, 700, 64, 2, 0),
    (1, 16, 2, 100, 900, 128, 1, 0),
    (3, 32, 8, 1, 5000, 128, 2, 0),
    (1, 4, 2, 64, 64, 128, 0, 16),
    (1, 6, 3, 127, 127, 128, 1, 0),
    (1, 24, 8, 5, 300, 64, 2, 32),
    (2, 8, 1, 33, 33, 128, 0, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window", PACKED)
def test_fwd_packed_rows(ta, B, Hq, Hkv, Lq, Lk, d, causal, window):
    """Heads of a kv group stacked in the tile rows, against the oracle."""
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 13 + Lk + d + Hq)
    scale = d ** -0.5
    o, lse = run_fwd(ta, x, causal, window, scale)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window)
    check_o(o, ro, "O")
    check_lse(lse, rl, "LSE")


# (B, Hq, Hkv, Lq, Lk, d, causal, window, n_split); n_split None: the library's choice
SPLIT = [
    (2, 8, 2, 1, 3000, 128, 2, 0, 8),
    (1, 4, 4, 64, 2048, 64, 2, 500, 5),
    (1, 2, 2, 300, 300, 128, 1, 0, 3),
    (1, 2, 1, 17, 5000, 128, 2, 0, None),
    (1, 2, 2, 200, 100, 128, 2, 0, 7),
    (1, 2, 2, 100, 900, 128, 0, 64, 4),
    (1, 2, 2, 50, 700, 128, 0, 0, 64),
    (2, 16, 4, 8, 4000, 128, 2, 0, None),
    (1, 12, 2, 40, 3000, 64, 2, 256, 6),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,n_split", SPLIT)
def test_fwd_split_kv(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, n_split):
    """Split-KV forward (slices merged by their LSE) against the oracle."""
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 5 + Lk + d + 3)
    scale = d ** -0.5
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o, lse = ta.attention_split(q, k, v, causal, window, scale, n_split)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")


# (B, Hq, Hkv, Lq, Lk, d, causal, window, seqlens_q, seqlens_k): padded batches
VARLEN = [
    (3, 4, 2, 300, 300, 128, 1, 0, [300, 129, 0], [300, 129, 0]),
    (3, 2, 2, 257, 400, 128, 2, 0, [1, 100, 257], [400, 37, 256]),
    (2, 4, 4, 200, 200, 64, 0, 0, [200, 77], [150, 200]),
    (2, 2, 1, 500, 500, 128, 1, 64, [500, 333], [500, 333]),
    (2, 2, 2, 300, 300, 128, 0, 50, [300, 128], [10, 300]),
    (3, 8, 2, 16, 600, 128, 2, 0, [16, 5, 0], [600, 17, 300]),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,lq,lk", VARLEN)
def test_fwd_varlen(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, lq, lk):
    """Per-sequence lengths of a padded batch against the oracle (padding rows: O = 0, LSE = -inf)."""
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 11 + Lk + d + 5)
    scale = d ** -0.5
    q, k, v = (to_dev(x[n]) for n in "qkv")
    tq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    tk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    o, lse = ta.attention(q, k, v, causal, window, scale, seqlens_q=tq, seqlens_k=tk)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window, seqlens_q=lq, seqlens_k=lk)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")


# (B, Hq, Hkv, Lq, Lk, d, causal, window, global_head, global_tail)
GLOBAL = [
    (1, 2, 2, 700, 700, 128, 0, 64, 1, 1),
    (1, 4, 2, 1000, 1000, 128, 1, 128, 4, 0),
    (2, 2, 1, 300, 500, 64, 2, 50, 130, 20),
    (1, 2, 2, 257, 257, 128, 0, 8, 0, 3),
    (1, 2, 2, 400, 400, 128, 0, 0, 5, 5),
    (1, 8, 2, 32, 900, 128, 2, 64, 4, 2),
]


# Block-sparse mask ("大模型高效注意力机制全解析" §4.1.2), block size b: blocks below,
# at and above the tile size, with causal (both alignments) and window masks,
# packed short queries, split-KV and global keys on top.
# (B, Hq, Hkv, Lq, Lk, d, causal, window, b, n_split, gh, gt)
SPARSE = [
    (1, 2, 2, 1024, 1024, 128, 0, 0, 64, 1, 0, 0),
    (2, 4, 2, 700, 700, 128, 1, 0, 128, 1, 0, 0),
    (1, 2, 1, 300, 500, 64, 2, 0, 50, 1, 0, 0),
    (1, 2, 2, 513, 513, 128, 0, 100, 200, 1, 0, 0),
    (1, 3, 3, 257, 257, 64, 1, 64, 1, 1, 0, 0),
    (2, 8, 2, 16, 2000, 128, 2, 0, 300, 1, 0, 0),
    (1, 2, 2, 100, 3000, 128, 0, 0, 256, 4, 0, 0),
    (1, 2, 2, 600, 600, 128, 0, 0, 64, 1, 2, 3),
    # Two row tiles per unit (no alternating slots) cut into key-range slices: the
    # slices of a walk that runs downwards.
    (1, 2, 2, 700, 900, 128, 0, 0, 64, 3, 0, 0),
    (2, 4, 4, 520, 520, 64, 1, 0, 100, 2, 0, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,b,ns,gh,gt", SPARSE)
def test_fwd_sparse_block(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, b, ns, gh, gt):
    """Block-sparse forward through attn_fwd_ex against the oracle."""
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 29 + Lk + d + b)
    scale = d ** -0.5
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(256, ta.lib.attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, ns)), dtype=torch.uint8,
                     device="cuda")
    m = ta.AttnMask(ta._causal_code(causal), window, gh, gt, None, None, b)
    st = ta.lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq,
                            Lk, d, scale, ctypes.byref(m), ns, ws.data_ptr(), ws.numel(), None)
    assert st == 0
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window, global_head=gh, global_tail=gt,
                             sparse_block=b)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,gh,gt", GLOBAL)
def test_fwd_global_tokens(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, gh, gt):
    """Global head/tail key positions on top of the window, against the oracle."""
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 17 + Lk + d + gh + 7 * gt)
    scale = d ** -0.5
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o, lse = ta.attention(q, k, v, causal, window, scale, global_head=gh, global_tail=gt)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window, global_head=gh, global_tail=gt)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")


def test_fwd_global_tokens_split_and_varlen(ta):
    """attn_fwd_ex with global tokens, per-sequence lengths and a split key walk at once."""
    import ctypes
    import torch
    B, Hq, Hkv, Lq, Lk, d, w, gh, gt, ns = 2, 4, 2, 100, 2000, 128, 96, 3, 2, 6
    lq, lk = [100, 37], [2000, 1500]
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=99)
    scale = d ** -0.5
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device="cuda")
    tq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    tk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    m = ta.AttnMask(2, w, gh, gt, tq.data_ptr(), tk.data_ptr(), 0)
    ws = torch.empty(ta.lib.attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, ns), dtype=torch.uint8, device="cuda")
    st = ta.lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq,
                            Lk, d, scale, ctypes.byref(m), ns, ws.data_ptr(), ws.numel(),
                            torch.cuda.current_stream().cuda_stream)
    assert st == 0
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, 2, w, seqlens_q=lq, seqlens_k=lk, global_head=gh,
                             global_tail=gt)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")


def test_fwd_no_keys(ta):
    """Lk = 0: every row sees nothing: O = 0, LSE = -inf."""
    import torch
    x = make_shape_inputs(1, 2, 2, 50, 1, 64, seed=5)
    q = to_dev(x["q"])
    k = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = ta.attention(q, k, k, False, 0, 0.125)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_fwd_sharp_softmax_rescales(ta):
    """Large logits (Q scaled by 8) force the lazy rescale path many times per row.

    Far sharper than any benchmark workload, so the max-abs bound is derived
    from the arithmetic instead: P enters P.V rounded to bf16 (relative error
    <= 2^-9 per weight, so <= 2^-9 max|V| on a convex combination) and O is
    rounded to bf16 once more (<= 2^-9 |O| <= 2^-9 max|V|).
    """
    x = make_shape_inputs(1, 2, 2, 1024, 1024, 128, seed=99, q_mult=8.0)
    o, lse = run_fwd(ta, x, True, 0, 128 ** -0.5)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], 128 ** -0.5, True, 0)
    vmax = float(np.max(np.abs(oracle.attention._f64(x["v"]))))
    assert np.max(np.abs(o - ro)) <= 2.0 ** -8 * vmax * 1.05
    from tests._util import rel_fro
    assert rel_fro(o, ro) <= 5e-3
    check_lse(lse, rl, "LSE")


def test_fwd_single_head_128(ta):
    w = WORKLOADS["single_head_128"]
    x = make_inputs(w)
    o, lse = run_fwd(ta, x, w.causal, w.window, w.scale)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window)
    check_o(o, ro, "O")
    check_lse(lse, rl, "LSE")


@pytest.mark.parametrize("name,heads", [
    ("mha_causal_4096", [(0, 0), (1, 31), (0, 17)]),
    ("gqa_causal_8192", [(0, 0), (3, 31), (2, 9)]),
    ("gqa_window_32768", [(0, 0), (0, 21)]),
    ("mha_sparse64_4096", [(0, 0), (1, 31)]),
])
def test_fwd_full_size_sampled_heads(ta, name, heads):
    """Full-size workloads in the benchmark's launch configuration; whole heads
    (independent units) are compared against the oracle."""
    w = WORKLOADS[name]
    x = make_inputs(w)
    o, lse = run_fwd(ta, x, w.causal, w.window, w.scale, w.sparse_block)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window, heads=heads,
                             sparse_block=w.sparse_block)
    for b, h in heads:
        check_o(o[b, h], ro[b, h], f"{name} O[{b},{h}]")
        check_lse(lse[b, h], rl[b, h], f"{name} LSE[{b},{h}]")
    assert np.all(np.isfinite(o))


# More units than SMs (several waves of CTAs): plain, alternating slots (G = 1
# with short queries, and packed GQA rows with sequences of no queries or no
# keys between full ones), split-KV, global keys, d = 64.
# (B, Hq, Hkv, Lq, Lk, d, causal, window, n_split, gh, gt, seqlens_q, seqlens_k)
MANY_UNITS = [
    (4, 32, 32, 300, 300, 128, 1, 0, 1, 0, 0, None, None),
    (8, 40, 40, 100, 700, 64, 2, 0, 1, 0, 0, None, None),
    (24, 32, 8, 16, 600, 128, 2, 0, 1, 0, 0, [16, 0, 5, 16, 0, 0, 9, 16] * 3, [600, 17, 300, 0, 600, 40, 9, 128] * 3),
    (2, 64, 8, 16, 5000, 128, 2, 0, 20, 0, 0, None, None),
    (4, 32, 8, 300, 300, 128, 0, 64, 1, 2, 2, None, None),
    (3, 48, 48, 257, 257, 64, 1, 100, 1, 0, 0, None, None),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,ns,gh,gt,lq,lk", MANY_UNITS)
def test_fwd_many_units(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, ns, gh, gt, lq, lk):
    """Problems with more units than SMs, through attn_fwd_ex, against the oracle."""
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=B * 31 + Hq + Lq + Lk + d)
    scale = d ** -0.5
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(256, ta.lib.attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, ns)), dtype=torch.uint8,
                     device="cuda")
    tq = torch.tensor(lq, dtype=torch.int32, device="cuda") if lq else None
    tk = torch.tensor(lk, dtype=torch.int32, device="cuda") if lk else None
    m = ta.AttnMask(ta._causal_code(causal), window, gh, gt, tq.data_ptr() if lq else None,
                    tk.data_ptr() if lk else None, 0)
    st = ta.lib.attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq,
                            Lk, d, scale, ctypes.byref(m), ns, ws.data_ptr(), ws.numel(), None)
    assert st == 0
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window, global_head=gh, global_tail=gt,
                             seqlens_q=lq, seqlens_k=lk)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")


@pytest.mark.parametrize("split", [False, True])
def test_fwd_decode_full_size(ta, split):
    """gqa_decode_32768 at full size (packed rows; with split=True the split-KV
    launch with the library's default slice count, as timed): sampled heads
    against the oracle."""
    w = WORKLOADS["gqa_decode_32768"]
    x = make_inputs(w)
    q, k, v = (to_dev(x[n]) for n in "qkv")
    if split:
        o, lse = ta.attention_split(q, k, v, w.causal, w.window, w.scale, None)
    else:
        o, lse = ta.attention(q, k, v, w.causal, w.window, w.scale)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    o, lse = to_f64(o), to_f64(lse)
    heads = [(0, 0), (3, 31), (1, 13), (2, 6)]
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window, heads=heads)
    for b, h in heads:
        check_o(o[b, h], ro[b, h], f"decode O[{b},{h}]")
        check_lse(lse[b, h], rl[b, h], f"decode LSE[{b},{h}]")
    assert np.all(np.isfinite(o))


def test_bounded_wait_reports_timeout(ta):
    """A wait that nothing completes gives up and reports ATTN_ERR_TIMEOUT;
    the context stays usable afterwards."""
    assert ta.lib.attn_selftest_wait_timeout(50_000_000, None) == 0
    st, site = ta.device_error()
    assert st == ta.ATTN_ERR_TIMEOUT and site == 1000
    assert ta.device_error()[0] == 0
    x = make_shape_inputs(1, 1, 1, 64, 64, 64, seed=1)
    o, lse = run_fwd(ta, x, True, 0, 0.125)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], 0.125, True, 0)
    check_o(o, ro)

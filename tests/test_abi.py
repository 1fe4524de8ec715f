"""The C-ABI library: loads, exports every declared symbol, validates arguments.

Runs on the CPU: only calls that must fail validation (or are empty) are made,
and those return before touching the GPU.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^ATTN_API\s+[\w\s\*]+?\b(\w+)\(", text, re.M)
    return names


@pytest.fixture(scope="module")
def ta():
    from tiled_exact_attention_02_b200 import build
    build.build()
    import tiled_exact_attention_02_b200 as ta
    return ta


def test_every_declared_symbol_is_exported(ta):
    names = _declared()
    assert {"attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_status_string",
            "attn_get_device_error"} <= set(names)
    lib = ctypes.CDLL(ta.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(ta):
    assert ta.status_string(0) == "ATTN_OK"
    assert ta.status_string(1) == "ATTN_ERR_INVALID_ARG"
    assert ta.status_string(4) == "ATTN_ERR_TIMEOUT"
    assert ta.status_string(77) == "ATTN_ERR_UNKNOWN"


P = 1 << 20  # a 16-byte aligned fake address: never dereferenced, validation fails first


def _fwd(ta, B=1, Hq=2, Hkv=2, Lq=8, Lk=8, d=64, scale=0.125, causal=0, window=0, q=P, k=P, v=P, o=P, lse=P):
    return ta.lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2), (dict(d=256), 2), (dict(Hq=3, Hkv=2), 1), (dict(Hkv=0), 1),
    (dict(B=-1), 1), (dict(Lq=-5), 1), (dict(causal=1, window=-1), 1), (dict(causal=3), 1), (dict(causal=-1), 1),
    (dict(scale=0.0), 1), (dict(scale=-1.0), 1), (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1), (dict(q=0), 1), (dict(o=P + 8), 1), (dict(lse=P + 4), 1),
    (dict(k=0), 1), (dict(v=P + 2), 1),
])
def test_fwd_rejects_bad_arguments(ta, kw, status):
    assert _fwd(ta, **kw) == status


@pytest.mark.parametrize("kw", [dict(B=0), dict(Hq=0, Hkv=0), dict(Lq=0)])
def test_fwd_empty_problem_is_a_no_op(ta, kw):
    assert _fwd(ta, q=0, k=0, v=0, o=0, lse=0, **kw) == 0


def _bwd(ta, B=1, Hq=2, Hkv=1, Lq=8, Lk=8, d=128, scale=0.1, causal=1, window=0, ptrs=None, ws=P, wsb=1 << 20):
    p = ptrs or [P] * 9
    return ta.lib.attn_bwd(*p, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=80), 2), (dict(Hq=3, Hkv=2), 1), (dict(window=-3, causal=0), 1), (dict(causal=3), 1), (dict(ws=0), 1),
    (dict(wsb=16), 1), (dict(ptrs=[P] * 5 + [0] + [P] * 3), 1), (dict(ptrs=[P] * 8 + [P + 1]), 1),
    (dict(scale=0.0), 1), (dict(ws=P + 64), 1),
])
def test_bwd_rejects_bad_arguments(ta, kw, status):
    assert _bwd(ta, **kw) == status


def test_bwd_workspace_size(ta):
    """D (fp32 per query row) and the fp32 dQ accumulator [B*Hq, Lq, d], each padded to 256 bytes."""
    n = ta.bwd_workspace_size(2, 4, 2, 101, 50, 64)
    rows = 2 * 4 * 101
    acc = rows * 64
    assert n == -(-rows * 4 // 256) * 256 + -(-acc * 4 // 256) * 256
    assert ta.bwd_workspace_size(0, 4, 2, 100, 50, 64) == 0
    assert ta.bwd_workspace_size(1, 3, 2, 100, 50, 64) == 0
    assert ta.bwd_workspace_size(1, 4, 2, 100, 50, 72) == 0


def test_fwd_split_workspace_size(ta):
    """n_split x (fp32 O rows x d + fp32 LSE rows), each part padded to 256 bytes; 0 for one slice."""
    ws = ta.lib.attn_fwd_split_workspace_size
    rows = 1 * 2 * 10
    assert ws(1, 2, 2, 10, 300, 64, 4) == -(-4 * rows * 64 * 4 // 256) * 256 + -(-4 * rows * 4 // 256) * 256
    assert ws(1, 2, 2, 10, 300, 64, 1) == 0
    assert ws(1, 2, 2, 10, 300, 64, 0) == 0 and ws(1, 2, 2, 10, 300, 64, 65) == 0
    assert ws(0, 2, 2, 10, 300, 64, 4) == 0


def test_fwd_split_default_is_in_range(ta):
    d = ta.lib.attn_fwd_split_default
    assert d(1, 8, 2, 1, 32768, 128, 2, 0) > 1          # a decode problem splits
    assert 1 <= d(8, 32, 8, 1, 32768, 128, 2, 0) <= 64
    assert d(2, 32, 32, 4096, 4096, 128, 1, 0) == 1     # a full grid does not
    assert d(1, 2, 2, 1, 100, 64, 2, 0) == 1            # a single key tile does not
    # Alternating-slot plans (few query rows per kv group) take the most slices that fit one wave of one CTA
    # per SM (148 SMs, the default without a device).  16 queries per head over 32768 keys, G = 4: 32 packed
    # units -> 4 slices (128 CTAs); 8 units -> 18; 64 units -> 2; 128 units -> 1.
    assert d(4, 32, 8, 16, 32768, 128, 2, 0) == 4
    assert d(1, 32, 8, 1, 32768, 128, 2, 0) == 18
    assert d(8, 32, 8, 16, 32768, 128, 2, 0) == 2
    assert d(16, 32, 8, 1, 4096, 128, 2, 0) == 1
    # ... but never a slice shorter than two key tiles: 8 units over 1024 keys (8 tiles) -> 4.
    assert d(1, 32, 8, 1, 1024, 128, 2, 0) == 4
    # Units with two slots of different rows (128 queries per head, G = 4: 32 units of 256 key tiles) are
    # compute-bound: the modelled waves give 9 slices (288 CTAs, two waves).
    assert d(1, 32, 8, 128, 32768, 128, 2, 0) == 9


def _split(ta, n_split=4, ws=P, wsb=1 << 20, **kw):
    a = dict(B=1, Hq=2, Hkv=2, Lq=8, Lk=300, d=64, scale=0.125, causal=2, window=0)
    a.update(kw)
    return ta.lib.attn_fwd_split(P, P, P, P, P, a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"], a["d"], a["scale"],
                                 a["causal"], a["window"], n_split, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(n_split=0), 1), (dict(n_split=65), 1), (dict(wsb=64), 1), (dict(ws=0), 1), (dict(ws=P + 16), 1),
    (dict(causal=3), 1), (dict(d=80), 2), (dict(Hq=3, Hkv=2), 1),
])
def test_fwd_split_rejects_bad_arguments(ta, kw, status):
    assert _split(ta, **kw) == status


def test_binding_has_no_cpu_path(ta):
    """The binding only marshals: no numpy/torch attention math in the package."""
    src = open(os.path.join(ROOT, "tiled_exact_attention_02_b200", "__init__.py")).read()
    for banned in ("softmax", "oracle", "matmul", "@", "scaled_dot_product"):
        assert banned not in src.replace("@staticmethod", ""), banned


def test_causal_argument_codes(ta):
    """The binding maps the causal argument to the ABI code (0 none, 1 top-left, 2 bottom-right)."""
    f = ta._causal_code
    assert [f(x) for x in (False, True, 0, 1, 2)] == [0, 1, 0, 1, 2]
    assert [f(x) for x in ("none", "top_left", "bottom_right")] == [0, 1, 2]
    with pytest.raises(ValueError):
        f("diagonal")


def test_fwd_ex_and_bwd_ex_validate_the_mask(ta):
    """attn_fwd_ex / attn_bwd_ex: a NULL mask, negative global counts and a bad
    slice count are rejected before any launch."""
    import ctypes
    m = ta.AttnMask(1, 0, -1, 0, None, None, 0)
    args = (P, P, P, P, P, 1, 2, 2, 8, 8, 64, 0.125)
    assert ta.lib.attn_fwd_ex(*args, None, 1, None, 0, None) == 1
    assert ta.lib.attn_fwd_ex(*args, ctypes.byref(m), 1, None, 0, None) == 1
    m.global_head = 0
    assert ta.lib.attn_fwd_ex(*args, ctypes.byref(m), 0, None, 0, None) == 1
    assert ta.lib.attn_fwd_ex(*args, ctypes.byref(m), 4, None, 0, None) == 1  # split needs a workspace
    m.global_tail = -2
    assert ta.lib.attn_bwd_ex(*([P] * 9), 1, 2, 2, 8, 8, 64, 0.125, ctypes.byref(m), P, 1 << 20, None) == 1
    assert ta.lib.attn_bwd_ex(*([P] * 9), 1, 2, 2, 8, 8, 64, 0.125, None, P, 1 << 20, None) == 1
    # Block-sparse block size: negative or above 2^28 is rejected.
    for bad in (-1, (1 << 28) + 1):
        m = ta.AttnMask(1, 0, 0, 0, None, None, bad)
        assert ta.lib.attn_fwd_ex(*args, ctypes.byref(m), 1, None, 0, None) == 1
        assert ta.lib.attn_bwd_ex(*([P] * 9), 1, 2, 2, 8, 8, 64, 0.125, ctypes.byref(m), P, 1 << 20, None) == 1


def test_attn_mask_layout_matches_header(ta):
    """The ctypes mirror of attn_mask has the header's field order and size."""
    import ctypes
    names = [f[0] for f in ta.AttnMask._fields_]
    assert names == ["causal", "window", "global_head", "global_tail", "seqlens_q", "seqlens_k", "sparse_block"]
    assert ctypes.sizeof(ta.AttnMask) == 40


def _host_size(ta, B=2, Hq=8, Hkv=2, Lq=300, Lk=500, d=128, bwd=1):
    return ta.lib.attn_step_host_buffer_size(B, Hq, Hkv, Lq, Lk, d, bwd)


def test_step_host_buffer_size(ta):
    a = lambda x: (x + 255) // 256 * 256
    B, Hq, Hkv, Lq, Lk, d = 2, 8, 2, 300, 500, 128
    nq, nk = B * Hq * Lq * d * 2, B * Hkv * Lk * d * 2
    # One kv head per chunk here (B * Hkv = 4 groups): LSE staged in 4 chunk slots of G * Lq floats each.
    fwd_only = a(nq) + 2 * a(nk) + a(nq) + a(4 * a(Hq // Hkv * Lq * 4))
    assert _host_size(ta, bwd=0) == fwd_only
    # Backward adds dO, dQ, dK, dV and one chunk's workspace.
    ws = ta.lib.attn_bwd_workspace_size(1, Hq // Hkv, 1, Lq, Lk, d)
    assert _host_size(ta, bwd=1) == fwd_only + 2 * a(nq) + 2 * a(nk) + a(ws)
    assert _host_size(ta, d=96) == 0
    assert _host_size(ta, Hq=3) == 0
    assert _host_size(ta, B=0) == 0


def _host(ta, buf=P << 4, nbytes=1 << 40, do=P, q=P, B=1, Hq=2, Hkv=2, Lq=8, Lk=8, d=64, scale=0.125, causal=0,
          window=0):
    return ta.lib.attn_step_host(q, P, P, do, P, P, P, P, P, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, buf,
                                 nbytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2), (dict(Hq=3), 1), (dict(causal=3), 1), (dict(scale=0.0), 1), (dict(window=-1), 1),
    (dict(q=0), 1), (dict(buf=0), 1), (dict(buf=(P << 4) + 16), 1), (dict(nbytes=100), 1),
    (dict(B=0), 0), (dict(Lq=0), 0),
])
def test_step_host_rejects_before_any_copy(ta, kw, status):
    assert _host(ta, **kw) == status


# ------------------------------------------------------------------ ring-attention block calls
def test_accumulate_calls_reject_bad_arguments(ta):
    lib = ta.lib
    ok = dict(B=1, Hq=2, Hkv=1, Lq=8, Lk=8, d=128)
    args = lambda **kw: [dict(ok, **kw)[n] for n in ("B", "Hq", "Hkv", "Lq", "Lk", "d")]
    # attn_fwd_accumulate: missing or misaligned accumulators, bad shapes, bad mask
    assert lib.attn_fwd_accumulate(P, P, P, 0, P, *args(), 0.1, 1, 0, 1, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_accumulate(P, P, P, P, P + 4, *args(), 0.1, 1, 0, 1, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_accumulate(P, P, P, P, P, *args(d=96), 0.1, 1, 0, 1, None) == ta.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fwd_accumulate(P, P, P, P, P, *args(Hq=3, Hkv=2), 0.1, 1, 0, 1, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_accumulate(P, P, P, P, P, *args(), 0.1, 4, 0, 1, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_accumulate(0, 0, 0, P, P, *args(Lq=0), 0.1, 1, 0, 1, None) == ta.ATTN_OK
    # attn_fwd_accumulate_finalize
    assert lib.attn_fwd_accumulate_finalize(P, P, 0, P, 1, 2, 8, 128, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_accumulate_finalize(P, P, P, P, 1, 2, 8, 72, None) == ta.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fwd_accumulate_finalize(0, 0, 0, 0, 0, 2, 8, 128, None) == ta.ATTN_OK
    # attn_bwd_accumulate: accumulators and workspace
    ws = 1 << 20
    assert lib.attn_bwd_accumulate(P, P, P, P, P, 0, P, *args(), 0.1, 1, 0, 1, P, ws, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_accumulate(P, P, P, P, P, P, P + 8, *args(), 0.1, 1, 0, 1, P, ws, None) == \
        ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_accumulate(P, P, P, P, P, P, P, *args(), 0.1, 1, 0, 1, P, 16, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_accumulate(P, P, P, P, P, P, P, *args(), 0.1, 1, 0, 1, 0, ws, None) == ta.ATTN_ERR_INVALID_ARG
    # attn_accumulator_to_bf16
    assert lib.attn_accumulator_to_bf16(P, P, 0, None) == ta.ATTN_OK
    assert lib.attn_accumulator_to_bf16(0, P, 16, None) == ta.ATTN_ERR_INVALID_ARG
    assert lib.attn_accumulator_to_bf16(P + 4, P, 16, None) == ta.ATTN_ERR_INVALID_ARG


def test_step_host_fail_hook_validates(ta):
    assert ta.lib.attn_selftest_step_host_fail_at(-2) == ta.ATTN_ERR_INVALID_ARG
    assert ta.lib.attn_selftest_step_host_fail_at(-1) == ta.ATTN_OK

"""Out-of-bounds write detection without a sanitizer: every output and
workspace buffer handed to the library sits between two guard regions of
seeded random bytes, and after the call (and a device synchronisation) the
guards must be unchanged.  Element-wise parity cannot see a store past the end
of a buffer; these checks can, on the shapes whose row and key offsets the
kernels compute themselves: ragged tails, packed query rows, per-sequence
lengths, split-KV slices, global keys, the block-sparse mask, alternating
slots, both head dimensions, the host-buffer step's staging buffer and the
ring attention accumulators.  The values are checked too (against the oracle)
so a case cannot pass by writing nothing."""

import numpy as np
import pytest

import oracle
from synth import make_shape_inputs
from tests._util import check_grad, check_lse, check_o, to_dev, to_f64

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side (a multiple of 256, so the payload keeps its alignment)


@pytest.fixture(scope="module")
def ta():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_exact_attention_02_b200 as ta
    return ta


class Guarded:
    """A tensor of `shape`/`dtype` inside a larger byte buffer whose guard
    bytes are random; `intact()` compares them with their initial values."""

    def __init__(self, shape, dtype, device="cuda", seed=0):
        import torch
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = nbytes
        rng = np.random.default_rng(seed)
        pattern = torch.from_numpy(rng.integers(0, 256, size=2 * GUARD + nbytes, dtype=np.uint8))
        self.buf = pattern.to(device) if device == "cuda" else pattern.clone().pin_memory()
        self.head = pattern[:GUARD].clone()
        self.tail = pattern[GUARD + nbytes:].clone()
        self.t = self.buf[GUARD:GUARD + nbytes].view(dtype).view(shape) if nbytes else \
            torch.empty(shape, dtype=dtype, device=device)

    def intact(self):
        import torch
        torch.cuda.synchronize()
        b = self.buf.cpu()
        return torch.equal(b[:GUARD], self.head) and torch.equal(b[GUARD + self.nbytes:], self.tail)


def _guarded_outputs(q, k, seed):
    import torch
    B, Hq, Lq, d = q.shape
    o = Guarded(tuple(q.shape), torch.bfloat16, seed=seed)
    lse = Guarded((B, Hq, Lq), torch.float32, seed=seed + 1)
    return o, lse


# (B, Hq, Hkv, Lq, Lk, d, causal, window, extra)
FWD_CASES = [
    (1, 2, 2, 7, 7, 128, 1, 0, {}),
    (2, 3, 3, 129, 129, 64, 1, 0, {}),                        # odd G = 1, two tiles: alternating slots off
    (1, 3, 1, 100, 333, 128, 0, 0, {}),                       # G = 3, one tile: alternating slots
    (3, 8, 2, 16, 1000, 128, 2, 0, {}),                       # packed rows (decode)
    (2, 8, 2, 40, 700, 64, 2, 64, {}),                        # packed rows across heads, window
    (2, 4, 2, 333, 333, 128, 1, 0, {"seqlens": ([333, 200], [333, 150])}),
    (1, 4, 2, 500, 500, 128, 0, 64, {"global": (3, 2)}),
    (2, 2, 2, 300, 300, 128, 0, 0, {"sparse": 64}),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,extra", FWD_CASES)
def test_forward_writes_stay_inside_o_and_lse(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, extra):
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq + Lk + d + 31)
    q, k, v = (to_dev(x[n]) for n in "qkv")
    scale = d ** -0.5
    o, lse = _guarded_outputs(q, k, Lq)
    kw, okw = {}, {}
    if "seqlens" in extra:
        lq, lk = extra["seqlens"]
        kw = dict(seqlens_q=torch.tensor(lq, dtype=torch.int32, device="cuda"),
                  seqlens_k=torch.tensor(lk, dtype=torch.int32, device="cuda"))
        okw = dict(seqlens_q=lq, seqlens_k=lk)
    if "global" in extra:
        kw = dict(global_head=extra["global"][0], global_tail=extra["global"][1])
        okw = dict(kw)
    if "sparse" in extra:
        kw = okw = dict(sparse_block=extra["sparse"])
    ta.fwd(q, k, v, o.t, lse.t, causal, window, scale, **kw)
    assert ta.device_error()[0] == 0
    assert o.intact() and lse.intact(), "a forward store left O or LSE"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window, **okw)
    check_o(to_f64(o.t), ro, "O")
    check_lse(to_f64(lse.t), rl, "LSE")


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,n_split",
                         [(4, 8, 2, 16, 3000, 128, 2, 0, 9), (1, 2, 2, 333, 2000, 64, 0, 0, 5),
                          (2, 4, 4, 129, 1500, 128, 2, 100, 3)])
def test_split_forward_writes_stay_inside_workspace(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, n_split):
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq + n_split)
    q, k, v = (to_dev(x[n]) for n in "qkv")
    scale = d ** -0.5
    o, lse = _guarded_outputs(q, k, 5)
    ws = Guarded((int(ta.lib.attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, n_split)),), torch.uint8, seed=9)
    ta.fwd_split(q, k, v, o.t, lse.t, n_split, ws.t, causal, window, scale)
    assert ta.device_error()[0] == 0
    assert o.intact() and lse.intact() and ws.intact()
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window)
    check_o(to_f64(o.t), ro, "O")
    check_lse(to_f64(lse.t), rl, "LSE")


BWD_CASES = [
    (1, 2, 2, 7, 7, 128, 1, 0, {}),
    (2, 4, 2, 200, 333, 64, 0, 0, {}),
    (1, 8, 2, 257, 257, 128, 1, 64, {}),
    (1, 4, 2, 16, 700, 128, 2, 0, {}),
    (3, 4, 2, 300, 300, 128, 1, 0, {"seqlens": ([300, 129, 1], [300, 129, 7])}),
    (1, 2, 2, 400, 400, 128, 0, 50, {"global": (2, 3)}),
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,d,causal,window,extra", BWD_CASES)
def test_backward_writes_stay_inside_gradients_and_workspace(ta, B, Hq, Hkv, Lq, Lk, d, causal, window, extra):
    import torch
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=Lq * 5 + Lk + d, with_do=True)
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    scale = d ** -0.5
    kw, okw = {}, {}
    if "seqlens" in extra:
        lq, lk = extra["seqlens"]
        kw = dict(seqlens_q=torch.tensor(lq, dtype=torch.int32, device="cuda"),
                  seqlens_k=torch.tensor(lk, dtype=torch.int32, device="cuda"))
        okw = dict(seqlens_q=lq, seqlens_k=lk)
    if "global" in extra:
        kw = dict(global_head=extra["global"][0], global_tail=extra["global"][1])
        okw = dict(kw)
    o, lse = ta.attention(q, k, v, causal, window, scale, **kw)
    dq = Guarded(tuple(q.shape), torch.bfloat16, seed=1)
    dk = Guarded(tuple(k.shape), torch.bfloat16, seed=2)
    dv = Guarded(tuple(v.shape), torch.bfloat16, seed=3)
    ws = Guarded((ta.bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d),), torch.uint8, seed=4)
    ta.bwd(q, k, v, o, lse, do, dq.t, dk.t, dv.t, ws.t, causal, window, scale, **kw)
    assert ta.device_error()[0] == 0
    for name, g in (("dQ", dq), ("dK", dk), ("dV", dv), ("workspace", ws)):
        assert g.intact(), f"a backward store left {name}"
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window, **okw)
    check_grad(to_f64(dq.t), rq, "dQ")
    check_grad(to_f64(dk.t), rk, "dK")
    check_grad(to_f64(dv.t), rv, "dV")


def test_host_step_writes_stay_inside_staging_and_host_outputs(ta):
    import torch
    B, Hq, Hkv, Lq, Lk, d, causal = 2, 6, 3, 130, 270, 128, 2
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=12, with_do=True)
    host = {n: torch.from_numpy(np.ascontiguousarray(x[n]).view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v", "do")}
    o = Guarded((B, Hq, Lq, d), torch.bfloat16, device="cpu", seed=21)
    lse = Guarded((B, Hq, Lq), torch.float32, device="cpu", seed=22)
    dq = Guarded((B, Hq, Lq, d), torch.bfloat16, device="cpu", seed=23)
    dk = Guarded((B, Hkv, Lk, d), torch.bfloat16, device="cpu", seed=24)
    dv = Guarded((B, Hkv, Lk, d), torch.bfloat16, device="cpu", seed=25)
    buf = Guarded((ta.step_host_buffer_size(B, Hq, Hkv, Lq, Lk, d, True),), torch.uint8, seed=26)
    ta.step_host(host["q"], host["k"], host["v"], o.t, lse.t, buf.t, do=host["do"], dq=dq.t, dk=dk.t, dv=dv.t,
                 causal=causal, scale=d ** -0.5)
    torch.cuda.synchronize()
    assert ta.device_error()[0] == 0
    for name, g in (("O", o), ("LSE", lse), ("dQ", dq), ("dK", dk), ("dV", dv), ("staging buffer", buf)):
        assert g.intact(), f"the host-buffer step wrote outside {name}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], d ** -0.5, causal, 0)
    check_o(to_f64(o.t), ro, "O")
    check_lse(to_f64(lse.t), rl, "LSE")


def test_ring_accumulators_stay_inside(ta):
    import torch
    from tiled_exact_attention_02_b200 import ring
    ops = ring.CudaOps(ta.lib)
    B, Hq, Hkv, L, d = 1, 4, 2, 200, 128  # 200-row chunks: ragged tiles
    x = make_shape_inputs(B, Hq, Hkv, L, 2 * L, d, seed=8, with_do=True)
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    scale = d ** -0.5
    o_acc = Guarded(tuple(q.shape), torch.float32, seed=31)
    lse_acc = Guarded(tuple(q.shape[:-1]), torch.float32, seed=32)
    for i in range(2):
        kk, vv = k[:, :, i * L:(i + 1) * L].contiguous(), v[:, :, i * L:(i + 1) * L].contiguous()
        ops.fwd_acc(q, kk, vv, o_acc.t, lse_acc.t, 0 if i == 0 else 1, i == 0, scale)
    assert o_acc.intact() and lse_acc.intact()
    o, lse = torch.empty_like(q), torch.empty(q.shape[:-1], dtype=torch.float32, device="cuda")
    ops.fwd_finalize(o_acc.t, lse_acc.t, o, lse)
    ws = ops.bwd_workspace(q, k)
    ops.bwd_pre(o, do, ws)
    dk_acc = Guarded((B, Hkv, L, d), torch.float32, seed=33)
    dv_acc = Guarded((B, Hkv, L, d), torch.float32, seed=34)
    kk, vv = k[:, :, L:].contiguous(), v[:, :, L:].contiguous()
    ops.bwd_acc(q, kk, vv, lse, do, dk_acc.t, dv_acc.t, ws, 1, True, scale)
    out = Guarded((B, Hkv, L, d), torch.bfloat16, seed=35)
    ops.to_bf16(dk_acc.t, out.t)
    assert ta.device_error()[0] == 0
    assert dk_acc.intact() and dv_acc.intact() and out.intact()
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, 2, 0)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")
    assert torch.equal(out.t, dk_acc.t.to(torch.bfloat16))

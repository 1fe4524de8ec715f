"""Ring (context-parallel) attention.

CPU, world sizes 2-4 over gloo (the exchange and the schedule):
  * every (query chunk, key chunk) block that the mask leaves visible is
    computed exactly once over all ranks, on the K/V data that actually
    arrived from the right rank, and the dK/dV accumulators come home having
    visited every rank whose queries see their block;
  * with float64 stand-ins for the block kernels (the oracle for the forward
    block, the textbook gradient with the global LSE for the backward block),
    the distributed forward and backward equal the oracle on the whole
    sequence.
GPU (one device; every rank's steps run in ring order in one process, which
is what the ring computes, without the exchange): the block kernels behind
the C ABI against the float64 oracle on the whole sequence, world 2, 4, 8,
both layouts, causal and not, GQA, d = 64 and 128.
"""

import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle  # noqa: E402
from synth import bf16_bits_to_f32, make_shape_inputs  # noqa: E402
from tests._util import check_grad, check_lse, check_o, to_dev, to_f64  # noqa: E402


def _ring():
    from tiled_exact_attention_02_b200 import ring
    return ring


# ------------------------------------------------------------------ schedule (host only)
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_covers_every_visible_block_once(world, layout, causal):
    ring = _ring()
    seen = {}
    for r in range(world):
        mine = ring.chunks_of_rank(r, world, layout)
        for t, (src, blocks) in enumerate(ring.schedule(r, world, layout, causal)):
            assert src == (r - t) % world
            theirs = ring.chunks_of_rank(src, world, layout)
            for qi, ki, m in blocks:
                key = (mine[qi], theirs[ki])
                assert key not in seen
                seen[key] = m
    n = ring.n_chunks(world, layout)
    want = {(a, b): (1 if a == b and causal else 0) for a in range(n) for b in range(n) if not causal or b <= a}
    assert seen == want


def test_zigzag_balances_causal_work():
    ring = _ring()
    world = 8
    # Work of a step in units of one full block (the diagonal block is half).
    for t in range(world):
        loads = {sum(0.5 if m == 1 else 1.0 for *_, m in ring.schedule(r, world, "zigzag", True)[t][1])
                 for r in range(world)}
        assert len(loads) == 1


def test_shard_roundtrip():
    ring = _ring()
    x = torch.arange(2 * 3 * 48 * 4, dtype=torch.float64).reshape(2, 3, 48, 4)
    for layout in ring.LAYOUTS:
        for world in (1, 2, 3):
            parts = [ring.shard(x, r, world, layout) for r in range(world)]
            assert torch.equal(ring.unshard(parts, world, layout), x)


# ------------------------------------------------------------------ float64 stand-ins (test only)
class F64Ops:
    """Block compute in float64 on CPU tensors, for the distributed tests.

    Forward block: the oracle on (q, k, v) with the block's mask, merged into
    the running (O, LSE) with the logsumexp rescale.  Backward block: the
    textbook softmax gradient with the final LSE and D of the query rows."""

    def empty_f32(self, shape, like):
        return torch.empty(shape, dtype=torch.float64)

    def empty_like(self, x):
        return torch.empty_like(x)

    def fwd_acc(self, q, k, v, o_acc, lse_acc, mask, init, scale):
        ob, lb = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), scale, mask, 0)
        ob, lb = torch.from_numpy(ob), torch.from_numpy(lb)
        if init:
            o_acc.copy_(ob)
            lse_acc.copy_(lb)
            return
        m = torch.maximum(lse_acc, lb)
        m = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
        wa, wb = torch.exp(lse_acc - m), torch.exp(lb - m)
        s = wa + wb
        o_acc.copy_(torch.where(s[..., None] > 0, (o_acc * wa[..., None] + ob * wb[..., None]) / s[..., None], 0.0))
        lse_acc.copy_(torch.where(s > 0, m + torch.log(s), torch.full_like(s, -np.inf)))

    def fwd_finalize(self, o_acc, lse_acc, o, lse):
        o.copy_(o_acc)
        lse.copy_(lse_acc)

    def bwd_workspace(self, q, k):
        return {}

    def bwd_pre(self, o, do, ws):
        ws["D"] = (o * do).sum(-1)
        ws["dq"] = torch.zeros_like(o)

    def bwd_acc(self, q, k, v, lse, do, dk_acc, dv_acc, ws, mask, init, scale):
        G = q.shape[1] // k.shape[1]
        kk, vv = k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
        S = scale * q @ kk.transpose(-1, -2)
        if mask == 1:
            Lq, Lk = S.shape[-2:]
            vis = torch.ones(Lq, Lk, dtype=torch.bool).tril()
            S = S.masked_fill(~vis, -np.inf)
        P = torch.exp(S - lse[..., None])
        dP = do @ vv.transpose(-1, -2)
        dS = P * (dP - ws["D"][..., None])
        ws["dq"] += scale * dS @ kk
        dk = (scale * dS.transpose(-1, -2) @ q).unflatten(1, (k.shape[1], G)).sum(2)
        dv = (P.transpose(-1, -2) @ do).unflatten(1, (k.shape[1], G)).sum(2)
        if init:
            dk_acc.copy_(dk)
            dv_acc.copy_(dv)
        else:
            dk_acc += dk
            dv_acc += dv

    def bwd_finalize(self, dq, ws, scale):
        dq.copy_(ws["dq"])

    def to_bf16(self, acc, out):
        out.copy_(acc)


class TraceOps(F64Ops):
    """Records which global chunks each block combined; the K/V and query
    tensors carry their global chunk index in every element."""

    def __init__(self):
        self.fwd_blocks, self.bwd_blocks = [], []

    def fwd_acc(self, q, k, v, o_acc, lse_acc, mask, init, scale):
        self.fwd_blocks.append((int(q.flatten()[0]), int(k.flatten()[0]), int(v.flatten()[0]), mask, bool(init)))
        if init:
            o_acc.zero_()

    def bwd_acc(self, q, k, v, lse, do, dk_acc, dv_acc, ws, mask, init, scale):
        qc, kc = int(q.flatten()[0]), int(k.flatten()[0])
        self.bwd_blocks.append((qc, kc, mask))
        # Each visit adds a bit that names the query chunk, so the accumulator
        # that comes home lists every query chunk that saw its block.
        if init:
            dk_acc.zero_()
            dv_acc.zero_()
        dk_acc += float(2 ** qc)
        dv_acc += float(kc)  # stays a multiple of the block's own chunk index

    def bwd_pre(self, o, do, ws):
        ws["D"] = torch.zeros(o.shape[:-1], dtype=torch.float64)
        ws["dq"] = torch.zeros_like(o)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))


def _trace_worker(rank, world, port, layout, causal, out):
    _init(rank, world, port)
    ring = _ring()
    n = ring.n_chunks(world, layout)
    full = torch.arange(n, dtype=torch.float64).repeat_interleave(4)[None, None, :, None].expand(1, 2, 4 * n, 3)
    q, k, v = (ring.shard(full.contiguous(), rank, world, layout) for _ in range(3))
    ops = TraceOps()
    ring.ring_attention_forward(q, k, v, layout=layout, causal=causal, ops=ops)
    o = torch.zeros_like(q)
    lse = torch.zeros(q.shape[:-1], dtype=torch.float64)
    dq, dk, dv = ring.ring_attention_backward(q, k, v, o, lse, q, layout=layout, causal=causal, ops=ops)
    out[rank] = (ops.fwd_blocks, ops.bwd_blocks, dk[:, 0, 0, 0, 0].tolist(), dv[:, 0, 0, 0, 0].tolist(),
                 ring.chunks_of_rank(rank, world, layout))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal", [(2, "zigzag", True), (3, "contiguous", True), (4, "zigzag", True),
                                                 (3, "zigzag", False), (2, "contiguous", False)])
def test_ring_exchange_delivers_the_right_blocks(world, layout, causal):
    ring = _ring()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_trace_worker, args=(world, _free_port(), layout, causal, out), nprocs=world,
                       start_method="spawn", join=True)
    n = ring.n_chunks(world, layout)
    want = {(a, b) for a in range(n) for b in range(n) if not causal or b <= a}
    fwd, bwd = [], []
    for r in range(world):
        fb, bb, dk, dv, mine = out[r]
        for qc, kc, vc, m, _ in fb:
            assert kc == vc and m == (1 if qc == kc and causal else 0)
        fwd += [(qc, kc) for qc, kc, *_ in fb]
        bwd += [(qc, kc) for qc, kc, _ in bb]
        # dK/dV accumulators of this rank's chunks came home with one bit per
        # query chunk that sees them.
        for i, c in enumerate(mine):
            assert dk[i] == sum(2.0 ** a for a in range(n) if (a, c) in want)
            assert dv[i] == c * sum(1 for a in range(n) if (a, c) in want)
    assert sorted(fwd) == sorted(want) and sorted(bwd) == sorted(want)


def _numeric_worker(rank, world, port, layout, causal, Hq, Hkv, out):
    _init(rank, world, port)
    ring = _ring()
    L, d = 12 * ring.n_chunks(world, layout), 8
    x = make_shape_inputs(1, Hq, Hkv, L, L, d, seed=5 + world, with_do=True)
    full = {n: torch.from_numpy(bf16_bits_to_f32(x[n]).astype(np.float64)) for n in ("q", "k", "v", "do")}
    q, k, v, do = (ring.shard(full[n], rank, world, layout) for n in ("q", "k", "v", "do"))
    ops = F64Ops()
    scale = d ** -0.5
    o, lse = ring.ring_attention_forward(q, k, v, layout=layout, causal=causal, scale=scale, ops=ops)
    dq, dk, dv = ring.ring_attention_backward(q, k, v, o, lse, do, layout=layout, causal=causal, scale=scale, ops=ops)
    out[rank] = tuple(t.numpy() for t in (o, lse, dq, dk, dv))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal,Hq,Hkv", [(2, "zigzag", True, 2, 1), (3, "contiguous", True, 2, 2),
                                                        (3, "zigzag", False, 4, 2), (4, "zigzag", True, 2, 2)])
def test_ring_forward_backward_match_the_oracle_on_gloo_ranks(world, layout, causal, Hq, Hkv):
    ring = _ring()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_numeric_worker, args=(world, _free_port(), layout, causal, Hq, Hkv, out), nprocs=world,
                       start_method="spawn", join=True)
    L, d = 12 * ring.n_chunks(world, layout), 8
    x = make_shape_inputs(1, Hq, Hkv, L, L, d, seed=5 + world, with_do=True)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], d ** -0.5, causal, 0)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], d ** -0.5, causal, 0)
    got = [ring.unshard([torch.from_numpy(out[r][i]) for r in range(world)], world, layout).numpy()
           for i in range(5)]
    for g, r in zip(got, (ro, rl, rq, rk, rv)):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------------ GPU: the block kernels, ring order on one device
def _serial_ring(ta, x, world, layout, causal, scale):
    """Every rank's steps in ring order (t outer, ranks inner): rank r at step
    t works on the K/V chunks of rank r - t, and the dK/dV accumulators of a
    rank's chunks are shared by whoever holds them, as the exchange would."""
    ring = _ring()
    full = {n: to_dev(x[n]) for n in ("q", "k", "v", "do")}
    sh = {n: [ring.shard(full[n], r, world, layout) for r in range(world)] for n in full}
    ops = ring.CudaOps(ta.lib)
    fw = [ring.RingForwardRank(sh["q"][r], r, world, layout, causal, scale, ops) for r in range(world)]
    for t in range(world):
        for r in range(world):
            src = (r - t) % world
            fw[r].step(t, sh["k"][src], sh["v"][src])
    res = [f.result() for f in fw]
    o = ring.unshard([a for a, _ in res], world, layout)
    lse = ring.unshard([b for _, b in res], world, layout)
    bw = [ring.RingBackwardRank(sh["q"][r], res[r][0], res[r][1], sh["do"][r], r, world, layout, causal, scale, ops,
                                k_like=sh["k"][r]) for r in range(world)]
    acc = [[torch.empty(sh["k"][r].shape, dtype=torch.float32, device="cuda") for _ in range(2)] for r in range(world)]
    for t in range(world):
        for r in range(world):
            src = (r - t) % world
            bw[r].step(t, sh["k"][src], sh["v"][src], acc[src][0], acc[src][1])
    dqs = [b.dq() for b in bw]
    dks, dvs = [], []
    for r in range(world):
        dk, dv = torch.empty_like(sh["k"][r]), torch.empty_like(sh["v"][r])
        ops.to_bf16(acc[r][0], dk)
        ops.to_bf16(acc[r][1], dv)
        dks.append(dk)
        dvs.append(dv)
    torch.cuda.synchronize()
    return o, lse, ring.unshard(dqs, world, layout), ring.unshard(dks, world, layout), ring.unshard(dvs, world,
                                                                                                     layout)


RING_CASES = [
    (1, 4, 2, 1024, 128, 2, "zigzag", True),
    (1, 4, 2, 1024, 128, 4, "zigzag", True),
    (1, 4, 2, 1024, 128, 8, "zigzag", True),
    (1, 4, 4, 1024, 128, 4, "contiguous", True),
    (2, 2, 2, 768, 64, 3, "contiguous", False),
    (1, 8, 1, 1536, 128, 4, "zigzag", False),
    (1, 2, 2, 4096, 128, 8, "contiguous", True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hkv,L,d,world,layout,causal", RING_CASES)
def test_ring_blocks_on_gpu_match_the_oracle(B, Hq, Hkv, L, d, world, layout, causal):
    import tiled_exact_attention_02_b200 as ta
    x = make_shape_inputs(B, Hq, Hkv, L, L, d, seed=L + world + d, with_do=True)
    scale = d ** -0.5
    o, lse, dq, dk, dv = _serial_ring(ta, x, world, layout, causal, scale)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, 0)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, 0)
    check_grad(to_f64(dq), rq, "dQ")
    check_grad(to_f64(dk), rk, "dK")
    check_grad(to_f64(dv), rv, "dV")


@pytest.mark.gpu
def test_accumulate_entry_points_match_the_whole_problem():
    """Keys cut into three blocks (the first two before every query, the last
    the diagonal block): the merged accumulators equal attn_fwd on the whole
    problem up to rounding, and dK/dV accumulated per block equal attn_bwd."""
    import tiled_exact_attention_02_b200 as ta
    ring = _ring()
    ops = ring.CudaOps(ta.lib)
    B, Hq, Hkv, Lc, d = 1, 4, 2, 256, 128
    x = make_shape_inputs(B, Hq, Hkv, Lc, 3 * Lc, d, seed=77, with_do=True)
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    scale = d ** -0.5
    o_acc = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse_acc = torch.empty(q.shape[:-1], dtype=torch.float32, device="cuda")
    blocks = [(0, 0), (1, 0), (2, 2)]  # (key block, C-ABI mask): causal = 2 aligns q with the last block
    for i, (kb, m) in enumerate(blocks):
        kk, vv = k[:, :, kb * Lc:(kb + 1) * Lc].contiguous(), v[:, :, kb * Lc:(kb + 1) * Lc].contiguous()
        ops.fwd_acc(q, kk, vv, o_acc, lse_acc, m, i == 0, scale)
    o, lse = torch.empty_like(q), torch.empty(q.shape[:-1], dtype=torch.float32, device="cuda")
    ops.fwd_finalize(o_acc, lse_acc, o, lse)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, 2, 0)
    check_o(to_f64(o), ro, "O")
    check_lse(to_f64(lse), rl, "LSE")
    ws = ops.bwd_workspace(q, k)
    ops.bwd_pre(o, do, ws)
    dk_acc = torch.empty(k[:, :, :Lc].shape, dtype=torch.float32, device="cuda")
    dv_acc = torch.empty_like(dk_acc)
    dks, dvs = [], []
    for kb, m in blocks:
        kk, vv = k[:, :, kb * Lc:(kb + 1) * Lc].contiguous(), v[:, :, kb * Lc:(kb + 1) * Lc].contiguous()
        ops.bwd_acc(q, kk, vv, lse, do, dk_acc, dv_acc, ws, m, True, scale)
        ops.bwd_acc(q, kk, vv, lse, do, dk_acc, dv_acc, ws, m, False, scale)  # added twice: 2x the block
        dks.append(dk_acc.clone() / 2)
        dvs.append(dv_acc.clone() / 2)
    dq = torch.empty_like(q)
    ops.bwd_finalize(dq, ws, scale)
    torch.cuda.synchronize()
    assert ta.device_error()[0] == 0
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, 2, 0)
    check_grad(to_f64(dq) / 2, rq, "dQ")  # every block's dQ was added twice
    check_grad(np.concatenate([d.double().cpu().numpy() for d in dks], axis=2), rk, "dK")
    check_grad(np.concatenate([d.double().cpu().numpy() for d in dvs], axis=2), rv, "dV")


def test_single_process_ring_needs_no_process_group():
    """Without torch.distributed initialised the ring has one rank: its one
    step is the whole problem (float64 stand-ins, against the oracle)."""
    ring = _ring()
    x = make_shape_inputs(1, 2, 1, 40, 40, 8, seed=3, with_do=True)
    full = {n: torch.from_numpy(bf16_bits_to_f32(x[n]).astype(np.float64)) for n in ("q", "k", "v", "do")}
    q, k, v, do = (ring.shard(full[n], 0, 1, "zigzag") for n in ("q", "k", "v", "do"))
    ops = F64Ops()
    o, lse = ring.ring_attention_forward(q, k, v, causal=True, scale=8 ** -0.5, ops=ops)
    dq, dk, dv = ring.ring_attention_backward(q, k, v, o, lse, do, causal=True, scale=8 ** -0.5, ops=ops)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], 8 ** -0.5, True, 0)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], 8 ** -0.5, True, 0)
    for g, r in zip((o, lse, dq, dk, dv), (ro, rl, rq, rk, rv)):
        np.testing.assert_allclose(ring.unshard([g], 1, "zigzag").numpy(), r, rtol=1e-10, atol=1e-12)

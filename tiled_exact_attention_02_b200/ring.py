"""Ring (context-parallel) attention over a torch.distributed process group.

"缩放定律与高效注意力" §5.1 (the table of three directions) names RingAttention
and LongFlashAttention as the way to longer contexts: sequence parallelism on
top of FlashAttention.  Here the sequence of every (batch, head) is cut into
equal chunks spread over the ranks of a group.  Each rank keeps its query
chunks; the key/value chunks travel around the ring (rank r sends to r + 1
and receives from r - 1), and at step t rank r holds the K/V chunks of rank
r - t.  Against each K/V block it runs the block-wise kernels of the C ABI:

  forward   attn_fwd_accumulate merges the block's attention into running fp32
            (O, LSE) accumulators (the online-softmax rescale of "高效注意力：
            FlashAttention 与线性注意力", 原理与机制, applied to whole blocks),
            attn_fwd_accumulate_finalize rounds them at the end;
  backward  attn_bwd_preprocess (D from the final O, zeroed dQ accumulator),
            attn_bwd_accumulate per block with the final LSE (dQ added into the
            local accumulator, the block's dK / dV added into fp32
            accumulators that travel with the block and arrive back at their
            owner after the last step), attn_bwd_finalize and
            attn_accumulator_to_bf16.

Layouts (how the global sequence is cut):
  contiguous  rank r holds chunk r of `world` chunks;
  zigzag      rank r holds chunks r and 2*world - 1 - r of 2*world chunks, so
              that under a causal mask every rank has the same work per step
              (a plain reading of "sequence parallelism" would be the
              contiguous cut; zigzag is the load-balanced one).
A rank's tensors are [C, B, H, Lc, d] (C = 1 or 2 chunks of Lc positions),
each chunk a contiguous [B, H, Lc, d] tensor.  Masks: causal (top-left over
the global positions) or none.  Between two chunks of equal length the
causal mask is either nothing (key chunk before the query chunk), the
diagonal block (the same chunk: causal = 1 of the C ABI), or everything
(key chunk after: the block is skipped).

Communication: K/V of the next step are exchanged with batched isend/irecv
while the current step computes; the dK/dV accumulators move after the
step's compute (they are its output).  Over NCCL the transfers go by NVLink
between the GPUs of a node.  Remote data is always received into local
memory before a kernel reads it.

The compute goes through an `ops` object: `CudaOps` (the default) calls the
C ABI; tests may pass another implementation with the same methods to check
the schedule and exchange on CPU ranks.
"""

from __future__ import annotations

import math

LAYOUTS = ("contiguous", "zigzag")


def chunks_of_rank(rank: int, world: int, layout: str) -> tuple:
    """Global chunk indices held by `rank`, in local order."""
    if layout == "contiguous":
        return (rank,)
    if layout == "zigzag":
        return (rank, 2 * world - 1 - rank)
    raise ValueError(f"layout must be one of {LAYOUTS}, got {layout!r}")


def n_chunks(world: int, layout: str) -> int:
    return world * len(chunks_of_rank(0, world, layout))


def block_mask(q_chunk: int, k_chunk: int, causal: bool):
    """C-ABI mask code of the block (query chunk, key chunk), chunks of equal
    length in global order: 0 every key visible, 1 the diagonal block, None
    no key visible (skipped)."""
    if not causal or k_chunk < q_chunk:
        return 0
    if k_chunk == q_chunk:
        return 1
    return None


def schedule(rank: int, world: int, layout: str, causal: bool) -> list:
    """For each ring step t: (source rank of the K/V chunks held at step t,
    [(local query chunk, local key chunk, mask code), ...])."""
    mine = chunks_of_rank(rank, world, layout)
    steps = []
    for t in range(world):
        src = (rank - t) % world
        theirs = chunks_of_rank(src, world, layout)
        blocks = []
        for qi, qc in enumerate(mine):
            for ki, kc in enumerate(theirs):
                m = block_mask(qc, kc, causal)
                if m is not None:
                    blocks.append((qi, ki, m))
        steps.append((src, blocks))
    # Every K/V chunk meets a query chunk of its own rank at step 0 (the
    # diagonal block, or any block without a causal mask), which initialises
    # its dK / dV accumulators before they travel.
    assert {ki for _, ki, _ in steps[0][1]} == set(range(len(mine)))
    return steps


def shard(x, rank: int, world: int, layout: str, seq_dim: int = 2):
    """This rank's chunks of a full tensor (sequence along `seq_dim`), stacked
    as [C, ...] with each chunk contiguous."""
    import torch
    n = n_chunks(world, layout)
    L = x.shape[seq_dim]
    if L % n:
        raise ValueError(f"sequence length {L} is not a multiple of {n} chunks")
    lc = L // n
    parts = [x.narrow(seq_dim, c * lc, lc) for c in chunks_of_rank(rank, world, layout)]
    return torch.stack(parts).contiguous()


def unshard(shards, world: int, layout: str, seq_dim: int = 2):
    """Inverse of `shard`: shards[r] is rank r's [C, ...] tensor."""
    import torch
    n = n_chunks(world, layout)
    order = [None] * n
    for r in range(world):
        for i, c in enumerate(chunks_of_rank(r, world, layout)):
            order[c] = shards[r][i]
    return torch.cat(order, dim=seq_dim)


class CudaOps:
    """Block compute through the C ABI (libtiledattn.so); torch only
    allocates device memory and supplies the current stream."""

    def __init__(self, lib=None):
        if lib is None:
            from . import lib
        self.lib = lib

    @staticmethod
    def _sp():
        import torch
        return torch.cuda.current_stream().cuda_stream

    def _check(self, st, what):
        from . import AttnError
        if st != 0:
            raise AttnError(st, what)

    def empty_f32(self, shape, like):
        import torch
        return torch.empty(shape, dtype=torch.float32, device=like.device)

    def empty_like(self, x):
        import torch
        return torch.empty_like(x)

    def fwd_acc(self, q, k, v, o_acc, lse_acc, mask, init, scale):
        B, Hq, Lq, d = q.shape
        Hkv, Lk = k.shape[1], k.shape[2]
        self._check(self.lib.attn_fwd_accumulate(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_acc.data_ptr(),
                                                 lse_acc.data_ptr(), B, Hq, Hkv, Lq, Lk, d, scale, mask, 0,
                                                 int(bool(init)), self._sp()), "attn_fwd_accumulate")

    def fwd_finalize(self, o_acc, lse_acc, o, lse):
        B, Hq, Lq, d = o.shape
        self._check(self.lib.attn_fwd_accumulate_finalize(o_acc.data_ptr(), lse_acc.data_ptr(), o.data_ptr(),
                                                          lse.data_ptr(), B, Hq, Lq, d, self._sp()),
                    "attn_fwd_accumulate_finalize")

    def bwd_workspace(self, q, k):
        import torch
        B, Hq, Lq, d = q.shape
        n = int(self.lib.attn_bwd_workspace_size(B, Hq, k.shape[1], Lq, k.shape[2], d))
        return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)

    def bwd_pre(self, o, do, ws):
        B, Hq, Lq, d = o.shape
        self._check(self.lib.attn_bwd_preprocess(o.data_ptr(), do.data_ptr(), B, Hq, Lq, d, ws.data_ptr(),
                                                 ws.numel(), self._sp()), "attn_bwd_preprocess")

    def bwd_acc(self, q, k, v, lse, do, dk_acc, dv_acc, ws, mask, init, scale):
        B, Hq, Lq, d = q.shape
        Hkv, Lk = k.shape[1], k.shape[2]
        self._check(self.lib.attn_bwd_accumulate(q.data_ptr(), k.data_ptr(), v.data_ptr(), lse.data_ptr(),
                                                 do.data_ptr(), dk_acc.data_ptr(), dv_acc.data_ptr(), B, Hq, Hkv,
                                                 Lq, Lk, d, scale, mask, 0, int(bool(init)), ws.data_ptr(),
                                                 ws.numel(), self._sp()), "attn_bwd_accumulate")

    def bwd_finalize(self, dq, ws, scale):
        B, Hq, Lq, d = dq.shape
        self._check(self.lib.attn_bwd_finalize(dq.data_ptr(), B, Hq, Lq, d, scale, ws.data_ptr(), ws.numel(),
                                               self._sp()), "attn_bwd_finalize")

    def to_bf16(self, acc, out):
        self._check(self.lib.attn_accumulator_to_bf16(acc.data_ptr(), out.data_ptr(), acc.numel(), self._sp()),
                    "attn_accumulator_to_bf16")


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


class RingForwardRank:
    """One rank's forward state: its query chunks and the running (O, LSE)
    accumulators, fed one K/V block per ring step."""

    def __init__(self, q, rank, world, layout="zigzag", causal=True, scale=None, ops=None):
        self.ops = ops or CudaOps()
        self.q = q
        self.scale = _scale(scale, q.shape[-1])
        self.steps = schedule(rank, world, layout, causal)
        self.o_acc = self.ops.empty_f32(tuple(q.shape), q)
        self.lse_acc = self.ops.empty_f32(tuple(q.shape[:-1]), q)
        self.fresh = [True] * q.shape[0]

    def step(self, t, k, v):
        """k, v: the [C, B, Hkv, Lc, d] chunks of rank steps[t][0]."""
        for qi, ki, mask in self.steps[t][1]:
            self.ops.fwd_acc(self.q[qi], k[ki], v[ki], self.o_acc[qi], self.lse_acc[qi], mask, self.fresh[qi],
                             self.scale)
            self.fresh[qi] = False

    def result(self):
        assert not any(self.fresh), "a query chunk met no key block"
        o = self.ops.empty_like(self.q)
        lse = self.ops.empty_f32(tuple(self.q.shape[:-1]), self.q)
        for c in range(self.q.shape[0]):
            self.ops.fwd_finalize(self.o_acc[c], self.lse_acc[c], o[c], lse[c])
        return o, lse


class RingBackwardRank:
    """One rank's backward state: D and the dQ accumulator of its query
    chunks; each step adds a K/V block's dK / dV into the accumulators that
    travel with that block."""

    def __init__(self, q, o, lse, do, rank, world, layout="zigzag", causal=True, scale=None, ops=None, k_like=None):
        self.ops = ops or CudaOps()
        self.q, self.lse, self.do = q, lse, do
        self.scale = _scale(scale, q.shape[-1])
        self.steps = schedule(rank, world, layout, causal)
        kl = k_like if k_like is not None else q
        self.ws = [self.ops.bwd_workspace(q[c], kl[0]) for c in range(q.shape[0])]
        for c in range(q.shape[0]):
            self.ops.bwd_pre(o[c], do[c], self.ws[c])

    def step(self, t, k, v, dk_acc, dv_acc):
        """k, v: the K/V chunks of rank steps[t][0]; dk_acc, dv_acc: their fp32
        accumulators (initialised at step 0 by their owner)."""
        for qi, ki, mask in self.steps[t][1]:
            self.ops.bwd_acc(self.q[qi], k[ki], v[ki], self.lse[qi], self.do[qi], dk_acc[ki], dv_acc[ki],
                             self.ws[qi], mask, t == 0 and self._first_use(ki, qi), self.scale)

    def _first_use(self, ki, qi):
        # At step 0 the first block of each local key chunk initialises its accumulators.
        for q2, k2, _ in self.steps[0][1]:
            if k2 == ki:
                return q2 == qi
        return False

    def dq(self):
        dq = self.ops.empty_like(self.q)
        for c in range(self.q.shape[0]):
            self.ops.bwd_finalize(dq[c], self.ws[c], self.scale)
        return dq


def _ring_peers(group):
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return 0, 1, 0, 0  # a single process: the ring has one rank and no exchange
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    g = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    return rank, world, g((rank + 1) % world), g((rank - 1) % world)


def _exchange(tensors, group, nxt, prv, ops):
    """Start sending `tensors` to the next rank and receiving the previous
    rank's into fresh buffers; returns (requests, received)."""
    import torch.distributed as dist
    recv = [ops.empty_like(x) for x in tensors]
    p2p = [dist.P2POp(dist.isend, x, nxt, group) for x in tensors]
    p2p += [dist.P2POp(dist.irecv, r, prv, group) for r in recv]
    return dist.batch_isend_irecv(p2p), recv


def ring_attention_forward(q, k, v, group=None, layout="zigzag", causal=True, scale=None, ops=None):
    """Forward of ring attention on this rank's chunks: q [C, B, Hq, Lc, d],
    k, v [C, B, Hkv, Lc, d] (bf16 CUDA tensors for CudaOps).  Returns this
    rank's O [C, B, Hq, Lc, d] and LSE [C, B, Hq, Lc] (fp32, natural log)."""
    ops = ops or CudaOps()
    rank, world, nxt, prv = _ring_peers(group)
    st = RingForwardRank(q, rank, world, layout, causal, scale, ops)
    cur = [k, v]
    for t in range(world):
        pending = _exchange(cur, group, nxt, prv, ops) if t + 1 < world else None
        st.step(t, *cur)
        if pending is not None:
            reqs, cur = pending
            for r in reqs:
                r.wait()
    return st.result()


def ring_attention_backward(q, k, v, o, lse, do, group=None, layout="zigzag", causal=True, scale=None, ops=None):
    """Backward of ring attention on this rank's chunks, from the forward's O
    and LSE: returns dQ, dK, dV of this rank's chunks (bf16 for CudaOps)."""
    ops = ops or CudaOps()
    rank, world, nxt, prv = _ring_peers(group)
    st = RingBackwardRank(q, o, lse, do, rank, world, layout, causal, scale, ops, k_like=k)
    cur = [k, v]
    acc = [ops.empty_f32(tuple(k.shape), k), ops.empty_f32(tuple(v.shape), v)]
    for t in range(world):
        pending = _exchange(cur, group, nxt, prv, ops) if t + 1 < world else None
        st.step(t, cur[0], cur[1], acc[0], acc[1])
        # The accumulators move on with their block; after the last step they
        # arrive back at the rank that owns the block.
        if world > 1:
            reqs, acc = _exchange(acc, group, nxt, prv, ops)
            for r in reqs:
                r.wait()
        if pending is not None:
            reqs, cur = pending
            for r in reqs:
                r.wait()
    dq = st.dq()
    dk, dv = ops.empty_like(k), ops.empty_like(v)
    ops.to_bf16(acc[0], dk)
    ops.to_bf16(acc[1], dv)
    return dq, dk, dv

"""Seeded synthetic inputs shared by the tests and the benchmark.

This module holds no attention arithmetic.  It only names the workloads and
draws their inputs: i.i.d. standard-normal float32 samples from numpy's PCG64
generator, rounded to bfloat16 (round-to-nearest-even).  Both the CUDA path and
the float64 oracle receive exactly these bfloat16 values; the oracle upcasts
them exactly.

Workloads (the pages measure on no public dataset; these shapes follow the
LLaMA-7B-sized attention the pages discuss in "缩放定律与高效注意力" §2.1 and
§3.5, the GQA head counts of "高效注意力" §3, and the sliding window of the
Mistral example on the same page):

  single_head_128   B=1, H=1,        L=128,   d=64,  non-causal
  mha_causal_4096   B=2, Hq=Hkv=32,  L=4096,  d=128, causal
  gqa_causal_8192   B=4, Hq=32/Hkv=8, L=8192, d=128, causal, Q scaled by 2
  gqa_window_32768  B=1, Hq=32/Hkv=8, L=32768, d=128, causal window 4096
  mha_causal_fwdbwd B=2, Hq=Hkv=32,  L=4096,  d=128, causal, plus dO
  gqa_decode_32768  B=4, Hq=32/Hkv=8, Lq=16 over Lk=32768, d=128, bottom-right
                    causal (new queries over a long cache, the KV-cache
                    setting of "高效注意力" §3)
  mha_sparse64_4096 B=2, Hq=Hkv=32,  L=4096,  d=128, block-sparse mask with
                    64 x 64 blocks (the block size of the example in
                    "大模型高效注意力机制全解析" §4.1.2), no causal mask
"""

from dataclasses import dataclass, field
import math

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    d: int
    causal: int              # 0 none, 1 top-left (j <= i), 2 bottom-right (j <= i + Lk - Lq)
    window: int = 0          # 0: no window; >0: causal band of w keys, or |i - j| < w without causal
    q_mult: float = 1.0      # applied after bf16 rounding (a power of two: exact)
    backward: bool = False
    seed: int = 42
    sparse_block: int = 0    # block-sparse mask block size (0: none)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def visible_pairs_per_head(self) -> int:
        """Number of (i, j) pairs with key j visible to query i."""
        off = self.Lk - self.Lq if self.causal == 2 else 0
        total = 0
        for i in range(self.Lq):
            if self.causal:
                hi = min(i + off + 1, self.Lk)
            else:
                hi = min(i + self.window, self.Lk) if self.window > 0 else self.Lk
            lo = max(0, i + off - self.window + 1) if self.window > 0 else 0
            if self.sparse_block > 0:
                s = i // self.sparse_block * self.sparse_block
                lo = max(lo, s - self.sparse_block)
                hi = min(hi, s + 2 * self.sparse_block - 1)
            total += max(0, hi - lo)
        return total

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 2 GEMMs of 2*d flops per visible pair."""
        return 4.0 * self.d * self.visible_pairs_per_head() * self.B * self.Hq

    def bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: 5 GEMMs (QK^T recompute, dV, dP, dQ, dK)."""
        return 2.5 * self.fwd_flops()


WORKLOADS = {
    w.name: w
    for w in [
        Workload("single_head_128", 1, 1, 1, 128, 128, 64, False, seed=42),
        Workload("mha_causal_4096", 2, 32, 32, 4096, 4096, 128, True, seed=43),
        Workload("gqa_causal_8192", 4, 32, 8, 8192, 8192, 128, True, q_mult=2.0, seed=44),
        Workload("gqa_window_32768", 1, 32, 8, 32768, 32768, 128, True, window=4096, seed=45),
        Workload("mha_causal_fwdbwd", 2, 32, 32, 4096, 4096, 128, True, backward=True, seed=46),
        # 16 new queries per sequence over a 32768-key cache (bottom-right causal)
        Workload("gqa_decode_32768", 4, 32, 8, 16, 32768, 128, 2, seed=47),
        Workload("mha_sparse64_4096", 2, 32, 32, 4096, 4096, 128, 0, seed=48, sparse_block=64),
    ]
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _draw(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw Q, K, V (and dO when the workload has a backward) as bf16 bits.

    Draw order is Q, K, V, dO from one PCG64 stream.  A q_mult other than 1 is
    a power of two, applied to the bf16 values (it only shifts exponents).
    Returns uint16 arrays of shape [B, H, L, d].
    """
    rng = np.random.default_rng(w.seed if seed is None else seed)
    q = _draw(rng, (w.B, w.Hq, w.Lq, w.d))
    k = _draw(rng, (w.B, w.Hkv, w.Lk, w.d))
    v = _draw(rng, (w.B, w.Hkv, w.Lk, w.d))
    if w.q_mult != 1.0:
        m = math.frexp(w.q_mult)
        assert m[0] == 0.5, "q_mult must be a power of two"
        q = f32_to_bf16_bits(bf16_bits_to_f32(q) * np.float32(w.q_mult))
    out = {"q": q, "k": k, "v": v}
    if w.backward:
        out["do"] = _draw(rng, (w.B, w.Hq, w.Lq, w.d))
    return out


def make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed, with_do=False, q_mult=1.0) -> dict:
    """Same recipe as make_inputs for an ad-hoc shape (edge-case tests)."""
    w = Workload("adhoc", B, Hq, Hkv, Lq, Lk, d, False, q_mult=q_mult,
                 backward=with_do, seed=seed)
    return make_inputs(w)

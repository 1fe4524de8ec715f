"""Seeded random problems, forward and backward, against the oracle.

Each case draws its shape and mask from a fixed seed: batch 1-3, group size
1-8, query and key lengths 1-700 (equal or not), d = 64 or 128, causal
alignment none / top-left / bottom-right, an optional window, optional
global keys or block-sparse mask, and optional per-sequence lengths.  The
draws are plain numpy from the case index, so a failure names a reproducible
problem.  Tolerances are those of the other parity tests, with the O max-abs
bound max(1e-2, 2^-8 max|V|) (see tests/_util.py o_maxabs_bound): random
shapes reach rows of few keys with |V| near 3, where the bf16 rounding of P
and of O alone can pass 1e-2.
"""

import numpy as np
import pytest

import oracle
from synth import bf16_bits_to_f32, make_shape_inputs
from tests._util import check_grad, check_lse, check_o, to_dev, to_f64

pytestmark = pytest.mark.gpu

N_CASES = 40


def draw(i):
    rng = np.random.default_rng(1000 + i)
    B = int(rng.integers(1, 4))
    G = int(rng.choice([1, 2, 3, 4, 8]))
    Hkv = int(rng.integers(1, 3))
    Hq = G * Hkv
    Lq = int(rng.integers(1, 701))
    Lk = Lq if rng.random() < 0.5 else int(rng.integers(1, 701))
    d = int(rng.choice([64, 128]))
    causal = int(rng.choice([0, 1, 2]))
    window = int(rng.integers(1, 400)) if rng.random() < 0.35 else 0
    extra = {}
    r = rng.random()
    if r < 0.15:
        extra = dict(global_head=int(rng.integers(0, 5)), global_tail=int(rng.integers(0, 5)))
    elif r < 0.3:
        extra = dict(sparse_block=int(rng.choice([1, 16, 64, 100, 128, 300])))
    elif r < 0.45:
        extra = dict(seqlens_q=[int(rng.integers(0, Lq + 1)) for _ in range(B)],
                     seqlens_k=[int(rng.integers(0, Lk + 1)) for _ in range(B)])
    return B, Hq, Hkv, Lq, Lk, d, causal, window, extra


@pytest.fixture(scope="module")
def ta():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import tiled_exact_attention_02_b200 as ta
    return ta


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_problem(ta, i):
    import torch
    B, Hq, Hkv, Lq, Lk, d, causal, window, extra = draw(i)
    x = make_shape_inputs(B, Hq, Hkv, Lq, Lk, d, seed=5000 + i, with_do=True)
    scale = d ** -0.5
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    kw = dict(extra)
    if "seqlens_q" in kw:
        kw["seqlens_q"] = torch.tensor(kw["seqlens_q"], dtype=torch.int32, device="cuda")
        kw["seqlens_k"] = torch.tensor(kw["seqlens_k"], dtype=torch.int32, device="cuda")
    o, lse = ta.attention(q, k, v, causal, window, scale, **kw)
    dq, dk, dv = ta.attention_backward(q, k, v, o, lse, do, causal, window, scale, **kw)
    st, site = ta.device_error()
    assert st == 0, f"device error {st} at site {site}"
    what = f"case {i}: B={B} Hq={Hq} Hkv={Hkv} Lq={Lq} Lk={Lk} d={d} causal={causal} window={window} {extra}"
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], scale, causal, window, **extra)
    vmax = float(np.max(np.abs(bf16_bits_to_f32(x["v"])))) if x["v"].size else 0.0
    check_o(to_f64(o), ro, what + " O", vmax=vmax)
    check_lse(to_f64(lse), rl, what + " LSE")
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, window, **extra)
    check_grad(to_f64(dq), rq, what + " dQ")
    check_grad(to_f64(dk), rk, what + " dK")
    check_grad(to_f64(dv), rv, what + " dV")

"""The O max-abs bound, checked on the CPU against the arithmetic it covers.

The forward's P enters P.V in bf16 and O leaves the kernel in bf16.  Done
exactly in float64 and rounded at just those two places, a causal head of
310 rows (d = 64, the seeded random-problem case 16) is already 1.024e-2 away
from the float64 definition: more than the flat 1e-2, within
o_maxabs_bound(max|V|) = max(1e-2, 2^-8 max|V|).  The rounding emulated here
is test code; the definition is the oracle's."""

import numpy as np

import oracle
from synth import bf16_bits_to_f32, f32_to_bf16_bits, make_shape_inputs
from tests._util import o_maxabs_bound


def _bf16(x):
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def test_bf16_p_and_o_alone_can_exceed_1e2_but_not_the_bound():
    B, Hq, Hkv, L, d = 2, 4, 2, 310, 64
    x = make_shape_inputs(B, Hq, Hkv, L, L, d, seed=5016, with_do=True)
    q, k, v = (bf16_bits_to_f32(x[n]).astype(np.float64) for n in "qkv")
    ref, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], d ** -0.5, True, 0)
    worst = 0.0
    vis = np.tril(np.ones((L, L), dtype=bool))
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            S = np.where(vis, q[b, h] @ k[b, g].T * d ** -0.5, -np.inf)
            p = np.exp(S - S.max(axis=1, keepdims=True))
            o = _bf16((_bf16(p) @ v[b, g]) / p.sum(axis=1, keepdims=True))
            worst = max(worst, float(np.abs(o - ref[b, h]).max()))
    vmax = float(np.abs(v).max())
    assert worst > 1e-2
    assert worst <= o_maxabs_bound(vmax)
    assert o_maxabs_bound(None) == 1e-2 and o_maxabs_bound(1.0) == 1e-2

"""The forward kernel's FMA-pipe exponential, checked on the CPU.

The kernel evaluates part of its 2^x values as 2^n * p(f) with n = round(x),
f = x - n in [-1/2, 1/2], p a degree-4 polynomial (Remez fit of 2^f, see
csrc/gen_exp2_poly.py) evaluated by Horner's rule with fused multiply-adds,
and 2^n applied by adding n to the exponent field.  This test re-evaluates
exactly that float32 recipe (each fused multiply-add rounded once, via a
float64 product-sum) and bounds its error against 2^x; it also checks that
the coefficients in the CUDA source are the generator's output.
"""

import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_exact_attention_02_b200", "csrc")
MAGIC = np.float32(12582912.0)  # 1.5 * 2^23


def source_coefficients():
    text = open(os.path.join(CSRC, "attn_fwd.cu")).read()
    cs = [np.float32(float(v)) for _, v in sorted(re.findall(r"EXP2_C(\d) = ([0-9.eE+-]+)f;", text))]
    assert len(cs) == 5
    return cs


def f32_fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def kernel_exp2(x, cs):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + MAGIC).astype(np.float32)
    n = (t - MAGIC).astype(np.float32)
    f = f32_fma(n, np.float32(-1.0), x)  # x - n
    p = f32_fma(np.full_like(f, cs[4]), f, np.full_like(f, cs[3]))
    for c in (cs[2], cs[1], cs[0]):
        p = f32_fma(p, f, np.full_like(f, c))
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_source_coefficients_match_generator():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "gen_exp2_poly.py"), "4"], capture_output=True,
                         text=True, check=True).stdout
    gen = [np.float32(float(v)) for v in re.findall(r"= ([0-9.eE+-]+)f;", out)]
    assert gen == source_coefficients()


def test_relative_error_bound():
    cs = source_coefficients()
    x = np.concatenate([np.linspace(-30.0, 8.0, 2_000_001, dtype=np.float32),
                        np.random.default_rng(0).uniform(-120, 8, 1_000_000).astype(np.float32)])
    got = kernel_exp2(x, cs).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 4e-6, rel.max()


def test_special_points():
    cs = source_coefficients()
    x = np.array([0.0, 1.0, -1.0, 8.0, 0.5, -0.5, -126.0], dtype=np.float32)
    got = kernel_exp2(x, cs)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=4e-6)
    # the clamp keeps very negative arguments finite and non-negative
    tiny = kernel_exp2(np.array([-1000.0, -127.0, -126.5], dtype=np.float32), cs)
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 2e-38)

"""The gradient checker itself (CPU): it must pass gradients that carry only
bf16-sized rounding noise and fail a single wrong row of a full-size head,
which the whole-tensor relative Frobenius bound alone cannot see (one zeroed
row of a 4096-row head moves that error by only about 1/64).

The reference gradients are the oracle's for one causal head of the fwd+bwd
workload's shape (L = 4096, d = 128); the planted mistakes are made here, in
copies of the oracle's output, never in the CUDA path."""

import numpy as np
import pytest

import oracle
from synth import make_shape_inputs
from tests._util import check_grad, rel_fro


@pytest.fixture(scope="module")
def grads():
    x = make_shape_inputs(1, 1, 1, 4096, 4096, 128, seed=46, with_do=True)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], 128 ** -0.5, True, 0)
    return {"dQ": rq[0, 0], "dK": rk[0, 0], "dV": rv[0, 0]}


def _noisy(ref, seed):
    # Element-wise relative noise of the size of a bf16 rounding (2^-9).
    rng = np.random.default_rng(seed)
    return ref * (1.0 + 2.0 ** -9 * rng.uniform(-1.0, 1.0, size=ref.shape))


@pytest.mark.parametrize("name", ["dQ", "dK", "dV"])
def test_rounding_noise_passes(grads, name):
    ref = grads[name]
    check_grad(_noisy(ref, 1), ref, name)


@pytest.mark.parametrize("name", ["dQ", "dK", "dV"])
@pytest.mark.parametrize("slip", ["zero_row", "negated_row", "scaled_row", "swapped_rows"])
def test_one_wrong_row_fails(grads, name, slip):
    ref = grads[name]
    got = _noisy(ref, 2)
    n = np.linalg.norm(ref, axis=1)
    r = int(np.argsort(n)[len(n) // 2])  # a row of median norm
    if slip == "zero_row":
        got[r] = 0.0
    elif slip == "negated_row":
        got[r] = -got[r]
    elif slip == "scaled_row":
        got[r] *= 1.1
    else:
        got[[r, r + 1]] = got[[r + 1, r]]
    if slip == "zero_row":
        # The whole-tensor bound alone would let this through.
        assert rel_fro(got, ref) <= 2e-2
    with pytest.raises(AssertionError):
        check_grad(got, ref, name)

"""Pins for the float64 oracle, checked against facts the pages and mathematics fix.

Every test here runs on the CPU.  Each pin is chosen so that a plausible slip
in the oracle (a dropped mask, a wrong sign, a transposed operand, a missing
scale, a wrong GQA head mapping) makes at least one of them fail; the last
group of tests plants such slips and checks that.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as oa
from synth import make_shape_inputs, bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(2024)


def _rand(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------- worked example
def test_golden_hand_worked_example():
    """Hand-derived 3x3 example (fixture cites the definition it follows)."""
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_3x3.json")))
    q = np.array(g["q"], float)[None, None]
    k = np.array(g["k"], float)[None, None]
    v = np.array(g["v"], float)[None, None]
    for case in g["cases"]:
        O, lse = oracle.attn_fwd(q, k, v, g["scale"], case["causal"], case["window"])
        np.testing.assert_allclose(O[0, 0], np.array(case["O"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, 0], np.array(case["LSE"]), rtol=0, atol=1e-14)
    bw = g["backward"]
    dq, dk, dv = oracle.attn_bwd(q, k, v, np.array(bw["dO"], float)[None, None],
                                 g["scale"], bw["causal"], bw["window"])
    np.testing.assert_allclose(dq[0, 0], bw["dQ"], atol=1e-14)
    np.testing.assert_allclose(dk[0, 0], bw["dK"], atol=1e-14)
    np.testing.assert_allclose(dv[0, 0], bw["dV"], atol=1e-14)


# ---------------------------------------------------------------- invariants
MASKS = [(False, 0), (True, 0), (True, 5), (True, 1), (True, 64), (False, 5), (False, 1)]


@pytest.mark.parametrize("causal,window", MASKS)
def test_rows_sum_to_one_masked_exact_zero(causal, window):
    """Each row of A sums to 1; invisible entries are exactly 0 (-inf logit)."""
    Lq, Lk, d = 37, 37, 8
    q, k = _rand(Lq, d), _rand(Lk, d)
    vis = oracle.visible_mask(Lq, Lk, causal, window)
    A, _ = oracle.attention_weights(q, k, 0.7, vis)
    np.testing.assert_allclose(A.sum(1), 1.0, atol=1e-14)
    assert np.all(A[~vis] == 0.0)
    assert np.all(A[vis] > 0.0)


def test_visible_mask_definition():
    """Causal: j <= i.  Window w: i - w < j <= i (w keys including self)."""
    vis = oracle.visible_mask(6, 6, True, 3)
    for i in range(6):
        assert list(np.nonzero(vis[i])[0]) == list(range(max(0, i - 2), i + 1))
    assert oracle.visible_mask(4, 4, False, 0).all()
    assert (oracle.visible_mask(5, 5, True, 0) == np.tril(np.ones((5, 5), bool))).all()


@pytest.mark.parametrize("causal,window", MASKS)
def test_output_in_convex_hull(causal, window):
    """Output row i is a convex combination of the visible V rows."""
    Lq = Lk = 29
    d = 6
    q, k, v = _rand(1, 1, Lq, d), _rand(1, 1, Lk, d), _rand(1, 1, Lk, d)
    O, _ = oracle.attn_fwd(q, k, v, 0.4, causal, window)
    vis = oracle.visible_mask(Lq, Lk, causal, window)
    for i in range(Lq):
        vv = v[0, 0][vis[i]]
        assert np.all(O[0, 0, i] <= vv.max(0) + 1e-12)
        assert np.all(O[0, 0, i] >= vv.min(0) - 1e-12)


@pytest.mark.parametrize("causal,window", MASKS)
def test_zero_query_gives_mean_of_visible(causal, window):
    """Q = 0: all visible logits equal, so O_i is the mean of visible V and LSE = ln(count)."""
    Lq = Lk = 23
    d = 5
    q = np.zeros((1, 1, Lq, d))
    k, v = _rand(1, 1, Lk, d), _rand(1, 1, Lk, d)
    O, lse = oracle.attn_fwd(q, k, v, 1.3, causal, window)
    vis = oracle.visible_mask(Lq, Lk, causal, window)
    for i in range(Lq):
        np.testing.assert_allclose(O[0, 0, i], v[0, 0][vis[i]].mean(0), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(vis[i].sum())) < 1e-14


def test_single_visible_key_returns_that_row():
    """Causal row 0 and window w=1 each see one key: O_i = V_j exactly, LSE = S_ij."""
    L, d = 11, 7
    q, k, v = _rand(1, 1, L, d), _rand(1, 1, L, d), _rand(1, 1, L, d)
    O, lse = oracle.attn_fwd(q, k, v, 0.3, True, 0)
    assert np.array_equal(O[0, 0, 0], v[0, 0, 0])
    assert abs(lse[0, 0, 0] - 0.3 * q[0, 0, 0] @ k[0, 0, 0]) < 1e-14
    O, lse = oracle.attn_fwd(q, k, v, 0.3, True, 1)
    assert np.array_equal(O[0, 0], v[0, 0])
    np.testing.assert_allclose(lse[0, 0], 0.3 * np.sum(q[0, 0] * k[0, 0], 1), atol=1e-14)


def test_two_sided_window_w1_is_the_diagonal():
    """Without causal, window 1 leaves each row its own key only: O = V, LSE = S_ii."""
    L, d = 9, 5
    q, k, v = _rand(1, 1, L, d), _rand(1, 1, L, d), _rand(1, 1, L, d)
    O, lse = oracle.attn_fwd(q, k, v, 0.7, False, 1)
    assert np.array_equal(O[0, 0], v[0, 0])
    np.testing.assert_allclose(lse[0, 0], 0.7 * np.sum(q[0, 0] * k[0, 0], 1), atol=1e-14)


def test_two_sided_window_counts_and_band():
    """Two-sided window w: row i sees min(i, w-1) keys before it, itself, and
    min(L-1-i, w-1) after it; the row-block band covers every visible column."""
    L, w = 23, 4
    vis = oracle.visible_mask(L, L, False, w)
    for i in range(L):
        assert vis[i].sum() == min(i, w - 1) + 1 + min(L - 1 - i, w - 1)
        assert vis[i, i] and not vis[i, max(0, i - w)] or i - w < 0
    for r0 in range(0, L, 5):
        r1 = min(L, r0 + 5)
        lo, hi = oracle.visible_band(r0, r1, L, False, w)
        cols = np.flatnonzero(vis[r0:r1].any(0))
        assert lo == cols.min() and hi == cols.max() + 1


def test_bottom_right_causal_equals_top_left_when_square():
    """causal = 2 aligns the last query with the last key; with Lq = Lk that is causal = 1."""
    L, d = 13, 4
    q, k, v = _rand(1, 2, L, d), _rand(1, 2, L, d), _rand(1, 2, L, d)
    for w in (0, 5):
        a = oracle.attn_fwd(q, k, v, 0.4, 1, w)
        b = oracle.attn_fwd(q, k, v, 0.4, 2, w)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_bottom_right_causal_is_a_suffix_of_the_square_case():
    """Queries Q over keys K with causal = 2 give the last Lq rows of causal = 1
    attention of [P; Q] over K, whatever the prefix rows P (the queries sit at
    positions Lk - Lq .. Lk - 1)."""
    Lq, Lk, d = 5, 17, 6
    q, k, v = _rand(1, 1, Lq, d), _rand(1, 1, Lk, d), _rand(1, 1, Lk, d)
    pre = _rand(1, 1, Lk - Lq, d)
    full = np.concatenate([pre, q], 2)
    for w in (0, 3, 40):
        O, lse = oracle.attn_fwd(q, k, v, 0.3, 2, w)
        Of, lf = oracle.attn_fwd(full, k, v, 0.3, 1, w)
        np.testing.assert_allclose(O, Of[:, :, Lk - Lq:], atol=1e-14)
        np.testing.assert_allclose(lse, lf[:, :, Lk - Lq:], atol=1e-14)


def test_bottom_right_single_query_sees_every_key():
    """A single query aligned to the last key sees the whole cache (no window)."""
    Lk, d = 21, 5
    q, k, v = _rand(1, 1, 1, d), _rand(1, 1, Lk, d), _rand(1, 1, Lk, d)
    np.testing.assert_allclose(oracle.attn_fwd(q, k, v, 0.5, 2, 0)[0], oracle.attn_fwd(q, k, v, 0.5, False, 0)[0],
                               atol=1e-14)


def test_bottom_right_with_more_queries_than_keys():
    """Lq > Lk with causal = 2: the first Lq - Lk rows see no key (O = 0, LSE = -inf, dQ = 0)."""
    Lq, Lk, d = 9, 4, 3
    q, k, v, do = _rand(1, 1, Lq, d), _rand(1, 1, Lk, d), _rand(1, 1, Lk, d), _rand(1, 1, Lq, d)
    O, lse = oracle.attn_fwd(q, k, v, 0.5, 2, 0)
    assert np.all(O[0, 0, :Lq - Lk] == 0) and np.all(np.isneginf(lse[0, 0, :Lq - Lk]))
    assert np.all(np.isfinite(lse[0, 0, Lq - Lk:]))
    dq, _, _ = oracle.attn_bwd(q, k, v, do, 0.5, 2, 0)
    assert np.all(dq[0, 0, :Lq - Lk] == 0)


def test_padded_batch_equals_separate_sequences():
    """Per-sequence lengths: each sequence of a padded batch is its own problem
    (evaluated here on the sliced arrays), padding rows are O = 0, LSE = -inf,
    and the padding's contents change nothing."""
    B, Hq, Hkv, Lq, Lk, d = 3, 4, 2, 11, 13, 5
    q, k, v, do = _rand(B, Hq, Lq, d), _rand(B, Hkv, Lk, d), _rand(B, Hkv, Lk, d), _rand(B, Hq, Lq, d)
    lq, lk = [11, 4, 0], [13, 9, 6]
    for causal, w in ((False, 0), (True, 0), (2, 0), (2, 3), (False, 3)):
        O, lse = oracle.attn_fwd(q, k, v, 0.4, causal, w, seqlens_q=lq, seqlens_k=lk)
        dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.4, causal, w, seqlens_q=lq, seqlens_k=lk)
        for b in range(B):
            sl = slice(b, b + 1)
            Ob, lb = oracle.attn_fwd(q[sl, :, :lq[b]], k[sl, :, :lk[b]], v[sl, :, :lk[b]], 0.4, causal, w)
            np.testing.assert_array_equal(O[b, :, :lq[b]], Ob[0])
            np.testing.assert_array_equal(lse[b, :, :lq[b]], lb[0])
            assert np.all(O[b, :, lq[b]:] == 0) and np.all(np.isneginf(lse[b, :, lq[b]:]))
            gb = oracle.attn_bwd(q[sl, :, :lq[b]], k[sl, :, :lk[b]], v[sl, :, :lk[b]], do[sl, :, :lq[b]], 0.4, causal, w)
            np.testing.assert_array_equal(dq[b, :, :lq[b]], gb[0][0])
            np.testing.assert_array_equal(dk[b, :, :lk[b]], gb[1][0])
            assert np.all(dq[b, :, lq[b]:] == 0) and np.all(dk[b, :, lk[b]:] == 0) and np.all(dv[b, :, lk[b]:] == 0)
        # garbage in the padding changes nothing
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        q2[1, :, 4:] = 1e3
        k2[1, :, 9:] = -7e2
        v2[2, :, 6:] = np.nan
        O2, l2 = oracle.attn_fwd(q2, k2, v2, 0.4, causal, w, seqlens_q=lq, seqlens_k=lk)
        np.testing.assert_array_equal(O2, O)
        np.testing.assert_array_equal(l2, lse)


def test_padded_batch_sequence_without_keys():
    """A sequence with queries but no keys (seqlens_k = 0): every one of its
    rows is fully masked, so O = 0 and LSE = -inf (no NaN); the other
    sequences are unaffected."""
    q, k, v = _rand(2, 2, 6, 4), _rand(2, 2, 9, 4), _rand(2, 2, 9, 4)
    O, lse = oracle.attn_fwd(q, k, v, 0.5, 2, 0, seqlens_q=[6, 4], seqlens_k=[9, 0])
    assert np.all(O[1] == 0.0) and np.all(np.isneginf(lse[1]))
    O0, lse0 = oracle.attn_fwd(q[:1], k[:1], v[:1], 0.5, 2, 0)
    np.testing.assert_array_equal(O[0], O0[0])
    np.testing.assert_array_equal(lse[0], lse0[0])
    dq, dk, dv = oracle.attn_bwd(q, k, v, _rand(2, 2, 6, 4), 0.5, 2, 0, seqlens_q=[6, 4], seqlens_k=[9, 0])
    assert np.all(dq[1] == 0.0) and np.all(dk[1] == 0.0) and np.all(dv[1] == 0.0)


def test_padded_batch_matches_torch_sdpa_key_padding_mask():
    """Per-sequence key lengths against torch SDPA with a key-padding mask built here."""
    B, H, L, d = 2, 2, 10, 4
    q, k, v = _rand(B, H, L, d), _rand(B, H, L, d), _rand(B, H, L, d)
    lk = [10, 6]
    O, _ = oracle.attn_fwd(q, k, v, 0.5, False, 0, seqlens_k=lk)
    keep = torch.arange(L)[None, :] < torch.tensor(lk)[:, None]
    mask = keep[:, None, None, :].expand(B, H, L, L)
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v)),
                                                           attn_mask=mask, scale=0.5)
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-12)


@pytest.mark.parametrize("causal,w,gh,gt", [(False, 4, 1, 1), (False, 3, 5, 0), (True, 4, 2, 0), (2, 3, 1, 2),
                                             (False, 0, 3, 3)])
def test_global_tokens_match_torch_sdpa(causal, w, gh, gt):
    """Leading / trailing global key positions on top of a window, against torch
    SDPA with the mask built here from its own expression."""
    B, H, Lq, Lk, d = 1, 2, 20, 20 if causal != 2 else 26, 6
    q, k, v = _rand(B, H, Lq, d), _rand(B, H, Lk, d), _rand(B, H, Lk, d)
    O, _ = oracle.attn_fwd(q, k, v, 0.4, causal, w, global_head=gh, global_tail=gt)
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    off = Lk - Lq if causal == 2 else 0
    base = torch.ones(Lq, Lk, dtype=torch.bool)
    if causal:
        base &= j <= i + off
        if w:
            base &= j > i + off - w
    elif w:
        base &= (i - j).abs() < w
    glob = ((j < gh) | (j >= Lk - gt)).expand(Lq, Lk)
    if causal:
        glob = glob & (j <= i + off)
    mask = base | glob
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v)),
                                                           attn_mask=mask, scale=0.4)
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-12)


def test_global_tokens_backward_finite_differences():
    """Gradient with global head/tail keys on a two-sided window, against central differences."""
    rng = np.random.default_rng(11)
    q, k, v, R = (rng.standard_normal((1, 2, 9, 3)) for _ in range(4))
    dq, dk, dv = oracle.attn_bwd(q, k, v, R, 0.5, False, 2, global_head=1, global_tail=2)
    eps = 1e-5
    for X, G in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = X[idx]
            X[idx] = old + eps
            fp = float(np.sum(oracle.attn_fwd(q, k, v, 0.5, False, 2, global_head=1, global_tail=2)[0] * R))
            X[idx] = old - eps
            fm = float(np.sum(oracle.attn_fwd(q, k, v, 0.5, False, 2, global_head=1, global_tail=2)[0] * R))
            X[idx] = old
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(G, num, atol=1e-6, rtol=0)


# ---------------------------------------------------------------- block-sparse mask
def _block_rule(Lq, Lk, b):
    """Closed form of the block-sparse construction, written independently of
    the oracle's loops: query i (block start s = b * floor(i / b)) sees keys
    max(0, s - b) <= j < min(Lk, s + 2b - 1)."""
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    s = (i // b) * b
    return (j >= (s - b).clamp(min=0)) & (j < (s + 2 * b - 1).clamp(max=Lk))


@pytest.mark.parametrize("Lq,Lk,b,causal,w", [(40, 40, 8, False, 0), (40, 40, 5, True, 0), (33, 50, 7, False, 0),
                                              (50, 33, 6, 2, 0), (40, 40, 8, False, 6), (30, 30, 3, True, 4)])
def test_block_sparse_matches_torch_sdpa(Lq, Lk, b, causal, w):
    """Block-sparse mask of "大模型高效注意力机制全解析" §4.1.2 (with causal / window
    masks on top) against torch SDPA with the mask from the closed-form rule."""
    q, k, v = _rand(1, 2, Lq, 5), _rand(1, 2, Lk, 5), _rand(1, 2, Lk, 5)
    O, _ = oracle.attn_fwd(q, k, v, 0.45, causal, w, sparse_block=b)
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    off = Lk - Lq if causal == 2 else 0
    mask = _block_rule(Lq, Lk, b)
    if causal:
        mask &= j <= i + off
        if w:
            mask &= j > i + off - w
    elif w:
        mask &= (i - j).abs() < w
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v)),
                                                           attn_mask=mask, scale=0.45)
    rows = mask.any(1).numpy()  # SDPA gives NaN on rows with no visible key
    np.testing.assert_allclose(O[0, :, rows], ref.numpy()[0, :, rows], atol=1e-12)
    assert np.all(O[0, :, ~rows] == 0.0)


def test_block_sparse_with_global_keys_matches_torch_sdpa():
    """Block-sparse mask and global keys together: the global keys are added on
    top of the block-sparse (and causal) band, as they are on top of a window."""
    Lq = Lk = 36
    b, gh, gt = 6, 2, 3
    q, k, v = _rand(1, 2, Lq, 5), _rand(1, 2, Lk, 5), _rand(1, 2, Lk, 5)
    for causal in (False, True):
        O, _ = oracle.attn_fwd(q, k, v, 0.4, causal, 0, global_head=gh, global_tail=gt, sparse_block=b)
        i = torch.arange(Lq)[:, None]
        j = torch.arange(Lk)[None, :]
        band = _block_rule(Lq, Lk, b)
        glob = ((j < gh) | (j >= Lk - gt)).expand(Lq, Lk)
        if causal:
            band = band & (j <= i)
            glob = glob & (j <= i)
        ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v)),
                                                               attn_mask=band | glob, scale=0.4)
        np.testing.assert_allclose(O, ref.numpy(), atol=1e-12)


def test_block_sparse_pages_example_counts():
    """The page's example (seq_len 1024, block 64): interior query blocks see
    3b - 1 keys, the first block 2b - 1, the last 2b; the total follows."""
    m = oracle.visible_mask(1024, 1024, False, 0, sparse_block=64)
    per_row = m.sum(1)
    assert set(per_row[:64]) == {127} and set(per_row[64:960]) == {191} and set(per_row[960:]) == {128}
    assert m.sum() == 64 * (127 + 14 * 191 + 128)


def test_block_sparse_degenerate_sizes():
    """b >= L: every query sees every key (plain attention); b = 1: query i
    sees keys i - 1 and i, the same as a causal window of two keys."""
    q, k, v = _rand(1, 2, 17, 4), _rand(1, 2, 17, 4), _rand(1, 2, 17, 4)
    O, lse = oracle.attn_fwd(q, k, v, 0.6, False, 0, sparse_block=17)
    O0, lse0 = oracle.attn_fwd(q, k, v, 0.6, False, 0)
    np.testing.assert_array_equal(O, O0)
    np.testing.assert_array_equal(lse, lse0)
    O, lse = oracle.attn_fwd(q, k, v, 0.6, False, 0, sparse_block=1)
    O2, lse2 = oracle.attn_fwd(q, k, v, 0.6, True, 2)
    np.testing.assert_allclose(O, O2, atol=1e-15)
    np.testing.assert_allclose(lse, lse2, atol=1e-15)


def test_block_sparse_backward_finite_differences():
    """Gradient under the block-sparse mask against central differences."""
    rng = np.random.default_rng(12)
    q, k, v, R = (rng.standard_normal((1, 2, 11, 3)) for _ in range(4))
    dq, dk, dv = oracle.attn_bwd(q, k, v, R, 0.5, False, 0, sparse_block=3)
    eps = 1e-5
    for X, G in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = X[idx]
            X[idx] = old + eps
            fp = float(np.sum(oracle.attn_fwd(q, k, v, 0.5, False, 0, sparse_block=3)[0] * R))
            X[idx] = old - eps
            fm = float(np.sum(oracle.attn_fwd(q, k, v, 0.5, False, 0, sparse_block=3)[0] * R))
            X[idx] = old
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(G, num, atol=1e-6, rtol=0)


def test_value_shift_and_score_shift_invariance():
    """V + 1 c^T gives O + 1 c^T; a per-row constant added to the logits changes nothing."""
    L, d = 19, 4
    q, k, v = _rand(1, 1, L, d), _rand(1, 1, L, d), _rand(1, 1, L, d)
    c = _rand(d)
    O, lse = oracle.attn_fwd(q, k, v, 0.5, True, 7)
    O2, _ = oracle.attn_fwd(q, k, v + c, 0.5, True, 7)
    np.testing.assert_allclose(O2, O + c, atol=1e-13)
    # Give every key the same component along u; shifting q along u adds a
    # per-row constant to its logits.
    u = np.zeros(d + 1)
    u[-1] = 1.0
    k1 = np.concatenate([k, np.ones((1, 1, L, 1))], -1)
    v1 = v
    q1 = np.concatenate([q, np.zeros((1, 1, L, 1))], -1)
    q2 = q1 + 3.0 * u
    Oa, la = oracle.attn_fwd(q1, k1, v1, 0.5, True, 7)
    Ob, lb = oracle.attn_fwd(q2, k1, v1, 0.5, True, 7)
    np.testing.assert_allclose(Ob, Oa, atol=1e-13)
    np.testing.assert_allclose(lb, la + 1.5, atol=1e-13)


def _online_softmax_attention(q, k, v, scale, vis, block):
    """The streaming recurrence of "高效注意力：FlashAttention 与线性注意力" (原理与机制):
    keep a running max m and running sum l per row; merge each key block by
    rescaling the old sum and the old output by e^{m_old - m_new}."""
    Lq, d = q.shape[0], v.shape[1]
    m = np.full(Lq, -np.inf)
    l = np.zeros(Lq)
    acc = np.zeros((Lq, d))
    for j0 in range(0, k.shape[0], block):
        s = scale * q @ k[j0:j0 + block].T
        s = np.where(vis[:, j0:j0 + block], s, -np.inf)
        m_new = np.maximum(m, s.max(1))
        safe = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
        p = np.exp(s - safe[:, None])
        l = l * alpha + p.sum(1)
        acc = acc * alpha[:, None] + p @ v[j0:j0 + block]
        m = m_new
    O = np.divide(acc, l[:, None], out=np.zeros_like(acc), where=l[:, None] > 0)
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m + np.log(l), -np.inf)
    return O, lse


@pytest.mark.parametrize("block", [1, 3, 7, 16, 64])
@pytest.mark.parametrize("causal,window", MASKS)
def test_block_split_online_softmax_equals_full(block, causal, window):
    L, d = 45, 8
    q, k, v = _rand(L, d), _rand(L, d), _rand(L, d)
    vis = oracle.visible_mask(L, L, causal, window)
    O, lse = oracle.attn_fwd(q[None, None], k[None, None], v[None, None], 0.35, causal, window)
    O2, lse2 = _online_softmax_attention(q, k, v, 0.35, vis, block)
    np.testing.assert_allclose(O2, O[0, 0], atol=1e-12)
    np.testing.assert_allclose(lse2, lse[0, 0], atol=1e-12)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (6, 1), (8, 8), (32, 8)])
def test_gqa_equals_mha_with_repeated_kv(Hq, Hkv):
    """Query head h uses K/V head h // (Hq/Hkv): equal to MHA with K/V repeated."""
    B, L, d = 2, 13, 4
    q = _rand(B, Hq, L, d)
    k, v = _rand(B, Hkv, L, d), _rand(B, Hkv, L, d)
    G = Hq // Hkv
    kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
    O, lse = oracle.attn_fwd(q, k, v, 0.5, True, 4)
    Or, lser = oracle.attn_fwd(q, kr, vr, 0.5, True, 4)
    np.testing.assert_array_equal(O, Or)
    np.testing.assert_array_equal(lse, lser)
    do = _rand(B, Hq, L, d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.5, True, 4)
    dqr, dkr, dvr = oracle.attn_bwd(q, kr, vr, do, 0.5, True, 4)
    np.testing.assert_allclose(dq, dqr, atol=1e-14)
    np.testing.assert_allclose(dk, dkr.reshape(B, Hkv, G, L, d).sum(2), atol=1e-13)
    np.testing.assert_allclose(dv, dvr.reshape(B, Hkv, G, L, d).sum(2), atol=1e-13)


# ---------------------------------------------------------------- backward
def _loss(q, k, v, R, scale, causal, window):
    O, _ = oracle.attn_fwd(q, k, v, scale, causal, window)
    return float(np.sum(O * R))


@pytest.mark.parametrize("Hq,Hkv,L,causal,window", [
    (2, 2, 9, False, 0), (2, 2, 9, True, 0), (2, 1, 8, True, 3), (2, 2, 7, True, 1),
    (4, 2, 6, False, 0), (2, 1, 9, False, 3), (2, 1, -5, 2, 0), (2, 2, -4, 2, 3),
])
def test_backward_matches_finite_differences(Hq, Hkv, L, causal, window):
    """Gradient of <R, O> against central differences, float64, to 1e-6.
    A negative L is a rectangular case: Lq = |L| queries over Lk = |L| + 4 keys."""
    rng = np.random.default_rng(7)
    d = 4
    Lq, Lk = (L, L) if L > 0 else (-L, -L + 4)
    q = rng.standard_normal((1, Hq, Lq, d))
    k = rng.standard_normal((1, Hkv, Lk, d))
    v = rng.standard_normal((1, Hkv, Lk, d))
    R = rng.standard_normal((1, Hq, Lq, d))
    scale = 0.6
    dq, dk, dv = oracle.attn_bwd(q, k, v, R, scale, causal, window)
    eps = 1e-5
    for X, G in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = X[idx]
            X[idx] = old + eps
            fp = _loss(q, k, v, R, scale, causal, window)
            X[idx] = old - eps
            fm = _loss(q, k, v, R, scale, causal, window)
            X[idx] = old
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(G, num, atol=1e-6, rtol=0)


def test_fully_masked_rows_are_zero():
    """Lq > Lk with a window leaves late rows with no visible key: O=0, LSE=-inf, dQ=0."""
    Lq, Lk, d, w = 12, 4, 3, 3
    q, k, v = _rand(1, 1, Lq, d), _rand(1, 1, Lk, d), _rand(1, 1, Lk, d)
    vis = oracle.visible_mask(Lq, Lk, True, w)
    dead = ~vis.any(1)
    assert dead.sum() > 0
    O, lse = oracle.attn_fwd(q, k, v, 0.5, True, w)
    assert np.all(O[0, 0][dead] == 0) and np.all(np.isneginf(lse[0, 0][dead]))
    assert np.all(np.isfinite(O))
    dq, dk, dv = oracle.attn_bwd(q, k, v, _rand(1, 1, Lq, d), 0.5, True, w)
    assert np.all(dq[0, 0][dead] == 0)
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


def test_row_blocking_is_invisible(monkeypatch):
    """Evaluating a head in small row blocks over their bands gives the same numbers."""
    L, d = 70, 8
    q, k, v, do = (_rand(1, 2, L, d) for _ in range(4))
    ref = oracle.attn_fwd(q, k, v, 0.4, True, 9)
    refb = oracle.attn_bwd(q, k, v, do, 0.4, True, 9)
    monkeypatch.setattr(oa, "_ROW_BLOCK_ELEMS", 3 * L)
    blk = oracle.attn_fwd(q, k, v, 0.4, True, 9)
    blkb = oracle.attn_bwd(q, k, v, do, 0.4, True, 9)
    for a, b in zip(ref + refb, blk + blkb):
        np.testing.assert_allclose(a, b, atol=1e-14)
    rows = np.array([0, 5, 33, 69])
    Orow, lrow = oracle.attn_fwd_rows(q, k, v, 0.4, True, 9, 0, 1, rows)
    np.testing.assert_allclose(Orow, ref[0][0, 1, rows], atol=1e-14)
    np.testing.assert_allclose(lrow, ref[1][0, 1, rows], atol=1e-14)


def test_row_blocks_sum_to_full_backward():
    """Row-block contributions (the benchmark's bounded CPU sample) add up to attn_bwd."""
    B, Hq, Hkv, L, d = 1, 4, 2, 50, 8
    q, do = _rand(B, Hq, L, d), _rand(B, Hq, L, d)
    k, v = _rand(B, Hkv, L, d), _rand(B, Hkv, L, d)
    O, lse = oracle.attn_fwd(q, k, v, 0.3, True, 11)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.3, True, 11)
    sk, sv = np.zeros_like(dk), np.zeros_like(dv)
    for h in range(Hq):
        for r0 in range(0, L, 16):
            r1 = min(L, r0 + 16)
            Ob, lb, dqb, lo, hi, dkb, dvb = oracle.attn_row_block(q, k, v, do, 0.3, True, 11, 0, h, r0, r1)
            np.testing.assert_allclose(Ob, O[0, h, r0:r1], atol=1e-14)
            np.testing.assert_allclose(lb, lse[0, h, r0:r1], atol=1e-14)
            np.testing.assert_allclose(dqb, dq[0, h, r0:r1], atol=1e-14)
            sk[0, h // 2, lo:hi] += dkb
            sv[0, h // 2, lo:hi] += dvb
    np.testing.assert_allclose(sk, dk, atol=1e-13)
    np.testing.assert_allclose(sv, dv, atol=1e-13)


# ---------------------------------------------------------------- library cross-checks
torch = pytest.importorskip("torch")


@pytest.mark.parametrize("Hq,Hkv,causal,window", [
    (4, 4, False, 0), (4, 4, True, 0), (4, 2, True, 0), (4, 1, True, 6), (2, 2, True, 1),
])
def test_matches_torch_sdpa_float64(Hq, Hkv, causal, window):
    """Special case that reduces to a library routine: torch CPU float64 SDPA (test only)."""
    B, L, d = 2, 33, 16
    q, k, v = _rand(B, Hq, L, d), _rand(B, Hkv, L, d), _rand(B, Hkv, L, d)
    O, _ = oracle.attn_fwd(q, k, v, 0.25, causal, window)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    G = Hq // Hkv
    tk, tv = tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1)
    mask = torch.from_numpy(oracle.visible_mask(L, L, causal, window))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.25)
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-12)


@pytest.mark.parametrize("Lq,Lk,w", [(7, 30, 0), (30, 30, 0), (12, 40, 6), (40, 12, 0)])
def test_bottom_right_causal_matches_torch_sdpa(Lq, Lk, w):
    """causal = 2 against torch SDPA with a lower-triangular mask shifted by Lk - Lq
    (built here with torch.tril), and the window as a band below it.  Rows
    with no visible key are compared as zeros (SDPA returns NaN there)."""
    B, Hq, Hkv, d = 1, 2, 1, 8
    q, k, v = _rand(B, Hq, Lq, d), _rand(B, Hkv, Lk, d), _rand(B, Hkv, Lk, d)
    O, _ = oracle.attn_fwd(q, k, v, 0.3, 2, w)
    mask = torch.ones(Lq, Lk, dtype=torch.bool).tril(diagonal=Lk - Lq)
    if w > 0:
        mask &= ~torch.ones(Lq, Lk, dtype=torch.bool).tril(diagonal=Lk - Lq - w)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    tk, tv = tk.repeat_interleave(Hq // Hkv, 1), tv.repeat_interleave(Hq // Hkv, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.3).numpy()
    dead = ~mask.any(1).numpy()
    ref[:, :, dead] = 0.0
    np.testing.assert_allclose(O, ref, atol=1e-12)


@pytest.mark.parametrize("w", [1, 4, 40])
def test_two_sided_window_matches_torch_sdpa(w):
    """Non-causal window against torch SDPA with the band |i - j| < w built here."""
    B, Hq, Hkv, L, d = 1, 4, 2, 37, 8
    q, k, v = _rand(B, Hq, L, d), _rand(B, Hkv, L, d), _rand(B, Hkv, L, d)
    O, _ = oracle.attn_fwd(q, k, v, 0.3, False, w)
    idx = torch.arange(L)
    band = (idx[:, None] - idx[None, :]).abs() < w
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    tk, tv = tk.repeat_interleave(2, 1), tv.repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=band, scale=0.3)
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-12)


def test_pages_fp32_experiment_magnitude():
    """"缩放定律与高效注意力" 实验 1: B=2,H=4,L=128,d=32, seed 42, fp32 manual vs fused
    attention differ by about 4.5e-7 (rounding order only).  Both fp32 results sit
    within that order of magnitude of the exact float64 oracle."""
    torch.manual_seed(42)
    B, H, L, d = 2, 4, 128, 32
    q, k, v = [torch.randn(B, H, L, d) for _ in range(3)]
    manual = (q @ k.transpose(-2, -1) / d ** 0.5).softmax(-1) @ v
    fused = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    exact, _ = oracle.attn_fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               1 / math.sqrt(d))
    e1 = np.abs(manual.double().numpy() - exact).max()
    e2 = np.abs(fused.double().numpy() - exact).max()
    assert e1 < 5e-6 and e2 < 5e-6
    assert (manual - fused).abs().max().item() < 5e-6


# ---------------------------------------------------------------- input recipe
def test_bf16_rounding_matches_torch():
    """The generator's float32 -> bf16 rounding is round-to-nearest-even."""
    from synth import f32_to_bf16_bits
    x = np.random.default_rng(3).standard_normal(10000).astype(np.float32) * 37
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0]
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_inputs_are_seeded_and_exact_bf16():
    a = make_shape_inputs(1, 2, 1, 5, 5, 8, seed=11, with_do=True)
    b = make_shape_inputs(1, 2, 1, 5, 5, 8, seed=11, with_do=True)
    for n in "q", "k", "v", "do":
        assert np.array_equal(a[n], b[n])
    x = bf16_bits_to_f32(a["q"])
    assert np.array_equal(x.view(np.uint32) & 0xFFFF, np.zeros_like(x, dtype=np.uint32))


# ---------------------------------------------------------------- planted slips
def _pins_pass():
    """Run a compact subset of the pins; False if any fails."""
    checks = [test_golden_hand_worked_example,
              lambda: test_zero_query_gives_mean_of_visible(True, 5),
              lambda: test_gqa_equals_mha_with_repeated_kv(4, 2),
              lambda: test_backward_matches_finite_differences(2, 1, 8, True, 3),
              lambda: test_matches_torch_sdpa_float64(4, 2, True, 0),
              lambda: test_block_sparse_matches_torch_sdpa(33, 50, 7, False, 0)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def test_pins_pass_unmodified():
    assert _pins_pass()


@pytest.mark.parametrize("slip", ["transpose", "no_mask", "dS_sign", "dk_no_scale", "gqa_map", "block_edge"])
def test_pins_catch_planted_slips(monkeypatch, slip):
    """Plant a plausible mistake in the oracle (CPU only) and check a pin fails."""
    if slip == "transpose":
        orig = oa.attention_weights
        monkeypatch.setattr(oa, "attention_weights",
                            lambda q, k, s, vis: _transposed_weights(orig, q, k, s, vis))
    elif slip == "no_mask":
        orig = oa.attention_weights
        monkeypatch.setattr(oa, "attention_weights",
                            lambda q, k, s, vis: orig(q, k, s, np.ones_like(vis)))
    elif slip == "dS_sign":
        monkeypatch.setattr(oa, "_head_bwd", _bwd_with(lambda A, dP, D: A * (dP + D)))
    elif slip == "dk_no_scale":
        monkeypatch.setattr(oa, "_head_bwd", _bwd_with(None, dk_scale=False))
    elif slip == "gqa_map":
        monkeypatch.setattr(oa, "_kv_head", lambda h, Hq, Hkv: h % Hkv)
    elif slip == "block_edge":
        # Each query block one key block too narrow on the right (j up to i + b - 2).
        orig = oa.sparse_block_mask
        monkeypatch.setattr(oa, "sparse_block_mask",
                            lambda rows, lo, hi, b, Lq, Lk: orig(rows, lo, hi, b, Lq, Lk)
                            & _drop_last_block_key(rows, lo, hi, b, Lk))
    assert not _pins_pass()


def _drop_last_block_key(rows, lo, hi, b, Lk):
    """Keep every key except the last one the block-sparse construction reaches."""
    rows = np.asarray(rows)
    s = (rows // b) * b
    last = np.minimum(Lk, s + 2 * b - 1) - 1
    return np.arange(lo, hi)[None, :] != last[:, None]


def _transposed_weights(orig, q, k, s, vis):
    # scores built as K Q^T instead of Q K^T (only changes square, unmasked cases)
    if q.shape[0] == k.shape[0]:
        S = s * (k @ q.T)
        S = np.where(vis, S, -np.inf)
        m = np.max(S, 1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0)
        E = np.where(vis, np.exp(S - m), 0)
        l = E.sum(1, keepdims=True)
        A = np.divide(E, l, out=np.zeros_like(E), where=l > 0)
        with np.errstate(divide="ignore"):
            return A, np.where(l[:, 0] > 0, m[:, 0] + np.log(l[:, 0]), -np.inf)
    return orig(q, k, s, vis)


def _bwd_with(ds_fn, dk_scale=True):
    def head_bwd(qh, kh, vh, doh, scale, causal, window, gl=(0, 0), sb=0):
        Lq, Lk = qh.shape[0], kh.shape[0]
        vis = oracle.visible_mask(Lq, Lk, causal, window, *gl, sparse_block=sb)
        A, _ = oa.attention_weights(qh, kh, scale, vis)
        O = A @ vh
        dP = doh @ vh.T
        D = np.sum(doh * O, 1, keepdims=True)
        dS = ds_fn(A, dP, D) if ds_fn else A * (dP - D)
        return scale * dS @ kh, (scale if dk_scale else 1.0) * dS.T @ qh, A.T @ doh
    return head_bwd

"""Plain float64 attention: the definition written out, no tiling, no online softmax.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Nothing here is shared
with the CUDA path: the two meet only on the seeded bf16 inputs.

Sources (page title and section):
  * "注意力优化：FlashAttention 与稀疏注意力", 核心公式 / 公式速览:
      S = Q K^T / sqrt(d_k); A = row softmax of S (each row sums to 1);
      output row i = sum_j A_ij V_j; a disallowed key j gets logit -inf
      before the softmax, so its weight is 0.
  * "高效注意力" §3 (MQA/GQA): several query heads share one K/V head.
  * "高效注意力" §4 and "大模型高效注意力机制全解析" §3.2.1 (sliding_window):
      each token attends to a window of nearby tokens.  Read here as the
      causal band  i - w < j <= i  (w keys, the query itself included), and,
      without a causal mask, as the two-sided band  i - w < j < i + w  (the
      "前后" (before and after) wording of the same section).
  * "大模型高效注意力机制全解析" §4.1.2 (block-sparse attention): the mask is
      built block by block: for each query block start i (step b) and each
      j from max(0, i - b) to min(L, i + b) - 1, the b x b block at (i, j) is
      set.  `sparse_block_mask` builds it exactly that way.
  * "缩放定律与高效注意力" §3.3: the backward pass needs only O and the per-row
      logsumexp; the gradient formulas themselves are the textbook softmax
      gradient (the pages do not print them).

Conventions (the readings the pages leave open):
  * Layout [B, H, L, d]; query head h reads K/V head h // (Hq // Hkv).
  * Causal alignment is top-left: key j visible to query i iff j <= i.
  * `scale` multiplies Q K^T; LSE is the natural log of sum_j exp(scale*S_ij)
    over visible j.
  * A row with no visible key has O = 0, LSE = -inf, dQ = 0 (no NaN).
"""

from __future__ import annotations

import numpy as np

# Rows per block when a head is evaluated in row blocks (bounds memory only;
# every row is still the plain definition over its visible columns).
_ROW_BLOCK_ELEMS = 1 << 24


def diag_offset(causal, Lq: int, Lk: int) -> int:
    """Key index of the causal diagonal for query row 0.

    causal = 1 (or True): top-left alignment, query i sees keys j <= i.
    causal = 2: bottom-right alignment, query i sits at position i + Lk - Lq
    of the key sequence (the last query row sees the last key), as when new
    queries attend to a longer cache of earlier keys.
    """
    return Lk - Lq if causal == 2 else 0


def sparse_block_mask(rows, lo: int, hi: int, b: int, Lq: int, Lk: int) -> np.ndarray:
    """The block-sparse mask of "大模型高效注意力机制全解析" §4.1.2 for query rows
    `rows` and key columns [lo, hi): the page's construction on an [Lq, Lk]
    matrix (query block starts i = 0, b, 2b, ... below Lq; for each, every j
    in [max(0, i - b), min(Lk, i + b)) sets the block rows i..i+b-1, keys
    j..j+b-1, clipped to the matrix), restricted to the rows asked for."""
    rows = np.asarray(rows)
    out = np.zeros((rows.size, hi - lo), dtype=bool)
    if rows.size == 0:
        return out
    r_min, r_max = int(rows.min()), int(rows.max())
    for i in range(0, Lq, b):
        if i + b <= r_min or i > r_max:
            continue  # this query block holds none of the rows
        sel = (rows >= i) & (rows < i + b)
        for j in range(max(0, i - b), min(Lk, i + b)):
            c0, c1 = max(j, lo), min(j + b, Lk, hi)
            if c0 < c1:
                out[np.ix_(sel, np.arange(c0 - lo, c1 - lo))] = True
    return out


def _visible(i, j, causal, window: int, off: int = 0, glob=(0, 0, 0), blk=None) -> np.ndarray:
    """Elementwise visibility of key j to query i (broadcasting arrays);
    `off` is diag_offset(causal, Lq, Lk); glob = (global_head, global_tail, Lk):
    the first global_head and the last global_tail key positions are visible
    to every query (still subject to the causal mask); blk: an optional
    block-sparse mask of the same shape, intersected with the causal and window
    masks before the global keys are added."""
    vis = np.ones(np.broadcast(i, j).shape, dtype=bool)
    if causal:
        vis &= j <= i + off
    if window > 0:
        vis &= j > i + off - window
        if not causal:
            vis &= j < i + window
    if blk is not None:
        vis &= blk
    gh, gt, lk = glob
    if gh > 0 or gt > 0:
        g = (j < gh) | (j >= lk - gt)
        if causal:
            g = g & (j <= i + off)
        vis = vis | g
    return vis


def visible_mask(Lq: int, Lk: int, causal, window: int, global_head: int = 0, global_tail: int = 0,
                 sparse_block: int = 0) -> np.ndarray:
    """Boolean [Lq, Lk]: True where key j is visible to query i.

    Causal: j <= i (causal = 2: j <= i + Lk - Lq).  Window w > 0: the w keys
    ending at the query's diagonal when causal (i - w < j <= i, "高效注意力" §4
    sliding window); without causal the band reaches w - 1 keys to either
    side, i - w < j < i + w (the two-sided "前后" reading of the same section).
    """
    blk = sparse_block_mask(np.arange(Lq), 0, Lk, sparse_block, Lq, Lk) if sparse_block > 0 else None
    return _visible(np.arange(Lq)[:, None], np.arange(Lk)[None, :], causal, window, diag_offset(causal, Lq, Lk),
                    (global_head, global_tail, Lk), blk)


def visible_band(r0: int, r1: int, Lk: int, causal, window: int, off: int = 0, glob=(0, 0, 0)) -> tuple[int, int]:
    """Columns [lo, hi) that can be visible to any row in [r0, r1)."""
    if causal:
        hi = min(Lk, r1 + off)
    elif window > 0 and glob[1] == 0:
        hi = min(Lk, r1 - 1 + window)
    else:
        hi = Lk
    lo = max(0, r0 + off - window + 1) if window > 0 and glob[0] == 0 else 0
    return lo, max(lo, hi)


def _f64(x) -> np.ndarray:
    if x.dtype == np.uint16:  # bf16 bits: widen exactly
        x = (x.astype(np.uint32) << 16).view(np.float32)
    return np.asarray(x, dtype=np.float64)


def attention_weights(q, k, scale: float, vis: np.ndarray):
    """Scores, weights and logsumexp for one head.

    q [Lq, d], k [Lk, d] float64; vis [Lq, Lk] bool.
    Returns (A, lse): A[i, j] = exp(S_ij) / sum_vis exp(S_ij) on visible
    entries and exactly 0 elsewhere; lse[i] = log sum_vis exp(S_ij).
    """
    if k.shape[0] == 0:  # no key at all (a sequence of a padded batch with no keys): every row is fully masked
        return np.zeros((q.shape[0], 0)), np.full(q.shape[0], -np.inf)
    S = scale * (q @ k.T)
    S = np.where(vis, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)          # fully masked row: any shift works
    E = np.where(vis, np.exp(S - m), 0.0)
    l = E.sum(axis=1, keepdims=True)
    A = np.divide(E, l, out=np.zeros_like(E), where=l > 0)
    with np.errstate(divide="ignore"):
        lse = np.where(l[:, 0] > 0, m[:, 0] + np.log(l[:, 0]), -np.inf)
    return A, lse


def _head_fwd(qh, kh, vh, scale, causal, window, rows=None, gl=(0, 0), sb=0):
    """O and LSE for the rows `rows` (default: all) of one head."""
    Lq, Lk = qh.shape[0], kh.shape[0]
    off = diag_offset(causal, Lq, Lk)
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    O = np.zeros((rows.size, vh.shape[1]))
    lse = np.full(rows.size, -np.inf)
    if rows.size == 0:
        return O, lse
    # Contiguous runs of rows are evaluated block by block over their band.
    step = max(1, _ROW_BLOCK_ELEMS // max(1, Lk))
    start = 0
    while start < rows.size:
        stop = min(rows.size, start + step)
        blk = rows[start:stop]
        r0, r1 = int(blk.min()), int(blk.max()) + 1
        glob = (gl[0], gl[1], Lk)
        lo, hi = visible_band(r0, r1, Lk, causal, window, off, glob)
        vis = _band_mask(blk, lo, hi, causal, window, off, glob, sb, Lq, Lk)
        A, l = attention_weights(qh[blk], kh[lo:hi], scale, vis)
        O[start:stop] = A @ vh[lo:hi]
        lse[start:stop] = l
        start = stop
    return O, lse


def _band_mask(rows, lo, hi, causal, window, off, glob=(0, 0, 0), sb=0, Lq=0, Lk=0):
    blk = sparse_block_mask(rows, lo, hi, sb, Lq, Lk) if sb > 0 else None
    return _visible(np.asarray(rows)[:, None], np.arange(lo, hi)[None, :], causal, window, off, glob, blk)


def _group(Hq: int, Hkv: int) -> int:
    if Hkv <= 0 or Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return Hq // Hkv


def _kv_head(h: int, Hq: int, Hkv: int) -> int:
    """K/V head read by query head h: contiguous groups of Hq/Hkv query heads."""
    return h // _group(Hq, Hkv)


def _lengths(seqlens, b: int, full: int) -> int:
    return full if seqlens is None else min(full, int(seqlens[b]))


def attn_fwd(q, k, v, scale: float, causal: bool = False, window: int = 0, heads=None, seqlens_q=None,
             seqlens_k=None, global_head: int = 0, global_tail: int = 0, sparse_block: int = 0):
    """O [B,Hq,Lq,d] and LSE [B,Hq,Lq] in float64.

    q: [B,Hq,Lq,d]; k, v: [B,Hkv,Lk,d] (float or bf16 bits as uint16).
    heads: optional list of (b, h) to evaluate; other heads are left NaN.
    seqlens_q / seqlens_k: optional per-sequence lengths of a padded batch
    ("大模型高效注意力机制全解析" §5.2.2: requests of different lengths are padded
    into one batch and each output is cut back to its own length):
    sequence b is its own attention problem over its first seqlens_q[b]
    queries and seqlens_k[b] keys (a bottom-right causal diagonal is placed by
    those lengths); padded query rows get O = 0 and LSE = -inf.
    sparse_block: b > 0 adds the block-sparse mask of "大模型高效注意力机制全解析"
    §4.1.2 with b x b blocks (each sequence of a padded batch builds it over
    its own lengths).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    O = np.full((B, Hq, Lq, v.shape[-1]), np.nan)
    lse = np.full((B, Hq, Lq), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        g = _kv_head(h, Hq, Hkv)
        nq, nk = _lengths(seqlens_q, b, Lq), _lengths(seqlens_k, b, Lk)
        O[b, h] = 0.0
        lse[b, h] = -np.inf
        O[b, h, :nq], lse[b, h, :nq] = _head_fwd(q[b, h, :nq], k[b, g, :nk], v[b, g, :nk], scale, causal, window,
                                                 gl=(global_head, global_tail), sb=sparse_block)
    return O, lse


def attn_fwd_rows(q, k, v, scale, causal, window, b, h, rows):
    """O and LSE for selected rows of one head (sampled checks at full size).

    Each row is evaluated from the definition over all of its visible keys.
    """
    Hq, Hkv = q.shape[1], k.shape[1]
    g = _kv_head(h, Hq, Hkv)
    rows = np.sort(np.asarray(rows))
    qh = _f64(q[b, h])
    kh = _f64(k[b, g])
    vh = _f64(v[b, g])
    Lq, Lk = qh.shape[0], kh.shape[0]
    off = diag_offset(causal, Lq, Lk)
    O = np.zeros((rows.size, qh.shape[1]))
    lse = np.zeros(rows.size)
    for n, i in enumerate(rows):
        lo, hi = visible_band(int(i), int(i) + 1, Lk, causal, window, off)
        vis = _band_mask([i], lo, hi, causal, window, off)
        A, l = attention_weights(qh[i:i + 1], kh[lo:hi], scale, vis)
        O[n] = (A @ vh[lo:hi])[0]
        lse[n] = l[0]
    return O, lse


def _rows_bwd(qh, kh, vh, doh, scale, causal, window, r0, r1, gl=(0, 0), sb=0):
    """Rows [r0, r1) of one head: their O and LSE, their dQ rows, and their
    contributions to dK and dV over the visible key band [lo, hi)."""
    Lq, Lk = qh.shape[0], kh.shape[0]
    off = diag_offset(causal, Lq, Lk)
    glob = (gl[0], gl[1], Lk)
    lo, hi = visible_band(r0, r1, Lk, causal, window, off, glob)
    vis = _band_mask(np.arange(r0, r1), lo, hi, causal, window, off, glob, sb, Lq, Lk)
    A, lse = attention_weights(qh[r0:r1], kh[lo:hi], scale, vis)
    O = A @ vh[lo:hi]
    dO = doh[r0:r1]
    dv = A.T @ dO                                # dV = A^T dO
    dP = dO @ vh[lo:hi].T                        # dP = dO V^T
    D = np.sum(dO * O, axis=1, keepdims=True)    # D_i = dO_i . O_i = sum_j A_ij dP_ij
    dS = A * (dP - D)                            # softmax Jacobian applied row by row
    dq = scale * (dS @ kh[lo:hi])                # S = scale Q K^T
    dk = scale * (dS.T @ qh[r0:r1])
    return lo, hi, O, lse, dq, dk, dv


def _head_bwd(qh, kh, vh, doh, scale, causal, window, gl=(0, 0), sb=0):
    """dQ, dK, dV for one (query head, kv head) pair; textbook softmax gradient."""
    Lq, Lk = qh.shape[0], kh.shape[0]
    dq = np.zeros_like(qh)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    step = max(1, _ROW_BLOCK_ELEMS // max(1, Lk))
    for r0 in range(0, Lq, step):
        r1 = min(Lq, r0 + step)
        lo, hi, _, _, dqb, dkb, dvb = _rows_bwd(qh, kh, vh, doh, scale, causal, window, r0, r1, gl, sb)
        dq[r0:r1] = dqb
        dk[lo:hi] += dkb
        dv[lo:hi] += dvb
    return dq, dk, dv


def attn_row_block(q, k, v, do, scale, causal, window, b, h, r0, r1):
    """Query rows [r0, r1) of head (b, h): O and LSE of those rows, their dQ
    rows, and their (partial) contributions to dK and dV of K/V head
    h // (Hq/Hkv), returned as (O, lse, dq, lo, hi, dk_part, dv_part) with
    dk_part/dv_part covering keys [lo, hi).  Summing the parts over all row
    blocks of all heads of a group gives attn_bwd's dK and dV."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = _kv_head(h, Hq, Hkv)
    lo, hi, O, lse, dq, dk, dv = _rows_bwd(_f64(q[b, h]), _f64(k[b, g]), _f64(v[b, g]), _f64(do[b, h]),
                                           scale, causal, window, r0, r1)
    return O, lse, dq, lo, hi, dk, dv


def attn_bwd(q, k, v, do, scale: float, causal: bool = False, window: int = 0, heads=None, seqlens_q=None,
             seqlens_k=None, global_head: int = 0, global_tail: int = 0, sparse_block: int = 0):
    """dQ [B,Hq,Lq,d], dK and dV [B,Hkv,Lk,d] in float64.

    dK/dV of a K/V head are summed over the query heads that share it.
    heads: optional list of (b, hkv): only those K/V heads (and all query
    heads of their groups) are evaluated; the rest is left NaN.
    seqlens_q / seqlens_k, global_head / global_tail, sparse_block: as
    attn_fwd; padded rows and keys get zero gradients.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    _group(Hq, Hkv)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    todo = heads if heads is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for b, g in todo:
        nq, nk = _lengths(seqlens_q, b, Lq), _lengths(seqlens_k, b, Lk)
        dk[b, g] = 0.0
        dv[b, g] = 0.0
        for h in (h for h in range(Hq) if _kv_head(h, Hq, Hkv) == g):
            dq[b, h] = 0.0
            dqh, dkh, dvh = _head_bwd(q[b, h, :nq], k[b, g, :nk], v[b, g, :nk], do[b, h, :nq], scale, causal, window,
                                      (global_head, global_tail), sparse_block)
            dq[b, h, :nq] = dqh
            dk[b, g, :nk] += dkh
            dv[b, g, :nk] += dvh
    return dq, dk, dv

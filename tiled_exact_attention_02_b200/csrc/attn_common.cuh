// attn_common.cuh - problem description and mask/tile classification shared by
// the forward and backward kernels and their host-side launchers.
//
// Visibility ("注意力优化：FlashAttention 与稀疏注意力", 公式速览: disallowed keys
// get -inf before the softmax; "高效注意力" §4: sliding window).  With
// off = Lk - Lq for causal = 2 (bottom-right alignment: query i sits at key
// position i + Lk - Lq) and off = 0 otherwise,
//   key j is visible to query i  iff  (!causal || j <= i + off)
//                                 && (window <= 0 || j > i + off - window)
//                                 && (causal || window <= 0 || j < i + window)
// i.e. a window is the w keys ending at the query's diagonal under a causal
// mask, and the two-sided band of w - 1 keys on either side of i without one.
// A tile of keys is skipped when no key in it is visible to any row of the
// query tile, processed without masking when every key is visible to every
// row, and masked element-wise otherwise.
#pragma once
#include <cuda.h>
#include <cstdint>

namespace tea {

struct Problem {
  int B, Hq, Hkv, Lq, Lk, d;
  int causal, window;  // causal: 0 none, 1 top-left, 2 bottom-right
  float scale;
  // Optional per-sequence lengths of a padded batch (device int32 [B], may be
  // null): sequence b uses only its first len_q[b] queries and len_k[b] keys
  // (clamped to [0, Lq] and [0, Lk]); Lq and Lk stay the padded extents that
  // every tensor is laid out with.
  const int* len_q = nullptr;
  const int* len_k = nullptr;
};

// The problem of sequence b: Lq and Lk replaced by its own lengths (for the
// masks and tile ranges; indexing keeps using the padded extents).
__device__ inline Problem seq_problem(const Problem& p, int b) {
  Problem s = p;
  if (p.len_q) s.Lq = p.len_q[b] < 0 ? 0 : (p.len_q[b] > p.Lq ? p.Lq : p.len_q[b]);
  if (p.len_k) s.Lk = p.len_k[b] < 0 ? 0 : (p.len_k[b] > p.Lk ? p.Lk : p.len_k[b]);
  return s;
}

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int imax(int a, int b) { return a > b ? a : b; }
__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Key index of query row 0's causal diagonal.
__host__ __device__ inline int diag_off(const Problem& p) { return p.causal == 2 ? p.Lk - p.Lq : 0; }

// Keys [key_lo, key_hi) visible to query row i (empty when key_lo >= key_hi).
__host__ __device__ inline void row_key_range(const Problem& p, int i, int& key_lo, int& key_hi) {
  if (i >= p.Lq) {  // a row past the (sequence's) queries sees nothing
    key_lo = key_hi = 0;
    return;
  }
  const int off = diag_off(p);
  key_hi = p.causal ? imin(p.Lk, i + off + 1) : (p.window > 0 ? imin(p.Lk, i + p.window) : p.Lk);
  key_lo = p.window > 0 ? imax(0, i + off - p.window + 1) : 0;
}

// Key tiles [lo, hi) (tiles of bn keys) holding any key visible to any query
// row in [q0, q1).  Empty range: lo == hi == 0.
__host__ __device__ inline void kv_tile_range(const Problem& p, int q0, int q1, int bn, int& lo, int& hi) {
  q1 = imin(q1, p.Lq);
  lo = hi = 0;
  if (q0 >= q1) return;
  const int off = diag_off(p);
  // The last row reaches furthest forward, the first row furthest back.
  const int key_hi = p.causal ? imin(p.Lk, q1 + off) : (p.window > 0 ? imin(p.Lk, q1 - 1 + p.window) : p.Lk);
  const int key_lo = p.window > 0 ? imax(0, q0 + off - p.window + 1) : 0;
  if (key_lo >= key_hi) return;
  lo = key_lo / bn;
  hi = cdiv(key_hi, bn);
}

// Query rows [q_lo, q_hi) that see any key in [k0, k1) (backward pass).
__host__ __device__ inline void q_row_range(const Problem& p, int k0, int k1, int& q_lo, int& q_hi) {
  k1 = imin(k1, p.Lk);
  q_lo = q_hi = 0;
  if (k0 >= k1) return;
  const int off = diag_off(p);
  // j <= i + off  =>  i >= k0 - off;  two-sided band: j < i + w  =>  i > k0 - w
  int lo = p.causal ? imax(0, k0 - off) : (p.window > 0 ? imax(0, k0 - p.window + 1) : 0);
  // j > i + off - w  =>  i < j - off + w
  int hi = p.window > 0 ? imin(p.Lq, (k1 - 1) - off + p.window) : p.Lq;
  if (lo >= hi) return;
  q_lo = lo;
  q_hi = hi;
}

}  // namespace tea

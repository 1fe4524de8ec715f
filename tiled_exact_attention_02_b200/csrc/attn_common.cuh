// attn_common.cuh - problem description and mask/tile classification shared by
// the forward and backward kernels and their host-side launchers.
//
// Visibility ("注意力优化：FlashAttention 与稀疏注意力", 公式速览: disallowed keys
// get -inf before the softmax; "高效注意力" §4: sliding window):
//   key j is visible to query i  iff  (!causal || j <= i)
//                                 && (window <= 0 || j > i - window)
//                                 && (causal || window <= 0 || j < i + window)
// i.e. a window is the w keys ending at i under a causal mask, and the
// two-sided band of w - 1 keys on either side of i without one.
// A tile of keys is skipped when no key in it is visible to any row of the
// query tile, processed without masking when every key is visible to every
// row, and masked element-wise otherwise.
#pragma once
#include <cuda.h>
#include <cstdint>

namespace tea {

struct Problem {
  int B, Hq, Hkv, Lq, Lk, d;
  int causal, window;
  float scale;
};

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int imax(int a, int b) { return a > b ? a : b; }
__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Keys [key_lo, key_hi) visible to query row i (may be empty).
__host__ __device__ inline void row_key_range(const Problem& p, int i, int& key_lo, int& key_hi) {
  key_hi = p.causal ? imin(p.Lk, i + 1) : (p.window > 0 ? imin(p.Lk, i + p.window) : p.Lk);
  key_lo = p.window > 0 ? imax(0, i - p.window + 1) : 0;
}

// Key tiles [lo, hi) (tiles of bn keys) holding any key visible to any query
// row in [q0, q1).  Empty range: lo == hi == 0.
__host__ __device__ inline void kv_tile_range(const Problem& p, int q0, int q1, int bn, int& lo, int& hi) {
  q1 = imin(q1, p.Lq);
  lo = hi = 0;
  if (q0 >= q1) return;
  // The last row reaches furthest forward.
  const int key_hi = p.causal ? imin(p.Lk, q1) : (p.window > 0 ? imin(p.Lk, q1 - 1 + p.window) : p.Lk);
  const int key_lo = p.window > 0 ? imax(0, q0 - p.window + 1) : 0;  // first row reaches furthest back
  if (key_lo >= key_hi) return;
  lo = key_lo / bn;
  hi = cdiv(key_hi, bn);
}

// Query rows [q_lo, q_hi) that see any key in [k0, k1) (backward pass).
__host__ __device__ inline void q_row_range(const Problem& p, int k0, int k1, int& q_lo, int& q_hi) {
  k1 = imin(k1, p.Lk);
  q_lo = q_hi = 0;
  if (k0 >= k1) return;
  // j <= i  =>  i >= k0;  two-sided band: j < i + w  =>  i > k0 - w
  int lo = p.causal ? k0 : (p.window > 0 ? imax(0, k0 - p.window + 1) : 0);
  int hi = p.window > 0 ? imin(p.Lq, (k1 - 1) + p.window) : p.Lq;  // j > i - w  =>  i < j + w
  if (lo >= hi) return;
  q_lo = lo;
  q_hi = hi;
}

}  // namespace tea

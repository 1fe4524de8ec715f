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
  // Global key positions ("大模型高效注意力机制全解析" §5.1.2 global_tokens
  // [0, -1]): the first global_head and the last global_tail keys of a
  // sequence are visible to every query besides the window, still subject
  // to the causal mask.
  int global_head = 0;
  int global_tail = 0;
  // Block-sparse mask ("大模型高效注意力机制全解析" §4.1.2), block size b
  // (0: none): intersected with the causal and window masks.
  int sparse_block = 0;
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

__host__ __device__ inline bool has_global(const Problem& p) { return p.global_head > 0 || p.global_tail > 0; }
// First key of the global tail (Lk when there is none).
__host__ __device__ inline int tail_start(const Problem& p) { return imax(0, p.Lk - p.global_tail); }

// Key j visible to query i through the global positions (not through the band).
__host__ __device__ inline bool global_visible(const Problem& p, int i, int j) {
  if (i >= p.Lq || j >= p.Lk) return false;
  if (!(j < p.global_head || j >= tail_start(p))) return false;
  return !p.causal || j <= i + diag_off(p);
}

// Block-sparse mask with b x b blocks: the page's construction sets, for the
// query block starting at s and every key start j in [s - b, s + b), the
// block of keys [j, j + b); their union is the key range
// [max(0, s - b), min(Lk, s + 2b - 1)), the same for every row of the block.
__host__ __device__ inline int sparse_key_lo(const Problem& p, int i) {
  const int b = p.sparse_block;
  return imax(0, i / b * b - b);
}
__host__ __device__ inline int sparse_key_hi(const Problem& p, int i) {
  const int b = p.sparse_block;
  return imin(p.Lk, i / b * b + 2 * b - 1);
}
// Query rows [lo, hi) whose block-sparse key range meets keys [k0, k1)
// (k0 < k1): block starts s with s + 2b - 1 > k0 and s - b < k1.
__host__ __device__ inline void sparse_key_rows(const Problem& p, int k0, int k1, int& lo, int& hi) {
  const int b = p.sparse_block;
  const int t = k0 - 2 * b + 2;  // smallest admissible block start, before rounding up to a block
  lo = t <= 0 ? 0 : cdiv(t, b) * b;
  hi = (cdiv(k1, b) + 1) * b;
}

// The key tiles a query tile walks, as three ranges in walk order: the global
// head tiles, the window band, the global tail tiles (an empty range has
// lo == hi).  norm() merges overlapping or touching ranges, so the walk is
// sorted and visits no tile twice.  Every index below is a constant, so the
// ranges stay in registers.
struct Segs {
  int lo[3] = {0, 0, 0}, hi[3] = {0, 0, 0};
  __host__ __device__ bool empty(int k) const { return lo[k] >= hi[k]; }
  __host__ __device__ int count() const {
    return (hi[0] - lo[0]) * !empty(0) + (hi[1] - lo[1]) * !empty(1) + (hi[2] - lo[2]) * !empty(2);
  }
  __host__ __device__ bool any() const { return !empty(0) || !empty(1) || !empty(2); }
  // Tile at position t of the walk (t < count()).
  __host__ __device__ int at(int t) const {
    int r = -1;
#pragma unroll
    for (int k = 0; k < 3; k++) {
      if (!empty(k) && r < 0) {
        const int len = hi[k] - lo[k];
        if (t < len) r = lo[k] + t;
        else t -= len;
      }
    }
    return r;
  }
  __host__ __device__ bool contains(int j) const {
    bool c = false;
#pragma unroll
    for (int k = 0; k < 3; k++)
      if (j >= lo[k] && j < hi[k]) c = true;
    return c;
  }
  // Merge range b into range a if they overlap or touch (both non-empty).
  __host__ __device__ void merge(int a, int b) {
    if (empty(a) || empty(b) || hi[a] < lo[b] || hi[b] < lo[a]) return;
    lo[a] = lo[a] < lo[b] ? lo[a] : lo[b];
    hi[a] = hi[a] > hi[b] ? hi[a] : hi[b];
    lo[b] = hi[b] = 0;
  }
  __host__ __device__ void norm() {
#pragma unroll
    for (int k = 0; k < 3; k++)
      if (empty(k)) lo[k] = hi[k] = 0;
    merge(1, 0);  // head into band
    merge(1, 2);  // tail into band
    merge(0, 2);  // tail into head (when the band is empty)
    merge(1, 0);  // a grown head into the band
  }
  // Range-wise union with another walk of the same shape.
  __host__ __device__ void unite(const Segs& o) {
#pragma unroll
    for (int k = 0; k < 3; k++) {
      if (o.empty(k)) continue;
      if (empty(k)) {
        lo[k] = o.lo[k], hi[k] = o.hi[k];
      } else {
        lo[k] = lo[k] < o.lo[k] ? lo[k] : o.lo[k];
        hi[k] = hi[k] > o.hi[k] ? hi[k] : o.hi[k];
      }
    }
    norm();
  }
  // Keep only tiles in [a, b).
  __host__ __device__ void clip(int a, int b) {
#pragma unroll
    for (int k = 0; k < 3; k++) {
      lo[k] = lo[k] > a ? lo[k] : a;
      hi[k] = hi[k] < b ? hi[k] : b;
      if (lo[k] >= hi[k]) lo[k] = hi[k] = 0;
    }
  }
};

// Keys [key_lo, key_hi) visible to query row i (empty when key_lo >= key_hi).
__host__ __device__ inline void row_key_range(const Problem& p, int i, int& key_lo, int& key_hi) {
  if (i >= p.Lq) {  // a row past the (sequence's) queries sees nothing
    key_lo = key_hi = 0;
    return;
  }
  const int off = diag_off(p);
  key_hi = p.causal ? imin(p.Lk, i + off + 1) : (p.window > 0 ? imin(p.Lk, i + p.window) : p.Lk);
  key_lo = p.window > 0 ? imax(0, i + off - p.window + 1) : 0;
  if (p.sparse_block > 0) {
    key_lo = imax(key_lo, sparse_key_lo(p, i));
    key_hi = imin(key_hi, sparse_key_hi(p, i));
  }
}

// Keys [key_lo, key_hi) spanning every key visible to any query row in
// [q0, q1) (the band; global keys not included).  Empty: key_lo >= key_hi.
__host__ __device__ inline void kv_key_range(const Problem& p, int q0, int q1, int& key_lo, int& key_hi) {
  q1 = imin(q1, p.Lq);
  key_lo = key_hi = 0;
  if (q0 >= q1) return;
  const int off = diag_off(p);
  // The last row reaches furthest forward, the first row furthest back.
  key_hi = p.causal ? imin(p.Lk, q1 + off) : (p.window > 0 ? imin(p.Lk, q1 - 1 + p.window) : p.Lk);
  key_lo = p.window > 0 ? imax(0, q0 + off - p.window + 1) : 0;
  if (p.sparse_block > 0) {
    // Both ends of every mask's key range only grow with the row.
    key_lo = imax(key_lo, sparse_key_lo(p, q0));
    key_hi = imin(key_hi, sparse_key_hi(p, q1 - 1));
  }
}

// Key tiles [lo, hi) (tiles of bn keys) holding any key visible to any query
// row in [q0, q1).  Empty range: lo == hi == 0.
__host__ __device__ inline void kv_tile_range(const Problem& p, int q0, int q1, int bn, int& lo, int& hi) {
  int key_lo, key_hi;
  kv_key_range(p, q0, q1, key_lo, key_hi);
  lo = hi = 0;
  if (key_lo >= key_hi) return;
  lo = key_lo / bn;
  hi = cdiv(key_hi, bn);
}

// Key tiles (of bn keys) holding any key visible to any query row in
// [q0, q1): the band of kv_tile_range plus the tiles of the global head and
// tail keys those rows may see.
__host__ __device__ inline Segs kv_tile_segs(const Problem& p, int q0, int q1, int bn) {
  Segs s;
  kv_tile_range(p, q0, q1, bn, s.lo[1], s.hi[1]);
  q1 = imin(q1, p.Lq);
  if (has_global(p) && q0 < q1) {
    // Under a causal mask the last row sees the most keys.
    const int lim = p.causal ? imin(p.Lk, q1 + diag_off(p)) : p.Lk;
    const int h = imin(p.global_head, lim);
    if (h > 0) s.lo[0] = 0, s.hi[0] = cdiv(h, bn);
    const int t0 = tail_start(p);
    if (p.global_tail > 0 && t0 < lim) s.lo[2] = t0 / bn, s.hi[2] = cdiv(lim, bn);
  }
  s.norm();
  return s;
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
  if (p.sparse_block > 0) {
    int slo, shi;
    sparse_key_rows(p, k0, k1, slo, shi);
    lo = imax(lo, slo);
    hi = imin(hi, shi);
  }
  // A global key in the tile is seen by every row (every row at or past it
  // under a causal mask); the band's rows lie inside that range.
  if (has_global(p)) {
    int jg = -1;
    if (k0 < p.global_head) jg = k0;
    else if (k1 > tail_start(p)) jg = imax(k0, tail_start(p));
    if (jg >= 0) {
      const int glo = p.causal ? imax(0, jg - off) : 0;
      if (glo < p.Lq) {
        lo = lo < hi ? imin(lo, glo) : glo;
        hi = p.Lq;
      }
    }
  }
  if (lo >= hi) return;
  q_lo = lo;
  q_hi = hi;
}

}  // namespace tea

// attn_fwd.cu - forward attention kernel for sm_100a.
//
// Algorithm ("缩放定律与高效注意力" §3.2; "高效注意力：FlashAttention 与线性注意力",
// 原理与机制): for a tile of 128 query rows, stream the visible key/value tiles
// of 128 keys, compute S = Q K^T on the tensor cores into tensor memory, keep
// a running row max m and row sum l, turn S into P = exp(scale*S - m) and
// accumulate O += P V, rescaling O and l by e^{m_old - m_new} when m grows.
// Only O (divided by l) and LSE = m + log l leave the chip.
//
// B200 mapping (one CTA per SM, 384 threads, 12 warps):
//   warp 0      TMA producer: two Q tiles, then a ring of K/V tiles
//   warp 1      tcgen05 issuer (one elected thread) and TMEM owner
//   warps 4-7   softmax for query slot 0 (thread = query row)
//   warps 8-11  softmax for query slot 1
// A CTA holds two query tiles ("slots") that share every K/V tile it loads:
// two heads of one GQA group at the same rows when the group size is even
// (K/V reuse across the group), otherwise two consecutive row tiles of one
// head.  Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 columns each; the
// bf16 P of a slot overwrites the first 64 columns of its S after S has been
// read, and feeds the P.V MMA straight from tensor memory.  While one slot's
// softmax runs, the tensor cores work on the other slot's P.V and next
// Q.K^T, so the exponentials of one slot overlap the MMAs of the other.
//
// Rescaling is lazy: a row's reference max is only raised when the new max
// exceeds it by more than 8 (in log2 units).  Any reference value gives the
// same O/l; keeping p <= 2^8 bounds the bf16 P and fp32 accumulators.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cmath>

#include "sm100.cuh"
#include "attn_common.cuh"
#include "attn_kernels.h"

namespace tea {

namespace fwd {

constexpr int BM = 128;        // query rows per slot
constexpr int BN = 128;        // keys per K/V tile
constexpr int THREADS = 384;
constexpr int PANEL = 16384;   // one 128-row x 128-byte swizzled panel
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int D>
struct Cfg {
  static constexpr int PANELS = D / 64;
  static constexpr int TILE = BM * D * 2;         // bytes of one Q, K or V tile
  static constexpr int NST = D == 128 ? 5 : 8;    // K/V ring stages (2.5 key tiles ahead at d = 128)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * TILE;
  static constexpr int OFF_BAR = OFF_KV + NST * TILE;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;  // barriers + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(NST <= 8, "barrier arrays");
};

struct Bars {
  uint64_t q_full[2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t merge;       // alternating slots: slot 1's row max and sum are in shared memory [4 warps]
  uint64_t drain;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
};

// TMEM columns of slot s: S (and P) at s_col(s), O at o_col(s).
__device__ __forceinline__ uint32_t s_col(int s) { return 128u * s; }
__device__ __forceinline__ uint32_t o_col(int s) { return 256u + 128u * s; }

// One CTA's work: two query tiles (slots).
struct Unit {
  int b, kvh;
  int head[2];
  int q0[2];
  Segs seg[2];       // key tiles of each slot, in walk order (band, plus global head/tail tiles)
  Segs useg;         // their union: the tiles the CTA streams
  int split;         // key-range slice of a split problem (0 otherwise)
  int alt;           // 1: both slots hold the same rows and take alternate key tiles of one range
  int down;          // 1: the walk runs from its last tile down (block-sparse masks, no global tokens)
  int koff;          // key tile j holds keys [j*BN + koff, (j+1)*BN + koff) (block-sparse masks; else 0)
};

// Walk accessors.  W = false (no global tokens): the walk is the band alone,
// which kv_tile_segs always keeps in range 1, so every accessor is the plain
// contiguous-range arithmetic and the rest of Segs is dead code.  Under a
// block-sparse mask the band is walked from its last tile down (`down`): on a
// B200 that measured 8% faster for 64-row blocks, while the causal and
// window workloads measured the same or slower that way, so they walk up.
template <bool W>
__device__ __forceinline__ int walk_count(const Segs& s) {
  if constexpr (W) return s.count();
  else return s.hi[1] > s.lo[1] ? s.hi[1] - s.lo[1] : 0;
}
template <bool W>
__device__ __forceinline__ int walk_at(const Segs& s, int t, bool down) {
  if constexpr (W) return s.at(t);
  else return down ? s.hi[1] - 1 - t : s.lo[1] + t;
}
template <bool W>
__device__ __forceinline__ bool walk_has(const Segs& s, int j) {
  if constexpr (W) return s.contains(j);
  else return j >= s.lo[1] && j < s.hi[1];
}

// Key tiles of query rows [q0, q1) as a walk.  Without global tokens the walk
// is the band alone (range 1), built directly: the general form's range
// merging is a long chain of dependent integer operations that every thread
// of a CTA runs before its first copy can start.
template <bool W>
__device__ __forceinline__ Segs tile_walk(const Problem& ps, int q0, int q1, int koff) {
  if constexpr (W) {
    return kv_tile_segs(ps, q0, q1, BN);
  } else {
    Segs s;
    int key_lo, key_hi;
    kv_key_range(ps, q0, q1, key_lo, key_hi);
    if (key_lo < key_hi) {
      s.lo[1] = (key_lo - koff) / BN;
      s.hi[1] = cdiv(key_hi - koff, BN);
    }
    return s;
  }
}

// Offset of the key-tile grid.  Under a block-sparse mask the band of a row
// tile starts on a block boundary, which need not be a tile boundary: 64-row
// blocks give 128-row tiles a band of 256 keys starting 64 keys before a tile
// boundary, three tiles on the aligned grid but two on a grid shifted by 64.
// So the grid starts at the unit's first visible key (mod BN); copies of the
// keys before 0 or past Lk read the tensor map's zero fill and are masked.
// Other masks keep the aligned grid.  koff <= every slot's first key.
template <bool W, bool DN>
__device__ __forceinline__ int grid_offset(const Problem& ps, int qa0, int qb0, int qa1, int qb1) {
  if (W || !DN || ps.sparse_block <= 0) return 0;
  int a0, b0, a1, b1;
  kv_key_range(ps, qa0, qb0, a0, b0);
  kv_key_range(ps, qa1, qb1, a1, b1);
  if (a0 >= b0 && a1 >= b1) return 0;
  const int lo = a0 >= b0 ? a1 : (a1 >= b1 ? a0 : imin(a0, a1));
  return lo % BN;
}

// The union of the two slots' walks (what the CTA streams); without global
// tokens the tiles between the two bands' ends.
template <bool W>
__device__ __forceinline__ Segs union_walk(const Segs& a, const Segs& b) {
  Segs u = a;
  if constexpr (W) {
    u.unite(b);
  } else if (b.lo[1] < b.hi[1]) {
    if (u.lo[1] < u.hi[1]) {
      u.lo[1] = imin(u.lo[1], b.lo[1]);
      u.hi[1] = imax(u.hi[1], b.hi[1]);
    } else {
      u.lo[1] = b.lo[1];
      u.hi[1] = b.hi[1];
    }
  }
  return u;
}

// Packed rows (short queries): row r of kv group (b, kvh) is query r % Lq of
// head kvh*G + r / Lq, i.e. Q read as [B*Hkv, G*Lq, d]; each unit takes two
// consecutive 128-row tiles of a group.  A tile inside one head sees the key
// tiles of its own query rows, a tile across heads those of all Lq rows.
template <bool W, bool DN>
__device__ __forceinline__ Unit decode_unit_packed(const FwdParams& P, int idx) {
  const Problem& p = P.prob;
  Unit u;
  const int G = p.Hq / p.Hkv;
  const int R = G * p.Lq;
  const int nq = cdiv(cdiv(R, BM), 2);
  const int grp = idx / nq;
  u.b = grp / p.Hkv;
  u.kvh = grp % p.Hkv;
  const int qi = idx % nq;
  const Problem ps = seq_problem(p, u.b);
  // Query rows of each slot's tile: its own rows inside one head, all Lq rows
  // of a head when it spans several.
  int qa[2], qb[2];
#pragma unroll
  for (int s = 0; s < 2; s++) {
    const int r0 = (2 * qi + s) * BM;
    const int r1 = imin(r0 + BM, R);
    u.head[s] = u.kvh * G;
    u.q0[s] = r0;
    if (r0 >= r1) {
      qa[s] = qb[s] = 0;
    } else if (r0 / p.Lq != (r1 - 1) / p.Lq) {
      qa[s] = 0;
      qb[s] = p.Lq;
    } else {
      qa[s] = r0 % p.Lq;
      qb[s] = (r1 - 1) % p.Lq + 1;
    }
  }
  u.koff = grid_offset<W, DN>(ps, qa[0], qb[0], qa[1], qb[1]);
#pragma unroll
  for (int s = 0; s < 2; s++) u.seg[s] = qa[s] < qb[s] ? tile_walk<W>(ps, qa[s], qb[s], u.koff) : Segs{};
  u.useg = union_walk<W>(u.seg[0], u.seg[1]);
  return u;
}

// A unit whose second slot would hold no rows instead gives both slots the
// first slot's rows; slot s then takes the key tiles at even (s = 0) or odd
// (s = 1) positions of the walk, and the two partial softmaxes are merged in
// the epilogue.  The two chains of softmax and MMAs then run side by side.
__device__ __forceinline__ void make_alternating(Unit& u) {
  u.alt = 1;
  u.q0[1] = u.q0[0];
  u.head[1] = u.head[0];
  u.seg[1] = u.seg[0];
  u.useg = u.seg[0];
}

template <bool W, bool DN>
__device__ __forceinline__ Unit decode_unit(const FwdParams& P, int idx) {
  if (P.packed) {
    Unit u = decode_unit_packed<W, DN>(P, idx);
    u.down = DN;
    u.alt = 0;
    if (P.alternate) make_alternating(u);
    return u;
  }
  const Problem& p = P.prob;
  Unit u;
  const int G = p.Hq / p.Hkv;
  const int nqt = cdiv(p.Lq, BM);
  // Work is grouped by heads (up to 8 head units per group, so the CTAs
  // running at one time share the K/V of a few heads in L2); inside a group
  // the query tiles go from last to first (late rows see the most keys under
  // a causal mask: heavy first).
  const int nh = P.pair_heads ? p.B * (p.Hq / 2) : p.B * p.Hq;  // head units
  const int nq = P.pair_heads ? nqt : cdiv(nqt, 2);              // query units per head unit
  constexpr int HG = 8;
  const int grp = idx / (HG * nq);
  const int hg = imin(HG, nh - grp * HG);
  const int rem = idx - grp * HG * nq;
  const int qi = nq - 1 - rem / hg;
  const int hu = grp * HG + rem % hg;
  if (P.pair_heads) {
    // Two heads of one GQA group, same query rows.
    u.b = hu / (p.Hq / 2);
    const int hp = hu % (p.Hq / 2);
    u.head[0] = 2 * hp;
    u.head[1] = 2 * hp + 1;
    u.q0[0] = u.q0[1] = qi * BM;
  } else {
    // Two consecutive row tiles of one head.  The later tile (under a causal
    // mask the one that sees one more key tile) takes slot 0, whose MMAs the
    // issuer takes first at each key tile: measured about 2.5% faster on a
    // causal 4096 workload.  Block-sparse masks (walked downwards) measured
    // 10% faster the other way round, and with alternating slots slot 0 must
    // hold the unit's only tile.
    const bool later_first = !P.alternate && p.sparse_block == 0;
    u.b = hu / p.Hq;
    u.head[0] = u.head[1] = hu % p.Hq;
    u.q0[0] = qi * 2 * BM + (later_first ? BM : 0);
    u.q0[1] = qi * 2 * BM + (later_first ? 0 : BM);
  }
  u.kvh = u.head[0] / G;
  const Problem ps = seq_problem(p, u.b);  // this sequence's lengths (padded batches)
  u.koff = grid_offset<W, DN>(ps, u.q0[0], u.q0[0] + BM, u.q0[1], u.q0[1] + BM);
  u.seg[0] = tile_walk<W>(ps, u.q0[0], u.q0[0] + BM, u.koff);
  u.seg[1] = tile_walk<W>(ps, u.q0[1], u.q0[1] + BM, u.koff);
  u.useg = union_walk<W>(u.seg[0], u.seg[1]);
  u.down = DN;
  u.alt = 0;
  if (P.alternate) make_alternating(u);
  return u;
}

// Unit of CTA `idx` when every unit's key walk is cut into n_split slices
// (consecutive CTAs take the slices of one unit): slice k keeps positions
// [k*n/ns, (k+1)*n/ns) of the union walk (n tiles), i.e. the tiles between
// the first and last of them, in each slot's walk as well.  An empty slice
// leaves both slots empty.
template <bool W, bool DN>
__device__ __forceinline__ Unit decode_unit_split(const FwdParams& P, int idx) {
  if (P.n_split <= 1) {
    Unit u = decode_unit<W, DN>(P, idx);
    u.split = 0;
    return u;
  }
  Unit u = decode_unit<W, DN>(P, idx / P.n_split);
  u.split = idx % P.n_split;
  const int n = walk_count<W>(u.useg);
  const int p0 = (int)((long long)u.split * n / P.n_split);
  const int p1 = (int)((long long)(u.split + 1) * n / P.n_split);
  // Tiles between the slice's first and last (either order, as the walk runs).
  int a = 0, b = 0;
  if (p0 < p1) {
    const int ja = walk_at<W>(u.useg, p0, u.down), jb = walk_at<W>(u.useg, p1 - 1, u.down);
    a = imin(ja, jb);
    b = imax(ja, jb) + 1;
  }
  u.useg.clip(a, b);
  u.seg[0].clip(a, b);
  u.seg[1].clip(a, b);
  return u;
}

// Slot walks: with alternating slots (never with global tokens) slot s takes
// positions s, s + 2, ... of the one contiguous range.
template <bool W>
__device__ __forceinline__ bool active(const Unit& u, int s, int j) {
  if (!W && u.alt)
    return walk_has<W>(u.seg[s], j) && ((u.down ? u.seg[s].hi[1] - 1 - j : j - u.seg[s].lo[1]) & 1) == s;
  return walk_has<W>(u.seg[s], j);
}
template <bool W>
__device__ __forceinline__ int slot_count(const Unit& u, const Segs& sg, int s) {
  const int n = walk_count<W>(sg);
  return (!W && u.alt) ? (n + 1 - s) / 2 : n;
}
template <bool W>
__device__ __forceinline__ int slot_at(const Unit& u, const Segs& sg, int s, int i) {
  if (!W && u.alt) return u.down ? sg.hi[1] - 1 - (2 * i + s) : sg.lo[1] + 2 * i + s;
  return walk_at<W>(sg, i, u.down);
}

// ------------------------------------------------------------------ producer
template <int D, bool W>
__device__ void producer(const FwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, const WaitGuard& g) {
  using C = Cfg<D>;
  const Problem& p = P.prob;
  tma_prefetch_desc(&P.tm_q);
  tma_prefetch_desc(&P.tm_k);
  tma_prefetch_desc(&P.tm_v);
#pragma unroll
  for (int s = 0; s < 2; s++) {
    if (walk_count<W>(u.seg[s]) == 0 || (s == 1 && u.alt)) continue;  // alternating slots share slot 0's Q
    mbar_arrive_expect_tx(&bars.q_full[s], C::TILE);
    for (int pnl = 0; pnl < C::PANELS; pnl++)
      tma_load_3d(smem + C::OFF_Q + s * C::TILE + pnl * PANEL, &P.tm_q, &bars.q_full[s], pnl * 64, u.q0[s],
                  P.packed ? u.b * p.Hkv + u.kvh : u.b * p.Hq + u.head[s]);
  }
  int issued = 0;
  const int un = walk_count<W>(u.useg);
  for (int t = 0; t < un; t++) {
    const int j = walk_at<W>(u.useg, t, u.down);
    for (int which = 0; which < 2; which++) {
      const int r = 2 * t + which;
      const int st = r % C::NST;
      const uint32_t ph = (r / C::NST) & 1;
      if (!mbar_wait(&bars.kv_empty[st], ph ^ 1, g, 1)) goto drain;
      mbar_arrive_expect_tx(&bars.kv_full[st], C::TILE);
      for (int pnl = 0; pnl < C::PANELS; pnl++)
        tma_load_3d(smem + C::OFF_KV + st * C::TILE + pnl * PANEL, which ? &P.tm_v : &P.tm_k, &bars.kv_full[st],
                    pnl * 64, j * BN + u.koff, u.b * p.Hkv + u.kvh);
      issued = r + 1;
    }
  }
  return;
drain:
  // A wait was abandoned: let every copy this warp started land before the
  // CTA exits (bounded, independent of the other roles).
  {
    WaitGuard g2 = g;
    for (int r = imax(0, issued - C::NST); r < issued; r++) mbar_wait_ignore_abort(&bars.kv_full[r % C::NST], (r / C::NST) & 1, g2);
#pragma unroll
    for (int s = 0; s < 2; s++)
      if (walk_count<W>(u.seg[s]) > 0 && !(s == 1 && u.alt)) mbar_wait_ignore_abort(&bars.q_full[s], 0, g2);
  }
}

// ------------------------------------------------------------------ MMA issuer
template <int D, bool W>
__device__ void mma_issuer(const FwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, uint32_t tmem,
                           const WaitGuard& g) {
  using C = Cfg<D>;
  const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
  const uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
  // Descriptors are built once; a slice at byte offset `off` inside a tile is
  // the tile's descriptor plus off / 16 (start-address field, no carry).
  const uint64_t q_kmaj = sw128_desc(smem_u32(smem + C::OFF_Q), 16, 1024);
  const uint64_t kv_kmaj = sw128_desc(smem_u32(smem + C::OFF_KV), 16, 1024);
  const uint64_t kv_mn = sw128_desc(smem_u32(smem + C::OFF_KV), PANEL, 1024);
  auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
  const int un = walk_count<W>(u.useg);
  if (un == 0) return;

  // K of walk position t sits in ring slot 2t, V in 2t + 1.
  auto stage_of = [&](int t, int which) { return (2 * t + which) % C::NST; };
  auto phase_of = [&](int t, int which) { return (uint32_t)(((2 * t + which) / C::NST) & 1); };

  auto issue_s = [&](int s, int t) {
    const uint64_t qd = adv(q_kmaj, s * C::TILE);
    const uint64_t kd = adv(kv_kmaj, stage_of(t, 0) * C::TILE);
#pragma unroll
    for (int kk = 0; kk < D / 16; kk++) {
      const uint32_t off = (kk / 4) * PANEL + (kk % 4) * 32;
      mma_ss(tmem + s_col(s), adv(qd, off), adv(kd, off), idesc_qk, kk > 0);
    }
    mma_commit(&bars.s_full[s]);
  };
  // Tiles of each slot's walk done so far, and the walk lengths.
  int done0 = 0, done1 = 0;
  const int n0 = walk_count<W>(u.seg[0]), n1 = walk_count<W>(u.seg[1]);

  for (int s = 0; s < 2; s++)
    if (walk_count<W>(u.seg[s]) > 0 && !mbar_wait(&bars.q_full[s], 0, g, 10)) goto out;

  {
    // Prologue: S for the first tile of the walk.
    const int j0 = walk_at<W>(u.useg, 0, u.down);
    if (!mbar_wait(&bars.kv_full[stage_of(0, 0)], phase_of(0, 0), g, 11)) goto out;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 2; s++)
      if (active<W>(u, s, j0)) issue_s(s, 0);
    mma_commit(&bars.kv_empty[stage_of(0, 0)]);
  }

  for (int t = 0; t < un; t++) {
    const int j = walk_at<W>(u.useg, t, u.down);
    if (!mbar_wait(&bars.kv_full[stage_of(t, 1)], phase_of(t, 1), g, 12)) goto out;
    const bool next = t + 1 < un;
    const int jn = next ? walk_at<W>(u.useg, t + 1, u.down) : -1;
    if (next) {
      if (!mbar_wait(&bars.kv_full[stage_of(t + 1, 0)], phase_of(t + 1, 0), g, 13)) goto out;
    }
    const uint64_t vd = adv(kv_mn, stage_of(t, 1) * C::TILE);
#pragma unroll
    for (int s = 0; s < 2; s++) {
      if (active<W>(u, s, j)) {
        const int done = s ? done1 : done0;
        const int ns = s ? n1 : n0;
        if (!mbar_wait(&bars.p_full[s], done & 1, g, 14 + s)) goto out;
        tc_fence_after();
        const uint32_t acc0 = done > 0;
#pragma unroll
        for (int kk = 0; kk < BN / 16; kk++)
          mma_ts(tmem + o_col(s), tmem + s_col(s) + kk * 8, adv(vd, kk * 2048), idesc_pv, kk > 0 ? 1u : acc0);
        if (done == ns - 1) mma_commit(&bars.o_full[s]);
        if (s) done1++; else done0++;
      }
      if (next && active<W>(u, s, jn)) issue_s(s, t + 1);
    }
    mma_commit(&bars.kv_empty[stage_of(t, 1)]);
    if (next) mma_commit(&bars.kv_empty[stage_of(t + 1, 0)]);
  }
out:
  // Drain: wait until every MMA this thread issued has completed.
  mma_commit(&bars.drain);
  mbar_wait_ignore_abort(&bars.drain, 0, g);
}

// ------------------------------------------------------------------ MMA issuer, alternating slots
// Walk position t belongs to slot t & 1 and both slots read slot 0's Q.  The
// S of a slot's next tile (position t + 2) is issued right after the P.V of
// its current one, so while one slot's softmax runs the other slot's MMAs
// have the tensor cores.
template <int D>
__device__ void mma_issuer_alt(const FwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, uint32_t tmem,
                               const WaitGuard& g) {
  using C = Cfg<D>;
  const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
  const uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
  const uint64_t q_kmaj = sw128_desc(smem_u32(smem + C::OFF_Q), 16, 1024);
  const uint64_t kv_kmaj = sw128_desc(smem_u32(smem + C::OFF_KV), 16, 1024);
  const uint64_t kv_mn = sw128_desc(smem_u32(smem + C::OFF_KV), PANEL, 1024);
  auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
  const int un = walk_count<false>(u.useg);
  if (un == 0) return;
  auto stage_of = [&](int t, int which) { return (2 * t + which) % C::NST; };
  auto phase_of = [&](int t, int which) { return (uint32_t)(((2 * t + which) / C::NST) & 1); };
  // S of slot s for walk position t (its K is in ring slot 2t); K released after.
  auto issue_s = [&](int s, int t) -> bool {
    if (!mbar_wait(&bars.kv_full[stage_of(t, 0)], phase_of(t, 0), g, 11)) return false;
    tc_fence_after();
    const uint64_t kd = adv(kv_kmaj, stage_of(t, 0) * C::TILE);
#pragma unroll
    for (int kk = 0; kk < D / 16; kk++) {
      const uint32_t off = (kk / 4) * PANEL + (kk % 4) * 32;
      mma_ss(tmem + s_col(s), adv(q_kmaj, off), adv(kd, off), idesc_qk, kk > 0);
    }
    mma_commit(&bars.s_full[s]);
    mma_commit(&bars.kv_empty[stage_of(t, 0)]);
    return true;
  };

  if (!mbar_wait(&bars.q_full[0], 0, g, 10)) goto out;
  if (!issue_s(0, 0)) goto out;
  if (un > 1 && !issue_s(1, 1)) goto out;
  for (int t = 0; t < un; t++) {
    const int s = t & 1;
    if (!mbar_wait(&bars.kv_full[stage_of(t, 1)], phase_of(t, 1), g, 12)) goto out;
    if (!mbar_wait(&bars.p_full[s], (t >> 1) & 1, g, 14 + s)) goto out;
    tc_fence_after();
    {
      const uint64_t vd = adv(kv_mn, stage_of(t, 1) * C::TILE);
      const uint32_t acc0 = t >= 2;
#pragma unroll
      for (int kk = 0; kk < BN / 16; kk++)
        mma_ts(tmem + o_col(s), tmem + s_col(s) + kk * 8, adv(vd, kk * 2048), idesc_pv, kk > 0 ? 1u : acc0);
    }
    if (t + 2 >= un) mma_commit(&bars.o_full[s]);
    mma_commit(&bars.kv_empty[stage_of(t, 1)]);
    if (t + 2 < un && !issue_s(s, t + 2)) goto out;
  }
out:
  mma_commit(&bars.drain);
  mbar_wait_ignore_abort(&bars.drain, 0, g);
}

// ------------------------------------------------------------------ softmax
// One warpgroup per slot; thread `row` owns query row q0 + row and TMEM lane
// `row` (warp w of the group may only touch lanes 32*(w%4) .. +31).
template <int D, bool W>
__device__ void softmax_slot(const FwdParams& P, const Unit& u, int s, uint8_t* smem, Bars& bars, uint32_t tmem,
                             const WaitGuard& g) {
  const Problem& p = P.prob;
  const int wl = (threadIdx.x / 32) % 4;
  const int lane = threadIdx.x % 32;
  const int row = wl * 32 + lane;
  // Slot fields as scalars (a runtime index into Unit would put it in local memory).
  const Segs walk = s ? u.seg[1] : u.seg[0];  // this slot's key tiles, in order
  const int n_walk = slot_count<W>(u, walk, s);
  int head_s = s ? u.head[1] : u.head[0];
  int q_row = (s ? u.q0[1] : u.q0[0]) + row;
  if (P.packed) {
    // Packed rows: this row's head and query; rows past the group's last
    // (the tile's zero-filled tail) get q_row = Lq, which sees nothing and is not written.
    const int pr = q_row;
    const int G = p.Hq / p.Hkv;
    head_s += pr / p.Lq;
    q_row = pr < G * p.Lq ? pr % p.Lq : p.Lq;
  }
  int key_lo, key_hi;  // the row's band
  int gh_hi = 0, gt_lo = 0, gt_hi = 0;  // global keys it also sees: [0, gh_hi) and [gt_lo, gt_hi)
  {
    const Problem ps = seq_problem(p, u.b);  // this sequence's lengths and masks
    row_key_range(ps, q_row, key_lo, key_hi);
    if (W && has_global(ps) && q_row < ps.Lq) {
      const int lim = ps.causal ? imin(ps.Lk, q_row + diag_off(ps) + 1) : ps.Lk;
      gh_hi = imin(ps.global_head, lim);
      gt_lo = tail_start(ps);
      gt_hi = ps.global_tail > 0 ? lim : 0;
      if (gt_hi <= gt_lo) gt_lo = gt_hi = 0;  // empty: the unsigned range test below needs lo <= hi
    }
    if (key_hi < key_lo) key_hi = key_lo;
  }
  const float c = P.scale_log2;
  const uint32_t lane_base = (uint32_t)(wl * 32) << 16;
  const uint32_t t_s = tmem + lane_base + s_col(s);
  const uint32_t t_o = tmem + lane_base + o_col(s);
  float m = -INFINITY;  // reference max, log2 units (scaled)
  float l = 0.f;        // running sum of exp2(c*S - m)

  for (int it = 0; it < n_walk; it++) {
    const int j = slot_at<W>(u, walk, s, it);
    if (!mbar_wait(&bars.s_full[s], it & 1, g, 20 + s)) return;
    tc_fence_after();
    uint32_t x[BN];
    // Element-wise mask only on tiles that straddle this row's visible range
    // (a per-row condition: it never guards a tcgen05 instruction, which the
    // whole warp must execute together).
    const int key0 = j * BN + u.koff;
    const bool masked = key0 < key_lo || key0 + BN > key_hi;
    auto mask_cols = [&](int c0, int c1) {
      if (W && (gh_hi > 0 || gt_hi > gt_lo)) {
        // Global keys on top of the band (rare: only global-token masks).
#pragma unroll
        for (int cc = c0; cc < c1; cc++) {
          const int key = key0 + cc;
          const bool vis = (unsigned)(key - key_lo) < (unsigned)(key_hi - key_lo) || key < gh_hi ||
                           (unsigned)(key - gt_lo) < (unsigned)(gt_hi - gt_lo);
          if (!vis) x[cc] = __float_as_uint(-INFINITY);
        }
      } else {
#pragma unroll
        for (int cc = c0; cc < c1; cc++) {
          const int key = key0 + cc;
          if (key < key_lo || key >= key_hi) x[cc] = __float_as_uint(-INFINITY);
        }
      }
    };
    float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
    auto max_cols = [&](int c0, int c1) {
#pragma unroll
      for (int cc = c0; cc < c1; cc += 8) {
        mx0 = max3(mx0, __uint_as_float(x[cc]), __uint_as_float(x[cc + 1]));
        mx1 = max3(mx1, __uint_as_float(x[cc + 2]), __uint_as_float(x[cc + 3]));
        mx2 = max3(mx2, __uint_as_float(x[cc + 4]), __uint_as_float(x[cc + 5]));
        mx3 = max3(mx3, __uint_as_float(x[cc + 6]), __uint_as_float(x[cc + 7]));
      }
    };
#pragma unroll
    for (int q = 0; q < BN / 32; q++) tmem_ld32p(t_s + 32 * q, x + 32 * q);
    tmem_wait_ld();
    if (masked) mask_cols(0, BN);
    max_cols(0, BN);
    const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
    const float m_cand = mx == -INFINITY ? -INFINITY : mx * c;
    const float m_new = fmaxf(m, m_cand);
    const bool need = m_new > m + RESCALE_THRESHOLD;
    const float alpha = need ? ex2_approx(m - m_new) : 1.f;
    if (need) {
      l *= alpha;
      m = m_new;
    }
    const float m_sub = m == -INFINITY ? 0.f : m;
    float s0 = 0.f, s1 = 0.f;
    // P packed two per 32-bit word, written over x[0 .. BN/2) as it goes
    // (x[2cc], x[2cc+1] are dead once read).
#pragma unroll
    for (int cc = 0; cc < BN / 2; cc++) {
      float a0, a1;
      fma2(a0, a1, __uint_as_float(x[2 * cc]), __uint_as_float(x[2 * cc + 1]), c, c, -m_sub, -m_sub);
      const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
      add2(s0, s1, s0, s1, p0, p1);
      x[cc] = pack_bf16x2(p0, p1);
    }
    l += s0 + s1;
    // P (bf16, two per column) replaces the first BN/2 columns of S.
    tmem_st32(t_s, x);
    tmem_st32(t_s + 32, x + 32);
    tmem_wait_st();
    if (__any_sync(0xffffffffu, need) && it > 0) {
      // O holds the sum over earlier tiles (the last P.V finished before this
      // S was produced) and the next P.V waits for p_full: bring O to the new
      // reference max now, after P is out of the registers.
#pragma unroll
      for (int q = 0; q < D / 32; q++) {
        uint32_t o[32];
        tmem_ld32p(t_o + 32 * q, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e++) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(t_o + 32 * q, o);
      }
      tmem_wait_st();
    }

    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.p_full[s]);
  }

  // Epilogue: O / l in bf16 and the natural-log LSE.
  const bool has = n_walk > 0;
  if (has) {
    if (!mbar_wait(&bars.o_full[s], 0, g, 22 + s)) return;
    tc_fence_after();
  }
  // Alternating slots: slot 1 hands its row max and sum to slot 0 through
  // shared memory (slot 1's Q tile, unused in this mode) and slot 0 merges
  // the two partial softmaxes: with M = max(m0, m1), O = O0 2^(m0-M) +
  // O1 2^(m1-M) and l = l0 2^(m0-M) + l1 2^(m1-M), exact up to rounding.
  float a_own = 1.f, a_oth = 0.f;
  bool oth = false;  // slot 1's O takes part
  const uint32_t t_o1 = tmem + lane_base + o_col(1);
  if (!W && u.alt) {
    float2* ml = reinterpret_cast<float2*>(smem + Cfg<D>::OFF_Q + Cfg<D>::TILE);
    if (s == 1) {
      ml[row] = make_float2(m, l);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.merge);
      return;
    }
    const int n1 = slot_count<W>(u, u.seg[1], 1);
    if (!mbar_wait(&bars.merge, 0, g, 26)) return;
    if (n1 > 0) {
      if (!mbar_wait(&bars.o_full[1], 0, g, 27)) return;
      tc_fence_after();
    }
    const float2 o1 = ml[row];
    const float M = fmaxf(m, o1.x);
    a_own = m == -INFINITY ? 0.f : ex2_approx(m - M);
    a_oth = (n1 == 0 || o1.x == -INFINITY) ? 0.f : ex2_approx(o1.x - M);
    oth = n1 > 0;
    l = l * a_own + o1.y * a_oth;
    m = M;
  }
  const bool write = q_row < p.Lq;
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  const float sc_own = a_own * inv_l, sc_oth = a_oth * inv_l;
  const size_t row_off = ((size_t)(u.b * p.Hq + head_s) * p.Lq + q_row);
  const float lse_row = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
  // Columns 16q .. 16q+15 of the row's normalised O (both slots' parts when merging).
  auto load_o = [&](int q, float (&f)[16]) {
    uint32_t o[16];
    if (has) {
      tmem_ld16(t_o + 16 * q, o);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; e++) f[e] = __uint_as_float(o[e]) * sc_own;
    } else {
#pragma unroll
      for (int e = 0; e < 16; e++) f[e] = 0.f;
    }
    if (oth) {
      tmem_ld16(t_o1 + 16 * q, o);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; e++) f[e] = fmaf(__uint_as_float(o[e]), sc_oth, f[e]);
    }
  };
  if (P.acc_mode) {
    // Running accumulators of earlier key blocks (ring attention): with the
    // old (O_a, LSE_a) and this block's (O_b, LSE_b), both normalised by
    // their own sums, M = max(LSE_a, LSE_b), w = exp(LSE - M):
    //   O = (w_a O_a + w_b O_b) / (w_a + w_b),  LSE = M + log(w_a + w_b),
    // the rescale of the online softmax applied to whole key blocks.  Each
    // row belongs to one CTA, so the read-modify-write does not race.
    float* accp = P.part_o + row_off * D;
    const float l_old = (write && !P.acc_init) ? P.part_lse[row_off] : -INFINITY;
    const float M = fmaxf(l_old, lse_row);
    const float w_old = l_old == -INFINITY ? 0.f : expf(l_old - M);
    const float w_new = lse_row == -INFINITY ? 0.f : expf(lse_row - M);
    const float wsum = w_old + w_new;
    const float c_old = wsum > 0.f ? w_old / wsum : 0.f, c_new = wsum > 0.f ? w_new / wsum : 0.f;
#pragma unroll
    for (int q = 0; q < D / 16; q++) {
      float f[16];
      load_o(q, f);
      if (write) {
        float4* a4 = reinterpret_cast<float4*>(accp + q * 16);
#pragma unroll
        for (int v = 0; v < 4; v++) {
          float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (w_old > 0.f) o4 = a4[v];
          a4[v] = make_float4(o4.x * c_old + f[4 * v] * c_new, o4.y * c_old + f[4 * v + 1] * c_new,
                              o4.z * c_old + f[4 * v + 2] * c_new, o4.w * c_old + f[4 * v + 3] * c_new);
        }
      }
    }
    if (write) P.part_lse[row_off] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
    return;
  }
  if (P.n_split > 1) {
    // One key-range slice of a split problem: fp32 O normalised by this
    // slice's own sum, and the slice's LSE; the merge kernel combines them.
    const size_t part_row = (size_t)u.split * ((size_t)p.B * p.Hq * p.Lq) + row_off;
    float4* outp = reinterpret_cast<float4*>(P.part_o + part_row * D);
#pragma unroll
    for (int q = 0; q < D / 16; q++) {
      float f[16];
      load_o(q, f);
      if (write) {
#pragma unroll
        for (int v = 0; v < 4; v++) outp[q * 4 + v] = make_float4(f[4 * v], f[4 * v + 1], f[4 * v + 2], f[4 * v + 3]);
      }
    }
    if (write) P.part_lse[part_row] = lse_row;
    return;
  }
  uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.o) + row_off * D);
#pragma unroll
  for (int q = 0; q < D / 16; q++) {
    float f[16];
    load_o(q, f);
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 8; e++) w[e] = pack_bf16x2(f[2 * e], f[2 * e + 1]);
    if (write) {
#pragma unroll
      for (int v = 0; v < 2; v++) out[q * 2 + v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
  }
  if (write) P.lse[row_off] = lse_row;
}

// ------------------------------------------------------------------ kernel
// W: the problem has global tokens (the key-tile walk may have several ranges).
// A: alternating slots (launched only for plans that use them, so the other
// variants carry none of that code).  DN: the walk runs downwards (block-sparse
// masks; a compile-time choice, since a run-time direction cost about 5% on
// the causal workloads).
template <int D, bool W, bool A, bool DN>
__global__ void __launch_bounds__(THREADS, 1) attn_fwd_kernel(const __grid_constant__ FwdParams P) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bars& bars = *reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  Unit u = decode_unit_split<W, DN>(P, blockIdx.x);
  if (!A || W) u.alt = 0;

  const WaitGuard g{P.err, &bars.abort_flag, P.limit_ns, 0};

  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    for (int s = 0; s < 2; s++) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.o_full[s], 1);
    }
    mbar_init(&bars.merge, 4);
    mbar_init(&bars.drain, 1);
    for (int st = 0; st < C::NST; st++) {
      mbar_init(&bars.kv_full[st], 1);
      mbar_init(&bars.kv_empty[st], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  // Registers: launched at 168 per thread (384 x 168); the load/MMA group
  // drops to 112, each softmax group takes 192 (128*112 + 256*192 <= 384*168).
  if (warp < 4) {
    regs_dec<112>();
    if (warp == 0) {
      if (lane == 0) producer<D, W>(P, u, smem, bars, g);
    } else if (warp == 1) {
      if (lane == 0) {
        if (!W && u.alt)
          mma_issuer_alt<D>(P, u, smem, bars, tmem, g);
        else
          mma_issuer<D, W>(P, u, smem, bars, tmem, g);
      }
    }
  } else {
    regs_inc<192>();
    softmax_slot<D, W>(P, u, (warp - 4) / 4, smem, bars, tmem, g);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ split merge
// Row i of a split problem: with w_k = exp(LSE_k - max_k LSE_k) over the
// slices k, O_i = sum_k w_k O_k / sum_k w_k and LSE_i = max + log(sum_k w_k)
// (each O_k is already normalised by its own slice's sum, so this is the
// exact softmax over the union of the slices).  A row no slice saw keeps
// O = 0 and LSE = -inf.  One warp per row, D / 32 elements per lane.
template <int D>
__global__ void __launch_bounds__(256) fwd_merge_kernel(const float* __restrict__ part_o,
                                                        const float* __restrict__ part_lse, uint16_t* __restrict__ o,
                                                        float* __restrict__ lse, int64_t rows, int n_split) {
  constexpr int PER = D / 32;
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float mx = -INFINITY;
  for (int k = 0; k < n_split; k++) mx = fmaxf(mx, part_lse[(int64_t)k * rows + row]);
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; e++) acc[e] = 0.f;
  float sum = 0.f;
  if (mx != -INFINITY) {
    for (int k = 0; k < n_split; k++) {
      const float lk = part_lse[(int64_t)k * rows + row];
      if (lk == -INFINITY) continue;
      const float w = expf(lk - mx);
      sum += w;
      const float* src = part_o + ((int64_t)k * rows + row) * D + lane * PER;
      if constexpr (PER == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        acc[0] += w * x.x, acc[1] += w * x.y, acc[2] += w * x.z, acc[3] += w * x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] += w * x.x, acc[1] += w * x.y;
      }
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  uint16_t* dst = o + row * D + lane * PER;
  if constexpr (PER == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) lse[row] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace fwd

cudaError_t launch_fwd_merge(const FwdParams& P, cudaStream_t stream) {
  const int64_t rows = (int64_t)P.prob.B * P.prob.Hq * P.prob.Lq;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (P.prob.d == 128)
    fwd::fwd_merge_kernel<128><<<grid, 256, 0, stream>>>(P.part_o, P.part_lse, static_cast<uint16_t*>(P.o), P.lse,
                                                          rows, P.n_split);
  else
    fwd::fwd_merge_kernel<64><<<grid, 256, 0, stream>>>(P.part_o, P.part_lse, static_cast<uint16_t*>(P.o), P.lse,
                                                         rows, P.n_split);
  return cudaGetLastError();
}


void fwd_plan(const Problem& p, int* n_units, int* pair_heads, int* packed, int* alternate) {
  const int G = p.Hq / p.Hkv;
  const int nqt = cdiv(p.Lq, fwd::BM);
  *packed = 0;
  *alternate = 0;
  if (G > 1 && p.Lq < fwd::BM) {
    // Fewer query rows than a tile: stack the G heads of a kv group in the
    // tile rows, so the group's K/V stream once per 256 rows (two slots).
    *packed = 1;
    *pair_heads = 0;
    *n_units = p.B * p.Hkv * cdiv(cdiv(G * p.Lq, fwd::BM), 2);
    *alternate = cdiv(G * p.Lq, fwd::BM) == 1;
  } else if (G % 2 == 0) {
    *pair_heads = 1;
    *n_units = p.B * (p.Hq / 2) * nqt;
  } else {
    *pair_heads = 0;
    *n_units = p.B * p.Hq * cdiv(nqt, 2);
    *alternate = nqt == 1;
  }
  // One slot of rows per unit: the second slot takes alternate key tiles of
  // the same rows (one contiguous key range, so not with global tokens).
  if (has_global(p)) *alternate = 0;
}

template <int D, bool W, bool A, bool DN = false>
static cudaError_t launch_fwd_d(const FwdParams& P, cudaStream_t stream) {
  constexpr int smem = fwd::Cfg<D>::SMEM;
  static std::atomic<unsigned char> ready[kMaxDevices];
  cudaError_t e = once_per_device(ready, [] {
    return cudaFuncSetAttribute(fwd::attn_fwd_kernel<D, W, A, DN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  fwd::attn_fwd_kernel<D, W, A, DN><<<P.n_units * imax(1, P.n_split), fwd::THREADS, smem, stream>>>(P);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_fwd_dd(const FwdParams& P, cudaStream_t stream) {
  if (has_global(P.prob)) return launch_fwd_d<D, true, false>(P, stream);
  const bool down = P.prob.sparse_block > 0;  // as decode_unit sets Unit::down
  if (P.alternate) return down ? launch_fwd_d<D, false, true, true>(P, stream) : launch_fwd_d<D, false, true>(P, stream);
  return down ? launch_fwd_d<D, false, false, true>(P, stream) : launch_fwd_d<D, false, false>(P, stream);
}

cudaError_t launch_fwd(const FwdParams& P, cudaStream_t stream) {
  if (P.n_units <= 0) return cudaSuccess;
  return P.prob.d == 128 ? launch_fwd_dd<128>(P, stream) : launch_fwd_dd<64>(P, stream);
}

}  // namespace tea

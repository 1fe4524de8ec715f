// attn_bwd.cu - backward attention kernels for sm_100a.
//
// Recompute backward ("缩放定律与高效注意力" §3.3: only O and the per-row
// logsumexp are kept from the forward pass; Q, K, V are read again and the
// scores rebuilt tile by tile).  The gradient itself is the textbook softmax
// gradient, which the pages do not print:
//   D_i = dO_i . O_i,  P = exp(scale*S - LSE),  dV = P^T dO,  dP = dO V^T,
//   dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three launches:
//   bwd_pre   D_i for every query row, and zero the fp32 dQ accumulator
//   bwd_main  one CTA per (batch, K/V head, tile of 128 keys); it loops over
//             the query heads of the GQA group and the query tiles that see
//             its keys, accumulating dK and dV in tensor memory for the whole
//             loop and adding each step's dQ contribution into the fp32
//             accumulator [B*Hq, Lq, d] (d = 128: TMA tensor reduce-add from a
//             staging tile; d = 64: vector red.global from registers)
//   bwd_post  dQ = scale * accumulator, rounded to bf16 (element-wise)
//
// bwd_main works in the transposed orientation, keys on the 128 TMEM lanes:
//   S^T = K Q^T and dP^T = V dO^T     (M = 128 keys, N = BM query rows)
//   dV += P^T dO and dK += dS^T Q     (M = 128 keys, N = d)
//   dQ^T = K^T dS^T  (d = 128)  or  dQ = dS K  (d = 64)   (M = 128, N = 64)
// so that one thread per key turns a row of S^T into P^T and dS^T, and the
// bf16 P^T and dS^T, written once to shared memory, serve both as the K-major
// A operand of dV/dK and as the MN-major operand of dQ.
// Warp roles (512 threads): warp 0 TMA, warps 1 and 2 MMA issuers, warps 4-7
// and 8-11 the per-key softmax gradient (each group takes half of a step's
// query columns), warps 12-15 the dQ drain.  Tensor memory at d = 128:
// S^T | dP^T | dV | dK | dQ^T | P^T | dS^T = 512 columns.  Q/dO tiles stream
// through a 3-stage ring.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cmath>

#include "sm100.cuh"
#include "attn_common.cuh"
#include "attn_kernels.h"

namespace tea {
namespace bwd {

constexpr int BN = 128;  // keys per CTA
constexpr int THREADS = 512;
constexpr int KPANEL = 16384;  // 128 rows x 128 bytes
constexpr float LOG2E = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int BM = D == 128 ? 64 : 128;  // query rows per step
  static constexpr int NBUF = D == 128 ? 2 : 1;   // dS^T (and P^T) shared-memory buffers
  // d = 128: P^T and dS^T also go to tensor memory and feed dV/dK as the A
  // operand from TMEM (no P^T tile in shared memory).  d = 64 has no TMEM
  // room for them and reads both from shared memory.
  static constexpr bool TS = D == 128;
  static constexpr int NQS = 3;                   // Q/dO ring stages
  // d = 128: the dQ^T tile of a step leaves through two 16 KB halves of a
  // staging area ([32 query rows][128 d] fp32 each) and a TMA tensor reduce-add.
  static constexpr int STG_BYTES = D == 128 ? 2 * 16384 : 0;
  static constexpr int KV_TILE = BN * D * 2;
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int Q_PANEL = BM * 128;
  static constexpr int PS_TILE = BN * BM * 2;
  static constexpr int CW = BM / 2;               // query columns per gradient warpgroup
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int OFF_Q = OFF_V + KV_TILE;
  static constexpr int OFF_DO = OFF_Q + NQS * Q_TILE;
  static constexpr int OFF_PT = OFF_DO + NQS * Q_TILE;
  static constexpr int OFF_DST = OFF_PT + (TS ? 0 : NBUF * PS_TILE);
  static constexpr int OFF_STG = OFF_DST + NBUF * PS_TILE;
  static constexpr int OFF_VEC = OFF_STG + STG_BYTES;  // [group][2 bufs][lse2 | D][CW] fp32
  static constexpr int OFF_BAR = OFF_VEC + 2 * 2 * 2 * CW * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t T_S = 0, T_DP = BM, T_DV = 2 * BM, T_DK = 2 * BM + D, T_DQ = 2 * BM + 2 * D;
  static constexpr uint32_t T_PT = T_DQ + 64, T_DST = T_PT + BM / 2;  // bf16 pairs (TS only)
  static_assert(T_DQ + 64 <= 512 && (!TS || T_DST + BM / 2 <= 512), "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(OFF_STG % 1024 == 0, "staging must be 1024-byte aligned");
};

// Barriers.  The MMA issuer pays for every wait and commit with tensor-core
// idle time (its issue queue is shallow), so each of its waits covers
// everything the next MMA group needs:
//   q_land[stage]    Q/dO of a step landed (TMA bytes; 1 arrival by the
//                    producer); it counts only the producer's copies, so the
//                    producer can wait for exactly those before the CTA exits
//   sq_ready[stage]  the previous step's S^T/dP^T were read out (8 gradient
//                    warps); the S^T/dP^T issuer waits on q_land first (by
//                    then the copy has almost always landed, so that wait is
//                    off the critical path) and then on this
//   grad_ready[2]    P^T/dS^T of a step written (8 gradient warps) and the
//                    previous step's dQ read out of TMEM (4 drain warps)
//   sdp_full         S^T/dP^T of a step complete
//   step_done        all MMAs of a step complete (dQ readable; P^T/dS^T and
//                    the dS^T tile may be overwritten)
//   q_empty[stage]   the step's Q/dO stage may be reloaded
struct Bars {
  uint64_t kv_full;
  uint64_t sq_ready[4], q_empty[4], q_land[4];  // Q/dO ring (up to 4 stages)
  uint64_t grad_ready[2];
  uint64_t sdp_full, step_done;
  uint64_t vec_full[2][2];  // [group][buffer]
  uint64_t stg_full[2], stg_free[2];  // dQ staging halves (d = 128)
  uint64_t dkv_full;
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
struct BarsFit {
  static_assert(sizeof(Bars) <= 256, "barrier block overflows its shared-memory slot");
};

struct Unit {
  int b, kvh, k0;
  int G, nq, qt_lo, n_steps;
};

template <int D>
__device__ __forceinline__ Unit decode_unit(const BwdParams& P, int idx) {
  const Problem& p = P.prob;
  Unit u;
  // Heads in groups of up to 8: the CTAs running at one time share the
  // Q/dO/K/V of a few heads in L2.  Inside a group, key tiles ascend (early
  // keys see the most queries under a causal mask: heavy first).
  const int nkt = cdiv(p.Lk, BN);
  const int heads = p.B * p.Hkv;
  constexpr int HG = 8;
  const int grp = idx / (HG * nkt);
  const int hg = imin(HG, heads - grp * HG);
  const int rem = idx - grp * HG * nkt;
  const int n = rem / hg;
  const int head = grp * HG + rem % hg;
  u.b = head / p.Hkv;
  u.kvh = head % p.Hkv;
  u.k0 = n * BN;
  u.G = p.Hq / p.Hkv;
  int q_lo, q_hi;
  q_row_range(seq_problem(p, u.b), u.k0, u.k0 + BN, q_lo, q_hi);
  constexpr int BM = Cfg<D>::BM;
  u.qt_lo = q_lo / BM;
  u.nq = q_hi > q_lo ? cdiv(q_hi, BM) - u.qt_lo : 0;
  u.n_steps = u.G * u.nq;
  return u;
}

// Step i of a unit: query head h (global head index) and first query row q0.
// Each head's query tiles are taken from the last down (under a causal mask
// the diagonal tile comes last); measured about 1% faster than upwards.
template <int D>
__device__ __forceinline__ void step_of(const Unit& u, int i, int& h, int& q0) {
  const int g = i / u.nq;
  h = u.kvh * u.G + g;
  q0 = (u.qt_lo + u.nq - 1 - i % u.nq) * Cfg<D>::BM;
}

// ------------------------------------------------------------------ producer
template <int D>
__device__ void producer(const BwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, const WaitGuard& g) {
  using C = Cfg<D>;
  const Problem& p = P.prob;
  tma_prefetch_desc(&P.tm_q);
  tma_prefetch_desc(&P.tm_do);
  tma_prefetch_desc(&P.tm_k);
  tma_prefetch_desc(&P.tm_v);
  mbar_arrive_expect_tx(&bars.kv_full, 2 * C::KV_TILE);
  for (int pnl = 0; pnl < D / 64; pnl++) {
    tma_load_3d(smem + C::OFF_K + pnl * KPANEL, &P.tm_k, &bars.kv_full, pnl * 64, u.k0, u.b * p.Hkv + u.kvh);
    tma_load_3d(smem + C::OFF_V + pnl * KPANEL, &P.tm_v, &bars.kv_full, pnl * 64, u.k0, u.b * p.Hkv + u.kvh);
  }
  int issued = 0;
  for (int i = 0; i < u.n_steps; i++) {
    const int st = i % C::NQS;
    if (!mbar_wait(&bars.q_empty[st], ((i / C::NQS) & 1) ^ 1, g, 1)) break;
    int h, q0;
    step_of<D>(u, i, h, q0);
    mbar_arrive_expect_tx(&bars.q_land[st], 2 * C::Q_TILE);
    for (int pnl = 0; pnl < D / 64; pnl++) {
      tma_load_3d(smem + C::OFF_Q + st * C::Q_TILE + pnl * C::Q_PANEL, &P.tm_q, &bars.q_land[st], pnl * 64, q0,
                  u.b * p.Hq + h);
      tma_load_3d(smem + C::OFF_DO + st * C::Q_TILE + pnl * C::Q_PANEL, &P.tm_do, &bars.q_land[st], pnl * 64, q0,
                  u.b * p.Hq + h);
    }
    issued = i + 1;
  }
  // Let every copy this warp started land before the CTA may exit (also after
  // an abort).  K/V have their own barrier.  A Q/dO load of step j is only
  // issued once step j - NQS has finished with its stage, so only the last
  // NQS loads can still be in flight, each the latest phase of its stage's
  // q_land barrier.
  mbar_wait_ignore_abort(&bars.kv_full, 0, g);
  for (int j = imax(0, issued - C::NQS); j < issued; j++)
    mbar_wait_ignore_abort(&bars.q_land[j % C::NQS], (j / C::NQS) & 1, g);
}


// ------------------------------------------------------------------ MMA issuer
// Two issuing threads keep the tensor core fed: each mbarrier wait costs the
// issuing thread about as long as an MMA, and the tensor core's issue queue is
// shallow, so while one issuer waits the other one issues.
template <int D, int ROLE>
__device__ void mma_issuer(const BwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, uint32_t tmem,
                           const WaitGuard& g) {
  using C = Cfg<D>;
  constexpr int BM = C::BM;
  const uint32_t idesc_s = idesc_bf16_f32(128, BM, 0, 0);
  const uint32_t idesc_dkv = idesc_bf16_f32(128, D, 0, 1);
  const uint32_t idesc_dq = idesc_bf16_f32(128, 64, 1, 1);
  // Shared-memory descriptors are built once; an operand slice at byte offset
  // `off` from a tile's start is that tile's descriptor plus off / 16 (the
  // start-address field; no carry since shared addresses are < 256 KB).
  const uint32_t k_addr = smem_u32(smem + C::OFF_K);
  const uint64_t k_kmaj = sw128_desc(k_addr, 16, 1024);                    // K as K-major A (S^T)
  const uint64_t v_kmaj = sw128_desc(smem_u32(smem + C::OFF_V), 16, 1024); // V as K-major A (dP^T)
  const uint64_t k_mn = sw128_desc(k_addr, KPANEL, 1024);                  // K as MN-major operand (dQ)
  const uint64_t q_kmaj = sw128_desc(smem_u32(smem + C::OFF_Q), 16, 1024);
  const uint64_t do_kmaj = sw128_desc(smem_u32(smem + C::OFF_DO), 16, 1024);
  const uint64_t q_mn = sw128_desc(smem_u32(smem + C::OFF_Q), C::Q_PANEL, 1024);
  const uint64_t do_mn = sw128_desc(smem_u32(smem + C::OFF_DO), C::Q_PANEL, 1024);
  const uint64_t pt_kmaj = sw128_desc(smem_u32(smem + C::OFF_PT), 16, 1024);
  const uint64_t ds_kmaj = sw128_desc(smem_u32(smem + C::OFF_DST), 16, 1024);
  const uint64_t ds_mn = sw128_desc(smem_u32(smem + C::OFF_DST), KPANEL, 1024);
  auto adv = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };

  // S^T = K Q^T and dP^T = V dO^T for step i (contraction over d).
  auto issue_sdp = [&](int i) {
    const uint32_t st_off = (uint32_t)(i % C::NQS) * C::Q_TILE;
    const uint64_t qd = adv(q_kmaj, st_off), dd = adv(do_kmaj, st_off);
#pragma unroll
    for (int kk = 0; kk < D / 16; kk++) {
      const uint32_t oa = (kk / 4) * KPANEL + (kk % 4) * 32;
      const uint32_t ob = (kk / 4) * C::Q_PANEL + (kk % 4) * 32;
      mma_ss(tmem + C::T_S, adv(k_kmaj, oa), adv(qd, ob), idesc_s, kk > 0);
    }
#pragma unroll
    for (int kk = 0; kk < D / 16; kk++) {
      const uint32_t oa = (kk / 4) * KPANEL + (kk % 4) * 32;
      const uint32_t ob = (kk / 4) * C::Q_PANEL + (kk % 4) * 32;
      mma_ss(tmem + C::T_DP, adv(v_kmaj, oa), adv(dd, ob), idesc_s, kk > 0);
    }
    mma_commit(&bars.sdp_full);
  };

  if (ROLE == 0) {
    // Issuer A: S^T and dP^T of every step.
    if (u.n_steps == 0) goto done;
    if (!mbar_wait(&bars.kv_full, 0, g, 10)) goto done;
    for (int i = 0; i < u.n_steps; i++) {
      // Q/dO of step i landed and S^T/dP^T of step i-1 read out.
      if (!mbar_wait(&bars.q_land[i % C::NQS], (i / C::NQS) & 1, g, 11)) goto done;
      if (!mbar_wait(&bars.sq_ready[i % C::NQS], (i / C::NQS) & 1, g, 12)) goto done;
      tc_fence_after();
      issue_sdp(i);
    }
  } else {
    // Issuer B: dV, dK and dQ of every step.
    if (u.n_steps == 0) goto done;
    if (!mbar_wait(&bars.kv_full, 0, g, 10)) goto done;
    for (int i = 0; i < u.n_steps; i++) {
      // P^T/dS^T of step i written and dQ of step i-1 read out of TMEM.
      if (!mbar_wait(&bars.grad_ready[i & 1], (i >> 1) & 1, g, 14)) goto done;
      tc_fence_after();
      const int buf = i % C::NBUF;
      const uint32_t st_off = (uint32_t)(i % C::NQS) * C::Q_TILE;
      const uint32_t ps_off = (uint32_t)buf * C::PS_TILE;
      const uint64_t qmn = adv(q_mn, st_off), domn = adv(do_mn, st_off);
      const uint32_t acc0 = i > 0;
      // dV += P^T dO and dK += dS^T Q (contraction over the BM query rows).
      if constexpr (C::TS) {
        // A operand from tensor memory: 16 query rows = 8 columns of bf16 pairs.
#pragma unroll
        for (int kk = 0; kk < BM / 16; kk++)
          mma_ts(tmem + C::T_DV, tmem + C::T_PT + kk * 8, adv(domn, kk * 2048), idesc_dkv, kk > 0 ? 1u : acc0);
#pragma unroll
        for (int kk = 0; kk < BM / 16; kk++)
          mma_ts(tmem + C::T_DK, tmem + C::T_DST + kk * 8, adv(qmn, kk * 2048), idesc_dkv, kk > 0 ? 1u : acc0);
      } else {
        const uint64_t pd = adv(pt_kmaj, ps_off), sd = adv(ds_kmaj, ps_off);
#pragma unroll
        for (int kk = 0; kk < BM / 16; kk++) {
          const uint32_t oa = (kk / 4) * KPANEL + (kk % 4) * 32;
          mma_ss(tmem + C::T_DV, adv(pd, oa), adv(domn, kk * 2048), idesc_dkv, kk > 0 ? 1u : acc0);
        }
#pragma unroll
        for (int kk = 0; kk < BM / 16; kk++) {
          const uint32_t oa = (kk / 4) * KPANEL + (kk % 4) * 32;
          mma_ss(tmem + C::T_DK, adv(sd, oa), adv(qmn, kk * 2048), idesc_dkv, kk > 0 ? 1u : acc0);
        }
      }
      // dQ contribution of this key tile (contraction over the 128 keys).
      const uint64_t dsmn = adv(ds_mn, ps_off);
#pragma unroll
      for (int kk = 0; kk < BN / 16; kk++) {
        if (D == 128)  // dQ^T = K^T dS^T: A = K (M = d), B = dS^T (N = query rows)
          mma_ss(tmem + C::T_DQ, adv(k_mn, kk * 2048), adv(dsmn, kk * 2048), idesc_dq, kk > 0);
        else  // dQ = dS K: A = dS^T viewed MN-major (M = query rows), B = K (N = d)
          mma_ss(tmem + C::T_DQ, adv(dsmn, kk * 2048), adv(k_mn, kk * 2048), idesc_dq, kk > 0);
      }
      // Everything of step i issued by B (and, causally, S^T/dP^T of step i
      // by A, which the gradient warps had to read first) is done when these
      // fire.
      mma_commit(&bars.step_done);
      mma_commit(&bars.q_empty[i % C::NQS]);
    }
  }
done:
  if (ROLE == 1) mma_commit(&bars.dkv_full);
  // Drain: every MMA this thread issued has completed (each issuer has its own barrier).
  mma_commit(&bars.drain[ROLE]);
  mbar_wait_ignore_abort(&bars.drain[ROLE], 0, g);
}

// ------------------------------------------------------------------ softmax gradient
// Two warpgroups share a step: group w takes query columns [w*CW, w*CW + CW).
// Thread `row` of a group owns key k0 + row (TMEM lane row) and turns its part
// of the S^T and dP^T rows into P^T = exp2(c*S - LSE*log2e) and
// dS^T = P^T * (dP^T - D), written as bf16 into the 128-byte-swizzled tiles.
// ACC: the accumulate variant (ring attention) adds dK / dV into fp32
// accumulators; it is a separate instantiation so that the ordinary kernel
// carries none of its code (with it the backward measured 2.4% slower).
template <int D, bool ACC>
__device__ void grad_rows(const BwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, uint32_t tmem, int grp,
                          const WaitGuard& g) {
  using C = Cfg<D>;
  constexpr int BM = C::BM;
  constexpr int CW = C::CW;
  const Problem& p = P.prob;
  const int row = threadIdx.x % 128;  // key row = TMEM lane
  const int wl = (threadIdx.x / 32) % 4;
  const int lane = threadIdx.x % 32;
  const int key = u.k0 + row;
  const int col0 = grp * CW;  // first query column of this group
  const uint32_t lane_base = (uint32_t)(wl * 32) << 16;
  // Queries [vis_lo, vis_hi) see this key.
  int vis_lo = 0, vis_hi = 0;
  const Problem ps = seq_problem(p, u.b);  // this sequence's lengths (padded batches)
  if (key < ps.Lk) {
    const int off = diag_off(ps);
    vis_lo = ps.causal ? imax(0, key - off) : (ps.window > 0 ? imax(0, key - ps.window + 1) : 0);
    vis_hi = ps.window > 0 ? imin(ps.Lq, key - off + ps.window) : ps.Lq;
    if (ps.sparse_block > 0) {
      int slo, shi;
      sparse_key_rows(ps, key, key + 1, slo, shi);
      vis_lo = imax(vis_lo, slo);
      vis_hi = imin(vis_hi, shi);
    }
    // A global key is seen by every query (at or past it under a causal mask).
    if (key < ps.global_head || key >= tail_start(ps)) {
      vis_lo = ps.causal ? imax(0, key - off) : 0;
      vis_hi = ps.Lq;
    }
  }
  const float c = P.scale_log2;
  float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC) + grp * (2 * 2 * CW);
  uint8_t* pt_base = smem + C::OFF_PT;
  uint8_t* dst_base = smem + C::OFF_DST;
  const uint32_t sw = (uint32_t)(row & 7);

  // LSE and D of the group's queries in step i: thread row < CW fetches query
  // q0 + col0 + row one step ahead (raw values; the load stays in flight
  // during the previous step) and publishes them to shared memory at the
  // step's start.  Rows past Lq: LSE = +inf (so p = 0) and D = 0.
  auto fetch = [&](int i, float& l, float& dv) {
    int h, q0;
    step_of<D>(u, i, h, q0);
    const int q = q0 + col0 + row;
    l = INFINITY;
    dv = 0.f;
    if (row < CW && q < ps.Lq) {
      const size_t r = (size_t)(u.b * p.Hq + h) * p.Lq + q;
      l = P.lse[r];
      dv = P.dvec[r];
    }
  };
  float next_l = INFINITY, next_d = 0.f;
  if (u.n_steps > 0) fetch(0, next_l, next_d);
  // Step 0 has no earlier S^T/dP^T to read out.
  __syncwarp();
  if (lane == 0) mbar_arrive(&bars.sq_ready[0]);

  for (int i = 0; i < u.n_steps; i++) {
    int h, q0;
    step_of<D>(u, i, h, q0);
    const int vb = i & 1;
    if (row < CW) {
      vec[(vb * 2 + 0) * CW + row] = next_l * LOG2E;
      vec[(vb * 2 + 1) * CW + row] = next_d;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.vec_full[grp][vb]);
    if (i + 1 < u.n_steps) fetch(i + 1, next_l, next_d);
    if (!mbar_wait(&bars.vec_full[grp][vb], (i >> 1) & 1, g, 20)) return;
    const float* lse2 = vec + (vb * 2 + 0) * CW;
    const float* dd = vec + (vb * 2 + 1) * CW;
    const int qc0 = q0 + col0;  // first query of this group's columns
    const bool full = vis_lo <= qc0 && qc0 + CW <= vis_hi;

    if (!mbar_wait(&bars.sdp_full, i & 1, g, 21)) return;
    tc_fence_after();
    const int buf = i % C::NBUF;
    uint8_t* pt_row = pt_base + buf * C::PS_TILE + row * 128;
    uint8_t* ds_row = dst_base + buf * C::PS_TILE + row * 128;

    // The group's CW columns are read from TMEM 32 at a time (S^T and dP^T);
    // P^T and dS^T are kept as packed bf16 pairs until the previous step's
    // MMAs have released their destinations.
    constexpr int NCH = CW / 32;
    uint32_t pw_all[CW / 2], dw_all[CW / 2];
    auto calc_chunk = [&](int ch, const uint32_t* sv, const uint32_t* dpv) {
#pragma unroll
      for (int e = 0; e < 16; e++) {
        float pr[2], dr[2];
#pragma unroll
        for (int z = 0; z < 2; z++) {
          const int col = e * 2 + z;     // column within the chunk
          const int qq = ch * 32 + col;  // column within the group
          float pv = ex2_approx(fmaf(__uint_as_float(sv[col]), c, -lse2[qq]));
          if (!full) {
            const int q = qc0 + qq;
            if (q < vis_lo || q >= vis_hi) pv = 0.f;
          }
          pr[z] = pv;
          dr[z] = pv * (__uint_as_float(dpv[col]) - dd[qq]);
        }
        pw_all[ch * 16 + e] = pack_bf16x2(pr[0], pr[1]);
        dw_all[ch * 16 + e] = pack_bf16x2(dr[0], dr[1]);
      }
    };
#pragma unroll
    for (int ch = 0; ch < NCH; ch++) {
      uint32_t sv[32], dpv[32];
      tmem_ld32p(tmem + lane_base + C::T_S + col0 + 32 * ch, sv);
      tmem_ld32p(tmem + lane_base + C::T_DP + col0 + 32 * ch, dpv);
      tmem_wait_ld();
      if (ch == NCH - 1) {
        // S^T / dP^T of this step are read: the next step's MMAs may overwrite them.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.sq_ready[(i + 1) % C::NQS]);
      }
      calc_chunk(ch, sv, dpv);
    }
    // The previous step's MMAs must be done with the TMEM P^T/dS^T and with
    // this dS^T (and P^T) shared-memory buffer.
    if (i > 0) {
      if (!mbar_wait(&bars.step_done, (i - 1) & 1, g, 22)) return;
      tc_fence_after();
    }
#pragma unroll
    for (int j4 = 0; j4 < CW / 8; j4++) {
      // 16-byte piece j of the row lives in panel j / 8, at chunk (j % 8) ^ (row % 8).
      const int j = col0 / 8 + j4;
      const uint32_t off = (uint32_t)(j / 8) * KPANEL + (((uint32_t)(j % 8) ^ sw) << 4);
      if constexpr (!C::TS)
        *reinterpret_cast<uint4*>(pt_row + off) =
            make_uint4(pw_all[4 * j4], pw_all[4 * j4 + 1], pw_all[4 * j4 + 2], pw_all[4 * j4 + 3]);
      *reinterpret_cast<uint4*>(ds_row + off) =
          make_uint4(dw_all[4 * j4], dw_all[4 * j4 + 1], dw_all[4 * j4 + 2], dw_all[4 * j4 + 3]);
    }
    if constexpr (C::TS) {
      tmem_st16(tmem + lane_base + C::T_PT + grp * 16, *reinterpret_cast<const uint32_t(*)[16]>(pw_all));
      tmem_st16(tmem + lane_base + C::T_DST + grp * 16, *reinterpret_cast<const uint32_t(*)[16]>(dw_all));
      tmem_wait_st();
    }
    fence_proxy_async_smem();  // generic-proxy stores -> tensor-core reads
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && i + 1 != P.stall_at) mbar_arrive(&bars.grad_ready[i & 1]);
  }

  // Epilogue: group 0 writes dV, group 1 writes scale * dK for its key.
  const bool has = u.n_steps > 0;
  if (has) {
    if (!mbar_wait(&bars.dkv_full, 0, g, 23)) return;
    tc_fence_after();
  }
  const bool write = key < p.Lk;
  const size_t off = ((size_t)(u.b * p.Hkv + u.kvh) * p.Lk + key) * D;
  uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(grp ? P.dk : P.dv) + off);
  const float f = grp ? P.scale : 1.f;
  const uint32_t colx = grp ? C::T_DK : C::T_DV;
  if constexpr (ACC) {
    // Accumulate mode (ring attention): this key block's dK / dV added into
    // fp32 accumulators; a key row belongs to one CTA, so no race.
    float4* acc = reinterpret_cast<float4*>((grp ? P.dk_acc : P.dv_acc) + off);
#pragma unroll
    for (int q = 0; q < D / 32; q++) {
      uint32_t o[32];
      if (has) {
        tmem_ld32p(tmem + lane_base + colx + 32 * q, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; e++) o[e] = 0u;
      }
      if (write) {
#pragma unroll
        for (int v = 0; v < 8; v++) {
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
          if (!P.dkv_init) a = acc[q * 8 + v];
          acc[q * 8 + v] = make_float4(a.x + __uint_as_float(o[4 * v]) * f, a.y + __uint_as_float(o[4 * v + 1]) * f,
                                       a.z + __uint_as_float(o[4 * v + 2]) * f, a.w + __uint_as_float(o[4 * v + 3]) * f);
        }
      }
    }
  } else {
#pragma unroll
  for (int q = 0; q < D / 32; q++) {
    uint32_t o[32];
    if (has) {
      tmem_ld32p(tmem + lane_base + colx + 32 * q, o);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; e++) o[e] = 0u;
    }
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; e++) w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * f, __uint_as_float(o[2 * e + 1]) * f);
    if (write) {
#pragma unroll
      for (int v = 0; v < 4; v++) out[q * 4 + v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
  }
  }
}

// ------------------------------------------------------------------ dQ drain
// Moves each step's fp32 dQ tile out of tensor memory into the accumulator
// [B*Hq, Lq, d] (the layout of dQ itself, so the final pass is element-wise):
//   d = 128 (dQ^T in TMEM, lane = d, 64 query columns): lane t writes element
//     (q, t) of a row-major staging half [32 queries][128 d] (for each q the
//     warp's 32 lanes fill 128 contiguous bytes: no bank conflict), and one
//     thread adds the half into the accumulator with a TMA tensor reduce-add
//     (element-wise atomic in L2; rows past Lq are clipped by the tensor's
//     bounds); two halves alternate so staging overlaps the reduce.
//   d = 64 (dQ in TMEM, lane = query, 64 d columns): the lane's row is 256
//     contiguous bytes of the accumulator, added with 16 vector red.global.
__device__ __forceinline__ void red_add_v4_f32(float* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}

__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// Wait until at most one committed bulk group still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

template <int D>
__device__ void dq_drain(const BwdParams& P, const Unit& u, uint8_t* smem, Bars& bars, uint32_t tmem,
                         const WaitGuard& g) {
  using C = Cfg<D>;
  const Problem& p = P.prob;
  const int t = threadIdx.x % 128;  // TMEM lane
  const int wl = (threadIdx.x / 32) % 4;
  const int lane = threadIdx.x % 32;
  const uint32_t lane_base = (uint32_t)(wl * 32) << 16;
  uint8_t* stg = smem + C::OFF_STG;
  int half = 0;  // staging halves used so far

  // Step 0 has no earlier dQ to read out.
  if (lane == 0) mbar_arrive(&bars.grad_ready[0]);
  for (int i = 0; i < u.n_steps; i++) {
    int h, q0;
    step_of<D>(u, i, h, q0);
    if (!mbar_wait(&bars.step_done, i & 1, g, 30)) break;
    tc_fence_after();
    uint32_t r[64];
    tmem_ld32p(tmem + lane_base + C::T_DQ, r);
    tmem_ld32p(tmem + lane_base + C::T_DQ + 32, r + 32);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.grad_ready[(i + 1) & 1]);  // dQ TMEM free for step i+1
    const int bh = u.b * p.Hq + h;
    if constexpr (D == 128) {
#pragma unroll
      for (int hh = 0; hh < 2; hh++, half++) {
        const int b = half & 1, use = half >> 1;
        // The reduce of this buffer's previous use must have read it.
        if (use > 0 && !mbar_wait(&bars.stg_free[b], (use - 1) & 1, g, 31)) goto out;
        float* col = reinterpret_cast<float*>(stg + b * 16384) + t;
#pragma unroll
        for (int qq = 0; qq < 32; qq++) col[qq * 128] = __uint_as_float(r[32 * hh + qq]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.stg_full[b]);
        if (t == 0) {
          if (!mbar_wait(&bars.stg_full[b], use & 1, g, 32)) goto out;
          // Query rows past Lq are clipped by the tensor bounds.
          tma_reduce_add_3d(&P.tm_dq, stg + b * 16384, 0, q0 + 32 * hh, bh);
          bulk_commit();
          bulk_wait_read_1();  // the previous half has been read
          if (half > 0) mbar_arrive(&bars.stg_free[(half - 1) & 1]);
        }
      }
    } else {
      // Lane t holds dQ row q0 + t.
      if (q0 + t < p.Lq) {
        float* rowp = P.dq_acc + ((size_t)bh * p.Lq + q0 + t) * D;
#pragma unroll
        for (int c = 0; c < 16; c++) red_add_v4_f32(rowp + 4 * c, r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
      }
    }
  }
out:
  // Every reduce this thread started is complete before the CTA may exit (also
  // after an abort, so that no bulk copy still reads the staging buffer).
  if (D == 128 && t == 0) bulk_wait_all();
}

// ------------------------------------------------------------------ kernel
// Per-thread register budgets after setmaxnreg (launch: 512 x 128):
// load/MMA group, gradient groups, dQ drain; 128*RM + 256*RG + 128*RQ <= 65536.
constexpr int RM = 96, RG = 152, RQ = 112;
constexpr int LAUNCH_REGS = 128;  // 65536 / 512
static_assert(128 * RM + 256 * RG + 128 * RQ <= THREADS * LAUNCH_REGS, "register budget");

template <int D, bool ACC>
__global__ void __launch_bounds__(THREADS, 1) attn_bwd_kernel(const __grid_constant__ BwdParams P) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bars& bars = *reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  (void)sizeof(BarsFit<D>);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const Unit u = decode_unit<D>(P, blockIdx.x);
  const WaitGuard g{P.err, &bars.abort_flag, P.limit_ns, 100};

  if (threadIdx.x == 0) {
    bars.abort_flag = 0;
    mbar_init(&bars.kv_full, 1);
    for (int s = 0; s < C::NQS; s++) {
      mbar_init(&bars.sq_ready[s], 8);  // 8 gradient warps
      mbar_init(&bars.q_empty[s], 1);
      mbar_init(&bars.q_land[s], 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(&bars.grad_ready[s], 8 + 4);  // 8 gradient warps + 4 drain warps
      mbar_init(&bars.vec_full[0][s], 4);
      mbar_init(&bars.vec_full[1][s], 4);
    }
    mbar_init(&bars.sdp_full, 1);
    mbar_init(&bars.step_done, 1);
    for (int b = 0; b < 2; b++) {
      mbar_init(&bars.stg_full[b], 4);  // 4 drain warps wrote their rows
      mbar_init(&bars.stg_free[b], 1);  // the reduce finished reading the half
    }
    mbar_init(&bars.dkv_full, 1);
    mbar_init(&bars.drain[0], 1);
    mbar_init(&bars.drain[1], 1);
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

  // Registers: 512 x 128 at launch, redistributed per warpgroup (RM, RG, RQ
  // above); the host refuses the launch at any other compiled count.
  if (warp < 4) {
    regs_set<RM, LAUNCH_REGS>();
    if (warp == 0) {
      if (lane == 0) producer<D>(P, u, smem, bars, g);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<D, 0>(P, u, smem, bars, tmem, g);
    } else if (warp == 2) {
      if (lane == 0) mma_issuer<D, 1>(P, u, smem, bars, tmem, g);
    }
  } else if (warp < 12) {
    regs_set<RG, LAUNCH_REGS>();
    grad_rows<D, ACC>(P, u, smem, bars, tmem, (warp - 4) / 4, g);
  } else {
    regs_set<RQ, LAUNCH_REGS>();
    dq_drain<D>(P, u, smem, bars, tmem, g);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ pre / post
// D_i = sum_c dO_ic * O_ic for every row (fp32), and zero the dQ accumulator.
// Threads in groups of d/8, each reading 8 bf16 of O and dO (16 bytes each).
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      float* __restrict__ dvec, float* __restrict__ dq_acc,
                                                      int64_t rows, int64_t acc_floats) {
  constexpr int TPR = D / 8;  // threads per row
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n = ((rows * TPR + 255) / 256) * 256;  // keep whole warps in the loop
  for (int64_t x = tid; x < n; x += stride) {
    const int64_t r = x / TPR;
    const int part = (int)(x % TPR);
    float acc = 0.f;
    if (r < rows) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + r * D + part * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(dO + r * D + part * 8);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; e++) {
        acc = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), acc);
        acc = fmaf(__uint_as_float(aw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), acc);
      }
    }
#pragma unroll
    for (int sh = TPR / 2; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
    if (r < rows && part == 0) dvec[r] = acc;
  }
  // The accumulator (a multiple of 4 floats) is zeroed with 16-byte stores.
  float4* z = reinterpret_cast<float4*>(dq_acc);
  for (int64_t x = tid; x < acc_floats / 4; x += stride) z[x] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// out = bf16(scale * acc), 8 elements (two float4 in, one uint4 out) per
// thread and iteration; a tail of fewer than 8 elements is converted one by
// one.  With scale = the softmax scale and acc the dQ accumulator this is the
// last backward phase (dQ = scale * dS K); with scale = 1 it rounds an fp32
// accumulator (ring attention's dK / dV).
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float* __restrict__ acc, uint16_t* __restrict__ out,
                                                          int64_t n, float scale) {
  const int64_t n8 = n / 8;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n8; x += stride) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * x];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * x + 1];
    reinterpret_cast<uint4*>(out)[x] =
        make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                   pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n8 * 8) {
    const int64_t i = n8 * 8 + threadIdx.x;
    out[i] = (uint16_t)(pack_bf16x2(acc[i] * scale, 0.f) & 0xFFFFu);
  }
}

}  // namespace bwd

static int elementwise_grid(int64_t work_threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (work_threads + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_bwd_pre(const void* o, const void* dO, float* dvec, float* dq_acc, int64_t rows, int d,
                           int64_t acc_floats, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int64_t work = rows * (d / 8) > acc_floats / 4 ? rows * (d / 8) : acc_floats / 4;
  const int grid = elementwise_grid(work);
  if (d == 128)
    bwd::bwd_pre_kernel<128><<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(o),
                                                        static_cast<const uint16_t*>(dO), dvec, dq_acc, rows,
                                                        acc_floats);
  else
    bwd::bwd_pre_kernel<64><<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(o),
                                                       static_cast<const uint16_t*>(dO), dvec, dq_acc, rows,
                                                       acc_floats);
  return cudaGetLastError();
}

cudaError_t launch_bwd_post(const float* dq_acc, void* dq, int64_t n, float scale, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int grid = elementwise_grid(n / 8 > 0 ? n / 8 : 1);
  bwd::f32_to_bf16_kernel<<<grid, 256, 0, stream>>>(dq_acc, static_cast<uint16_t*>(dq), n, scale);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* acc, void* out, size_t n, cudaStream_t stream) {
  return launch_bwd_post(acc, out, (int64_t)n, 1.f, stream);
}

template <int D, bool ACC>
static cudaError_t launch_bwd_d(const BwdParams& P, cudaStream_t stream) {
  constexpr int smem = bwd::Cfg<D>::SMEM;
  static std::atomic<unsigned char> ready[kMaxDevices];
  const cudaError_t e = once_per_device(ready, [] {
    cudaError_t r =
        cudaFuncSetAttribute(bwd::attn_bwd_kernel<D, ACC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (r != cudaSuccess) return r;
    // setmaxnreg redistributes the registers the block was launched with: the
    // split above is only valid at exactly LAUNCH_REGS per thread.
    return check_launch_regs(reinterpret_cast<const void*>(bwd::attn_bwd_kernel<D, ACC>), bwd::LAUNCH_REGS);
  });
  if (e != cudaSuccess) return e;
  bwd::attn_bwd_kernel<D, ACC><<<P.n_units, bwd::THREADS, smem, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdParams& P, cudaStream_t stream) {
  if (P.n_units <= 0) return cudaSuccess;
  const bool acc = P.dk_acc != nullptr;
  if (P.prob.d == 128) return acc ? launch_bwd_d<128, true>(P, stream) : launch_bwd_d<128, false>(P, stream);
  return acc ? launch_bwd_d<64, true>(P, stream) : launch_bwd_d<64, false>(P, stream);
}

}  // namespace tea

// attn_kernels.h - internal interface between the C ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>
#include "attn_common.cuh"

namespace tea {

struct FwdParams {
  CUtensorMap tm_q;  // [B*Hq, Lq, d] bf16, box 64 x 128 x 1, 128-byte swizzle ([B*Hkv, G*Lq, d] if packed)
  CUtensorMap tm_k;  // [B*Hkv, Lk, d]
  CUtensorMap tm_v;  // [B*Hkv, Lk, d]
  Problem prob;
  void* o;           // bf16 [B, Hq, Lq, d]
  float* lse;        // fp32 [B, Hq, Lq]
  float scale_log2;  // scale * log2(e)
  int pair_heads;    // 1: a CTA takes two heads of one GQA group at the same rows
  int packed;        // 1: short queries; a tile's 128 rows run over the G heads of one kv group
  int alternate;     // 1: each unit has one slot of rows; both slots take them, on alternate key tiles
  int n_units;       // work units (two query tiles each); the grid is n_units * n_split CTAs
  int n_split;       // key-range slices per unit (1: the CTA writes O and LSE itself)
  float* part_o;     // n_split > 1: fp32 [n_split][B*Hq][Lq][d], O of each slice normalised by its own sum
  float* part_lse;   // n_split > 1: fp32 [n_split][B*Hq][Lq], natural-log LSE of each slice (-inf: empty)
  // acc_mode (n_split == 1): part_o / part_lse are running fp32 accumulators
  // [B*Hq][Lq][d] and [B*Hq][Lq] of earlier key blocks (O normalised by its own
  // sum, natural-log LSE); the epilogue merges this launch's result into them
  // (acc_init: overwrites them instead) and writes no bf16 O.
  int acc_mode;
  int acc_init;
  int* err;          // device error word
  uint64_t limit_ns; // bounded-wait limit
};

struct BwdParams {
  CUtensorMap tm_q;   // [B*Hq, Lq, d], box 64 x BM x 1 (BM = query rows per step)
  CUtensorMap tm_do;  // [B*Hq, Lq, d], same box
  CUtensorMap tm_k;   // [B*Hkv, Lk, d], box 64 x 128 x 1
  CUtensorMap tm_v;   // [B*Hkv, Lk, d], same box
  Problem prob;
  const float* lse;   // fp32 [B, Hq, Lq], natural log (forward output)
  const float* dvec;  // fp32 [B, Hq, Lq], D_i = dO_i . O_i (workspace)
  float* dq_acc;      // fp32 [B*Hq, Lq, d]: dQ / scale summed over key tiles (workspace)
  CUtensorMap tm_dq;  // dq_acc as 3-D [B*Hq, Lq, d], box 128 x 32 x 1, no swizzle (d = 128)
  void* dk;           // bf16 [B, Hkv, Lk, d]
  void* dv;           // bf16 [B, Hkv, Lk, d]
  // Accumulate mode (both non-null): dK (already scaled) and dV are added into
  // these fp32 [B, Hkv, Lk, d] buffers instead of written to dk / dv
  // (dkv_init: stored instead of added).
  float* dk_acc;
  float* dv_acc;
  int dkv_init;
  // Self-test of the abort path (0 otherwise): with k > 0 the gradient warps
  // withhold their arrival for step k - 1, so a bounded wait runs out and the
  // kernel takes its abort path (attn_selftest_bwd_abort).
  int stall_at;
  float scale;
  float scale_log2;
  int n_units;        // CTAs: B * Hkv * key tiles
  int* err;
  uint64_t limit_ns;
};

// Kernels that move registers between warp roles with setmaxnreg are only
// correct at the register count their split was written for: a launch at any
// other count is refused before it starts.
inline cudaError_t check_launch_regs(const void* kernel, int expected) {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return e;
  return a.numRegs == expected ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// Per-device one-time set-up of a kernel (its dynamic shared-memory limit, the
// register-count check): `fn` runs until it first succeeds on the current
// device, later launches on that device skip it.  Concurrent first calls may
// both run it, which is harmless.
constexpr int kMaxDevices = 64;
template <typename Fn>
inline cudaError_t once_per_device(std::atomic<unsigned char> (&done)[kMaxDevices], Fn&& fn) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return fn();
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = fn();
  if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
  return e;
}

// Query rows per backward step for head dimension d.
inline int bwd_block_m(int d) { return d == 128 ? 64 : 128; }

// Workspace layout of the backward: D (fp32 [B*Hq*Lq], padded to 256 bytes), then
// the dQ accumulator fp32 [B*Hq, Lq, d].

cudaError_t launch_bwd_pre(const void* o, const void* dO, float* dvec, float* dq_acc, int64_t rows, int d,
                           int64_t acc_floats, cudaStream_t stream);
cudaError_t launch_bwd(const BwdParams& P, cudaStream_t stream);
// dq = bf16(scale * dq_acc), n elements.
cudaError_t launch_bwd_post(const float* dq_acc, void* dq, int64_t n, float scale, cudaStream_t stream);
// out[i] = bf16(acc[i]) (round to nearest even), n elements.
cudaError_t launch_f32_to_bf16(const float* acc, void* out, size_t n, cudaStream_t stream);

// Number of CTAs of the forward grid and whether heads are paired.
void fwd_plan(const Problem& p, int* n_units, int* pair_heads, int* packed, int* alternate);
// The C ABI's shape, mask and scale checks (ATTN_OK or the status to return).
int validate_problem(int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window);
// Records `step` and the error's text for attn_last_cuda_error; returns ATTN_ERR_CUDA.
int record_cuda_error(const char* step, cudaError_t e);
cudaError_t launch_fwd(const FwdParams& P, cudaStream_t stream);
// Combine n_split partial (O, LSE) of every row into bf16 O and fp32 LSE.
cudaError_t launch_fwd_merge(const FwdParams& P, cudaStream_t stream);

}  // namespace tea

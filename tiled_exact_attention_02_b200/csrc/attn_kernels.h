// attn_kernels.h - internal interface between the C ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "attn_common.cuh"

namespace tea {

struct FwdParams {
  CUtensorMap tm_q;  // [B*Hq, Lq, d] bf16, box 64 x 128 x 1, 128-byte swizzle
  CUtensorMap tm_k;  // [B*Hkv, Lk, d]
  CUtensorMap tm_v;  // [B*Hkv, Lk, d]
  Problem prob;
  void* o;           // bf16 [B, Hq, Lq, d]
  float* lse;        // fp32 [B, Hq, Lq]
  float scale_log2;  // scale * log2(e)
  int pair_heads;    // 1: a CTA takes two heads of one GQA group at the same rows
  int n_units;       // CTAs in the grid
  int* err;          // device error word
  uint64_t limit_ns; // bounded-wait limit
};

// Number of CTAs of the forward grid and whether heads are paired.
void fwd_plan(const Problem& p, int* n_units, int* pair_heads);
cudaError_t launch_fwd(const FwdParams& P, cudaStream_t stream);

}  // namespace tea

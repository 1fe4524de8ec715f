// noalloc.cu - attn_bwd for callers that cannot allocate device memory.
//
// attn_bwd needs a workspace (the per-row D values and an fp32 dQ
// accumulator) that the caller allocates.  Some callers cannot call cudaMalloc
// at all: a plugin running inside a host framework that owns every device
// allocation and hands out none, or code on a latency-critical path where
// cudaMalloc's implicit synchronisation and possible failure are not
// acceptable.  attn_bwd_noalloc serves them: it runs the same three backward
// phases with the workspace carved out of a fixed array in this library's
// own device memory, and allocates nothing.
//
// The array below is a file-scope __device__ object: every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits.  In host
// code its name is only a host-side stand-in, not a device address, so the
// device address is looked up with cudaGetSymbolAddress, once per device,
// with that device current, and passed to the kernels.
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "../../include/tiledattn.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices];

// Device address of the scratch array on the current device (set-up on the
// first call per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return ATTN_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                     int causal, int window, void* stream) {
  const size_t need = attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d);
  if (need > kNoallocScratchBytes) return ATTN_ERR_UNSUPPORTED;  // problem too large for the built-in scratch
  void* scratch = nullptr;
  if (need > 0) {
    const int st = scratch_address(&scratch);
    if (st != ATTN_OK) return st;
  }
  // The preprocess phase zeroes the dQ accumulator and rewrites D on every
  // call, so nothing left in the array by an earlier call is read.
  return attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, scratch,
                  need > 0 ? kNoallocScratchBytes : 0, stream);
}

}  // extern "C"

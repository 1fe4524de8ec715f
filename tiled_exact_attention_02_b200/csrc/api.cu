// api.cu - the C ABI: argument validation, TMA descriptors, launches, and the
// per-device error word.  See include/tiledattn.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdio>
#include <mutex>

#include "../../include/tiledattn.h"
#include "attn_kernels.h"
#include "sm100.cuh"

namespace tea {

// Error word of each device the library runs on: kernels record a bounded
// wait they gave up on; attn_get_device_error reads and clears it.
__device__ int g_dev_err;

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s without progress

std::mutex g_mu;
int* g_err_addr[kMaxDevices];

thread_local char g_last_err[256];

// Record a failed CUDA call for attn_last_cuda_error and map it to ATTN_ERR_CUDA.
int cuda_fail(const char* step, cudaError_t e) {
  snprintf(g_last_err, sizeof(g_last_err), "%s: %s (%d)", step, cudaGetErrorString(e), (int)e);
  return ATTN_ERR_CUDA;
}
int cu_fail(const char* step, CUresult r) {
  snprintf(g_last_err, sizeof(g_last_err), "%s: CUresult %d", step, (int)r);
  return ATTN_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Resolve the driver's tensor-map encoder once (no link-time libcuda dependency).
int get_encoder(EncodeTiledFn* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return cuda_fail("cudaGetDriverEntryPoint", e);
    if (q != cudaDriverEntryPointSuccess || !p) return cu_fail("cuTensorMapEncodeTiled lookup", CUDA_ERROR_NOT_FOUND);
    g_encode = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = g_encode;
  return ATTN_OK;
}

// Device address of the current device's error word (looked up once per device).
int get_err_word(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail("cudaGetDevice", cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dev_err);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress", e);
    g_err_addr[dev] = static_cast<int*>(p);
  }
  *out = g_err_addr[dev];
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared shape checks.  Returns ATTN_OK, or the error to report.
int check_shape(int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Lq < 0 || Lk < 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv == 0 && Hq > 0) return ATTN_ERR_INVALID_ARG;
  if (Hkv > 0 && Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (Hq == 0 && Hkv > 0) return ATTN_ERR_INVALID_ARG;
  if (causal < 0 || causal > 2) return ATTN_ERR_INVALID_ARG;
  if (window < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale <= 0.f) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  // Index arithmetic limits: rows per tensor and grid size stay in int range.
  if ((int64_t)B * Hq > (1 << 24) || (int64_t)B * Hkv > (1 << 24)) return ATTN_ERR_UNSUPPORTED;
  if (Lq > (1 << 28) || Lk > (1 << 28)) return ATTN_ERR_UNSUPPORTED;
  if ((int64_t)B * Hq * ((Lq + 127) / 128) >= (int64_t)1 << 31) return ATTN_ERR_UNSUPPORTED;
  if ((int64_t)B * Hkv * ((Lk + 127) / 128) >= (int64_t)1 << 31) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// 3-D map over a [BH, L, d] bf16 tensor, box 64 x box_rows x 1, 128-byte
// swizzle.  Rows past L inside a box read as zero.
int make_map(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, int BH, int L, int d, int box_rows = 128) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)(L > 0 ? L : 1), (cuuint64_t)(BH > 0 ? BH : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)(L > 0 ? L : 1)};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : cu_fail("cuTensorMapEncodeTiled", r);
}

__global__ void selftest_wait_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const WaitGuard g{err, &abort_flag, limit_ns, 0};
  // Nothing ever arrives on `bar`: the wait must give up by itself.
  mbar_wait(&bar, 0, g, 1000);
  __syncthreads();
}

}  // namespace

int validate_problem(int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window) {
  return check_shape(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
}

int record_cuda_error(const char* step, cudaError_t e) { return cuda_fail(step, e); }

}  // namespace tea

using namespace tea;

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

// Forward for every entry point: lens_q / lens_k optional per-sequence
// lengths (device int32 [B]); n_split > 1 cuts each unit's key range into
// slices written to `workspace` and merged.
// acc_o != NULL: accumulate mode (attn_fwd_accumulate): the result is merged
// into the fp32 accumulators acc_o / acc_lse (acc_init: written into them)
// and o / lse are not used.
static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, const int* lens_q,
                    const int* lens_k, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal,
                    int window, int gh, int gt, int sb, int n_split, void* workspace, void* stream,
                    float* acc_o = nullptr, float* acc_lse = nullptr, int acc_init = 0) {
  int st = check_shape(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (gh < 0 || gt < 0 || sb < 0 || sb > (1 << 28)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || Lq == 0) return ATTN_OK;
  if (acc_o) {
    if (!acc_lse || !aligned16(acc_o) || !aligned16(acc_lse) || n_split != 1) return ATTN_ERR_INVALID_ARG;
    o = acc_o;  // placeholders for the checks below; the kernel writes only the accumulators
    lse = acc_lse;
  }
  if (!q || !o || !lse || !aligned16(q) || !aligned16(o) || !aligned16(lse)) return ATTN_ERR_INVALID_ARG;
  if (Lk > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return ATTN_ERR_INVALID_ARG;
  if ((lens_q && (reinterpret_cast<uintptr_t>(lens_q) & 3u)) || (lens_k && (reinterpret_cast<uintptr_t>(lens_k) & 3u)))
    return ATTN_ERR_INVALID_ARG;
  EncodeTiledFn enc;
  if ((st = get_encoder(&enc)) != ATTN_OK) return st;
  FwdParams P;
  memset(&P, 0, sizeof(P));
  P.prob = Problem{B, Hq, Hkv, Lq, Lk, d, causal, window, scale};
  P.prob.len_q = lens_q;
  P.prob.len_k = lens_k;
  P.prob.global_head = gh;
  P.prob.global_tail = gt;
  P.prob.sparse_block = sb;
  // With Lk == 0 nothing reads K/V; map Q's memory so the descriptors stay valid.
  const void* kp = Lk > 0 ? k : q;
  const void* vp = Lk > 0 ? v : q;
  fwd_plan(P.prob, &P.n_units, &P.pair_heads, &P.packed, &P.alternate);
  // Packed rows read Q as [B*Hkv, G*Lq, d]: the G heads of a kv group are adjacent in memory.
  if ((st = P.packed ? make_map(enc, &P.tm_q, q, B * Hkv, (Hq / Hkv) * Lq, d) : make_map(enc, &P.tm_q, q, B * Hq, Lq, d)) !=
      ATTN_OK)
    return st;
  if ((st = make_map(enc, &P.tm_k, kp, Lk > 0 ? B * Hkv : B * Hq, Lk > 0 ? Lk : Lq, d)) != ATTN_OK) return st;
  if ((st = make_map(enc, &P.tm_v, vp, Lk > 0 ? B * Hkv : B * Hq, Lk > 0 ? Lk : Lq, d)) != ATTN_OK) return st;
  P.o = o;
  P.lse = lse;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.n_split = n_split;
  if (acc_o) {
    P.acc_mode = 1;
    P.acc_init = acc_init != 0;
    P.part_o = acc_o;
    P.part_lse = acc_lse;
    P.o = nullptr;
    P.lse = nullptr;
  }
  if (n_split > 1) {
    const size_t rows = (size_t)B * Hq * Lq;
    P.part_o = static_cast<float*>(workspace);
    P.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                          ((size_t)n_split * rows * d * 4 + 255) / 256 * 256);
    if ((int64_t)P.n_units * n_split > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
  }
  if ((st = get_err_word(&P.err)) != ATTN_OK) return st;
  P.limit_ns = kWaitLimitNs;
  cudaError_t e = launch_fwd(P, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("attn_fwd launch", e);
  if (n_split > 1) {
    e = launch_fwd_merge(P, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("attn_fwd_split merge launch", e);
  }
  return ATTN_OK;
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
             int Lk, int d, float scale, int causal, int window, void* stream) {
  return fwd_impl(q, k, v, o, lse, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0, 0, 0, 1, nullptr,
                  stream);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* seqlens_q,
                    const int* seqlens_k, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal,
                    int window, void* stream) {
  return fwd_impl(q, k, v, o, lse, seqlens_q, seqlens_k, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0, 0, 0, 1,
                  nullptr, stream);
}

// ------------------------------------------------------------------ split-KV forward
static constexpr int kMaxSplit = 64;

size_t attn_fwd_split_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d, int n_split) {
  if (check_shape(B, Hq, Hkv, Lq, Lk, d, 1.f, 0, 0) != ATTN_OK) return 0;
  if (n_split < 1 || n_split > kMaxSplit || B == 0 || Hq == 0 || Lq == 0) return 0;
  if (n_split == 1) return 0;
  const size_t rows = (size_t)B * Hq * Lq;
  return ((size_t)n_split * rows * d * 4 + 255) / 256 * 256 + ((size_t)n_split * rows * 4 + 255) / 256 * 256;
}

int attn_fwd_split_default(int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal, int window) {
  if (check_shape(B, Hq, Hkv, Lq, Lk, d, 1.f, causal, window) != ATTN_OK) return 1;
  if (B == 0 || Hq == 0 || Lq == 0 || Lk == 0) return 1;
  Problem p{B, Hq, Hkv, Lq, Lk, d, causal, window, 1.f};
  int n_units, pair, packed, alternate;
  fwd_plan(p, &n_units, &pair, &packed, &alternate);
  int sms = 148;
  int dev;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = (Lk + 127) / 128;
  const int n_max = imin(kMaxSplit, imax(1, tiles / 2));
  // Units with alternating slots hold few query rows (decoding): they stream
  // K/V and are bound by HBM once a wave fills the GPU, so more CTAs do not
  // shorten the stream, while a second wave adds its prologue, its partial
  // (O, LSE) writes and a tail that streams at one SM's rate.  Take the most
  // slices that still fit in one wave (measured on a B200 over decode shapes
  // of 8-64 kv groups and 4k-128k keys: always the fastest or within 2%).
  if (alternate) return imax(1, imin(n_max, sms / imax(1, n_units)));
  // Otherwise (compute-bound units) pick the slice count with the least
  // estimated time: waves of one CTA per SM, each as long as a slice's key
  // tiles plus about two tiles of fixed cost (Q load, pipeline fill,
  // epilogue); no slice shorter than two tiles.
  int best = 1;
  double best_t = 0;
  for (int n = 1; n <= n_max; n++) {
    const double waves = (double)((n_units * (int64_t)n + sms - 1) / sms);
    const double t = waves * ((double)tiles / n + 2.0);
    if (n == 1 || t < best_t) best = n, best_t = t;
  }
  return best;
}

int attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
                   int Lk, int d, float scale, int causal, int window, int n_split, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (n_split < 1 || n_split > kMaxSplit) return ATTN_ERR_INVALID_ARG;
  if (n_split == 1) return attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, stream);
  const int st = check_shape(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lq == 0) return ATTN_OK;
  const size_t need = attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, n_split);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return ATTN_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0, 0, 0, n_split,
                  workspace, stream);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d) {
  if (check_shape(B, Hq, Hkv, Lq, Lk, d, 1.f, 0, 0) != ATTN_OK) return 0;
  if (B == 0 || Hq == 0 || Lq == 0) return 0;
  const size_t rows = (size_t)B * Hq * Lq;
  const size_t dsz = (rows * 4 + 255) / 256 * 256;                                    // D, fp32
  const size_t dq = ((size_t)B * Hq * Lq * d * 4 + 255) / 256 * 256;                // dQ accumulator, fp32
  return dsz + dq;
}

// Workspace layout: D (fp32 [rows], padded to 256 bytes), then the fp32 dQ accumulator.
static int split_workspace(int B, int Hq, int Lq, int d, void* workspace, size_t workspace_bytes, float** dvec,
                           float** dq_acc) {
  const size_t need = attn_bwd_workspace_size(B, Hq, 1, Lq, 1, d);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return ATTN_ERR_INVALID_ARG;
  const size_t rows = (size_t)B * Hq * Lq;
  *dvec = static_cast<float*>(workspace);
  *dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + (rows * 4 + 255) / 256 * 256);
  return ATTN_OK;
}

int attn_bwd_preprocess(const void* o, const void* dO, int B, int Hq, int Lq, int d, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int st = check_shape(B, Hq, Hq > 0 ? 1 : 0, Lq, 1, d, 1.f, 0, 0);
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lq == 0) return ATTN_OK;
  if (!o || !dO || !aligned16(o) || !aligned16(dO)) return ATTN_ERR_INVALID_ARG;
  float *dvec, *dq_acc;
  if ((st = split_workspace(B, Hq, Lq, d, workspace, workspace_bytes, &dvec, &dq_acc)) != ATTN_OK) return st;
  const cudaError_t e = launch_bwd_pre(o, dO, dvec, dq_acc, (int64_t)B * Hq * Lq, d,
                                       (int64_t)B * Hq * Lq * d, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : cuda_fail("attn_bwd_preprocess launch", e);
}

// dk_acc != NULL: accumulate mode (attn_bwd_accumulate): dK and dV are added
// into the fp32 accumulators dk_acc / dv_acc (dkv_init: stored into them),
// and dk / dv are not used.
static int bwd_main_impl(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk,
                         void* dv, const int* lens_q, const int* lens_k, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                         float scale, int causal, int window, int gh, int gt, int sb, void* workspace,
                         size_t workspace_bytes, void* stream, float* dk_acc = nullptr, float* dv_acc = nullptr,
                         int dkv_init = 0, int stall_at = 0, uint64_t limit_ns = kWaitLimitNs) {
  int st = check_shape(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
  if (st == ATTN_OK && (gh < 0 || gt < 0 || sb < 0 || sb > (1 << 28))) st = ATTN_ERR_INVALID_ARG;
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lk == 0) return ATTN_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dk_acc) {
    if (!dv_acc || !aligned16(dk_acc) || !aligned16(dv_acc)) return ATTN_ERR_INVALID_ARG;
    dk = dk_acc;  // placeholders for the checks below; the kernel writes only the accumulators
    dv = dv_acc;
  }
  if (!k || !v || !dk || !dv || !aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv))
    return ATTN_ERR_INVALID_ARG;
  if (Lq == 0) {  // no query: dK = dV = 0 (an accumulator is only cleared when initialised here)
    if (dk_acc && !dkv_init) return ATTN_OK;
    const size_t kv_bytes = (size_t)B * Hkv * Lk * d * (dk_acc ? 4 : 2);
    cudaError_t e = cudaMemsetAsync(dk, 0, kv_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, s);
    return e == cudaSuccess ? ATTN_OK : cuda_fail("cudaMemsetAsync dK/dV", e);
  }
  if (!q || !lse || !dO || !aligned16(q) || !aligned16(lse) || !aligned16(dO)) return ATTN_ERR_INVALID_ARG;
  float *dvec, *dq_acc;
  if ((st = split_workspace(B, Hq, Lq, d, workspace, workspace_bytes, &dvec, &dq_acc)) != ATTN_OK) return st;
  EncodeTiledFn enc;
  if ((st = get_encoder(&enc)) != ATTN_OK) return st;
  BwdParams P;
  memset(&P, 0, sizeof(P));
  if ((lens_q && (reinterpret_cast<uintptr_t>(lens_q) & 3u)) || (lens_k && (reinterpret_cast<uintptr_t>(lens_k) & 3u)))
    return ATTN_ERR_INVALID_ARG;
  P.prob = Problem{B, Hq, Hkv, Lq, Lk, d, causal, window, scale};
  P.prob.len_q = lens_q;
  P.prob.len_k = lens_k;
  P.prob.global_head = gh;
  P.prob.global_tail = gt;
  P.prob.sparse_block = sb;
  const int bm = bwd_block_m(d);
  if ((st = make_map(enc, &P.tm_q, q, B * Hq, Lq, d, bm)) != ATTN_OK) return st;
  if ((st = make_map(enc, &P.tm_do, dO, B * Hq, Lq, d, bm)) != ATTN_OK) return st;
  if ((st = make_map(enc, &P.tm_k, k, B * Hkv, Lk, d, 128)) != ATTN_OK) return st;
  if ((st = make_map(enc, &P.tm_v, v, B * Hkv, Lk, d, 128)) != ATTN_OK) return st;
  P.lse = lse;
  P.dvec = dvec;
  P.dq_acc = dq_acc;
  if (d == 128) {
    // dQ accumulator as a 3-D fp32 tensor [B*Hq, Lq, d]: each step's 64-query
    // tile is added as two boxes of 32 query rows x 128 d (rows past a head's
    // Lq fall outside the tensor and are dropped).
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)Lq, (cuuint64_t)B * Hq};
    cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)Lq * d * 4};
    cuuint32_t box[3] = {128, 32, 1};
    cuuint32_t es[3] = {1, 1, 1};
    const CUresult r = enc(&P.tm_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dq_acc, dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cu_fail("cuTensorMapEncodeTiled dQ", r);
  }
  P.dk = dk;
  P.dv = dv;
  if (dk_acc) {
    P.dk_acc = dk_acc;
    P.dv_acc = dv_acc;
    P.dkv_init = dkv_init != 0;
  }
  P.scale = scale;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.n_units = B * Hkv * ((Lk + 127) / 128);
  P.stall_at = stall_at;
  if ((st = get_err_word(&P.err)) != ATTN_OK) return st;
  P.limit_ns = limit_ns;
  const cudaError_t e = launch_bwd(P, s);
  return e == cudaSuccess ? ATTN_OK : cuda_fail("attn_bwd_main launch", e);
}

int attn_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk, void* dv,
                  int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return bwd_main_impl(q, k, v, lse, dO, dk, dv, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0,
                       0, 0, workspace, workspace_bytes, stream);
}

int attn_bwd_main_varlen(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk,
                         void* dv, const int* seqlens_q, const int* seqlens_k, int B, int Hq, int Hkv, int Lq, int Lk,
                         int d, float scale, int causal, int window, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return bwd_main_impl(q, k, v, lse, dO, dk, dv, seqlens_q, seqlens_k, B, Hq, Hkv, Lq, Lk, d, scale, causal, window,
                       0, 0, 0, workspace, workspace_bytes, stream);
}

int attn_bwd_finalize(void* dq, int B, int Hq, int Lq, int d, float scale, void* workspace, size_t workspace_bytes,
                      void* stream) {
  int st = check_shape(B, Hq, Hq > 0 ? 1 : 0, Lq, 1, d, scale, 0, 0);
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lq == 0) return ATTN_OK;
  if (!dq || !aligned16(dq)) return ATTN_ERR_INVALID_ARG;
  float *dvec, *dq_acc;
  if ((st = split_workspace(B, Hq, Lq, d, workspace, workspace_bytes, &dvec, &dq_acc)) != ATTN_OK) return st;
  const cudaError_t e = launch_bwd_post(dq_acc, dq, (int64_t)B * Hq * Lq * d, scale, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : cuda_fail("attn_bwd_finalize launch", e);
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, const int* lens_q, const int* lens_k, int B, int Hq, int Hkv, int Lq,
                    int Lk, int d, float scale, int causal, int window, int gh, int gt, int sb, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int st = check_shape(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (gh < 0 || gt < 0 || sb < 0 || sb > (1 << 28)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0) return ATTN_OK;
  if (Lq == 0 || Lk == 0) {
    if (Lq == 0)  // dK = dV = 0
      return bwd_main_impl(q, k, v, lse, dO, dk, dv, lens_q, lens_k, B, Hq, Hkv, Lq, Lk, d, scale, causal, window,
                           gh, gt, sb, workspace, workspace_bytes, stream);
    // No key: every row is fully masked, dQ = 0.
    if (!dq || !aligned16(dq)) return ATTN_ERR_INVALID_ARG;
    const cudaError_t e = cudaMemsetAsync(dq, 0, (size_t)B * Hq * Lq * d * 2, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : cuda_fail("cudaMemsetAsync dQ", e);
  }
  // Validate every pointer before the first launch.
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return ATTN_ERR_INVALID_ARG;
  float *dvec, *dq_acc;
  if ((st = split_workspace(B, Hq, Lq, d, workspace, workspace_bytes, &dvec, &dq_acc)) != ATTN_OK) return st;
  if ((st = attn_bwd_preprocess(o, dO, B, Hq, Lq, d, workspace, workspace_bytes, stream)) != ATTN_OK) return st;
  if ((st = bwd_main_impl(q, k, v, lse, dO, dk, dv, lens_q, lens_k, B, Hq, Hkv, Lq, Lk, d, scale, causal, window,
                          gh, gt, sb, workspace, workspace_bytes, stream)) != ATTN_OK)
    return st;
  return attn_bwd_finalize(dq, B, Hq, Lq, d, scale, workspace, workspace_bytes, stream);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
             void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window,
             void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0,
                  0, 0, workspace, workspace_bytes, stream);
}

int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, const int* seqlens_q, const int* seqlens_k, int B, int Hq, int Hkv,
                    int Lq, int Lk, int d, float scale, int causal, int window, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, seqlens_q, seqlens_k, B, Hq, Hkv, Lq, Lk, d, scale, causal, window,
                  0, 0, 0, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ accumulate (ring attention)
int attn_fwd_accumulate(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, int B, int Hq,
                        int Hkv, int Lq, int Lk, int d, float scale, int causal, int window, int init, void* stream) {
  if (!o_acc || !lse_acc) return ATTN_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0, 0, 0,
                  1, nullptr, stream, o_acc, lse_acc, init);
}

int attn_fwd_accumulate_finalize(const float* o_acc, const float* lse_acc, void* o, float* lse, int B, int Hq, int Lq,
                                 int d, void* stream) {
  const int st = check_shape(B, Hq, Hq > 0 ? 1 : 0, Lq, 1, d, 1.f, 0, 0);
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lq == 0) return ATTN_OK;
  if (!o_acc || !lse_acc || !o || !lse || !aligned16(o_acc) || !aligned16(lse_acc) || !aligned16(o) ||
      !aligned16(lse))
    return ATTN_ERR_INVALID_ARG;
  FwdParams P;
  memset(&P, 0, sizeof(P));
  P.prob = Problem{B, Hq, 1, Lq, 1, d, 0, 0, 1.f};
  P.part_o = const_cast<float*>(o_acc);
  P.part_lse = const_cast<float*>(lse_acc);
  P.o = o;
  P.lse = lse;
  P.n_split = 1;  // one "slice": O = the accumulator rounded to bf16, LSE copied
  const cudaError_t e = launch_fwd_merge(P, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : cuda_fail("attn_fwd_accumulate_finalize launch", e);
}

int attn_bwd_accumulate(const void* q, const void* k, const void* v, const float* lse, const void* dO, float* dk_acc,
                        float* dv_acc, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal,
                        int window, int init, void* workspace, size_t workspace_bytes, void* stream) {
  if (!dk_acc || !dv_acc) return ATTN_ERR_INVALID_ARG;
  return bwd_main_impl(q, k, v, lse, dO, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal,
                       window, 0, 0, 0, workspace, workspace_bytes, stream, dk_acc, dv_acc, init);
}

int attn_accumulator_to_bf16(const float* acc, void* out, size_t n, void* stream) {
  if (n == 0) return ATTN_OK;
  if (!acc || !out || !aligned16(acc) || !aligned16(out)) return ATTN_ERR_INVALID_ARG;
  if (n > ((size_t)1 << 40)) return ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_f32_to_bf16(acc, out, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : cuda_fail("attn_accumulator_to_bf16 launch", e);
}

const char* attn_last_cuda_error(void) { return g_last_err; }

int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
                int Lk, int d, float scale, const attn_mask* mask, int n_split, void* workspace,
                size_t workspace_bytes, void* stream) {
  if (!mask) return ATTN_ERR_INVALID_ARG;
  if (n_split < 1 || n_split > kMaxSplit) return ATTN_ERR_INVALID_ARG;
  if (n_split > 1) {
    const int st = check_shape(B, Hq, Hkv, Lq, Lk, d, scale, mask->causal, mask->window);
    if (st != ATTN_OK) return st;
    const size_t need = attn_fwd_split_workspace_size(B, Hq, Hkv, Lq, Lk, d, n_split);
    if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need))
      return ATTN_ERR_INVALID_ARG;
  }
  return fwd_impl(q, k, v, o, lse, mask->seqlens_q, mask->seqlens_k, B, Hq, Hkv, Lq, Lk, d, scale, mask->causal,
                  mask->window, mask->global_head, mask->global_tail, mask->sparse_block, n_split, workspace, stream);
}

int attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
                void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, const attn_mask* mask,
                void* workspace, size_t workspace_bytes, void* stream) {
  if (!mask) return ATTN_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, mask->seqlens_q, mask->seqlens_k, B, Hq, Hkv, Lq, Lk, d, scale,
                  mask->causal, mask->window, mask->global_head, mask->global_tail, mask->sparse_block, workspace,
                  workspace_bytes, stream);
}

int attn_get_device_error(void* stream, int* site) {
  int* addr = nullptr;
  int st = get_err_word(&addr);
  if (st != ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail("cudaStreamSynchronize", e);
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_dev_err, sizeof(int));
  if (e != cudaSuccess) return cuda_fail("read error word", e);
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail("clear error word", e);
  if (site) *site = word >> 8;
  return (word & 0xFF) == DEV_TIMEOUT ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

int attn_selftest_bwd_abort(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                            float scale, int causal, int window, int stall_step, int64_t limit_ns, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (stall_step < 0 || limit_ns <= 0 || limit_ns > (int64_t)10000000000ll) return ATTN_ERR_INVALID_ARG;
  int st = check_shape(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lq == 0 || Lk == 0) return ATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if ((st = attn_bwd_preprocess(o, dO, B, Hq, Lq, d, workspace, workspace_bytes, stream)) != ATTN_OK) return st;
  if ((st = bwd_main_impl(q, k, v, lse, dO, dk, dv, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, causal, window, 0,
                          0, 0, workspace, workspace_bytes, stream, nullptr, nullptr, 0, stall_step + 1,
                          (uint64_t)limit_ns)) != ATTN_OK)
    return st;
  return attn_bwd_finalize(dq, B, Hq, Lq, d, scale, workspace, workspace_bytes, stream);
}

int attn_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > (int64_t)10000000000ll) return ATTN_ERR_INVALID_ARG;
  int* err = nullptr;
  int st = get_err_word(&err);
  if (st != ATTN_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, (uint64_t)limit_ns);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : cuda_fail("selftest launch", e);
}

}  // extern "C"

// host_step.cu - the attention step with host buffers, copies overlapped with
// the kernels.
//
// attn_step_host takes Q, K, V (and dO) in host memory, runs the forward (and
// the backward) on the device, and writes O and LSE (and dQ, dK, dV) back to
// host memory, staging everything in one device buffer that the caller owns.
// The problem is cut into chunks of whole kv-head groups of one sequence;
// each chunk is an independent attention problem (a kv head's dK and dV only
// depend on its own G query heads).  Chunk c's inputs are copied in on one
// stream, its kernels run on a second and its outputs are copied out on a
// third, so with page-locked host memory the copies in both directions run
// at the same time as each other and as the kernels of neighbouring chunks.
// The caller's stream first orders the internal streams after its earlier
// work and then waits for the last copy out, so the call is asynchronous like
// every other entry point.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <vector>

#include "../../include/tiledattn.h"
#include "attn_kernels.h"

namespace {

// About eight chunks: with 16 or 32 the fwd+bwd workload's step measured the
// same (it is bound by the PCIe copies), with fewer the copies in and out of
// the first and last chunks are exposed for longer.
constexpr int kTargetChunks = 8;

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Chunk index at which the next attn_step_host call pretends that its copy
// in failed (-1: none), set by attn_selftest_step_host_fail_at; it exercises
// the error path after earlier chunks are already queued, without a GPU fault.
std::atomic<int> g_fail_at{-1};

// Byte offsets of every staged tensor inside the device buffer.  LSE is
// staged per chunk (a chunk's rows start at any multiple of 4 bytes inside
// the whole LSE, and the kernels want 16-byte aligned pointers).  The backward
// workspace `ws` (D and the fp32 dQ accumulator) is one region shared by all
// chunks: that is only safe because every chunk's kernels run in order on the
// single compute stream, so chunk c's attn_bwd starts after chunk c-1's has
// finished with it.
struct Staging {
  size_t q, k, v, dO, o, lse, lse_chunk, dq, dk, dv, ws, ws_bytes, total;
};

// kv heads per chunk: about kTargetChunks chunks over the B * Hkv groups,
// never across a sequence.
int kv_per_chunk(int B, int Hkv) {
  const long long groups = (long long)B * Hkv;
  long long kc = (groups + kTargetChunks - 1) / kTargetChunks;
  if (kc < 1) kc = 1;
  if (kc > Hkv) kc = Hkv;
  return (int)kc;
}

Staging staging(int B, int Hq, int Hkv, int Lq, int Lk, int d, bool bwd) {
  Staging s{};
  const size_t nq = (size_t)B * Hq * Lq * d * 2, nk = (size_t)B * Hkv * Lk * d * 2;
  const int kc = kv_per_chunk(B, Hkv);
  const int G = Hq / Hkv;
  const size_t n_chunks = (size_t)B * ((Hkv + kc - 1) / kc);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  s.q = take(nq);
  s.k = take(nk);
  s.v = take(nk);
  s.o = take(nq);
  s.lse_chunk = align256((size_t)kc * G * Lq * 4);
  s.lse = take(s.lse_chunk * n_chunks);
  if (bwd) {
    s.dO = take(nq);
    s.dq = take(nq);
    s.dk = take(nk);
    s.dv = take(nk);
    s.ws_bytes = attn_bwd_workspace_size(1, kc * G, kc, Lq, Lk, d);
    s.ws = take(s.ws_bytes);
  }
  s.total = off;
  return s;
}


// Streams and events of one call; released on every return path.  A stream
// or event destroyed with work still pending is released once that work ends.
// If the call fails after work was queued (`quiesce` still set), the
// destructor first waits for the three internal streams, so that no copy of
// an earlier chunk still reads or writes the caller's buffers when the error
// is returned.
struct CallResources {
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> events;
  bool quiesce = false;
  ~CallResources() {
    if (quiesce) {
      for (cudaStream_t s : {s_in, s_comp, s_out})
        if (s) cudaStreamSynchronize(s);
    }
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_comp) cudaStreamDestroy(s_comp);
    if (s_out) cudaStreamDestroy(s_out);
  }
  cudaError_t event(cudaEvent_t* e) {
    cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
    if (r == cudaSuccess) events.push_back(*e);
    return r;
  }
};

}  // namespace

extern "C" {

size_t attn_step_host_buffer_size(int B, int Hq, int Hkv, int Lq, int Lk, int d, int with_backward) {
  if (tea::validate_problem(B, Hq, Hkv, Lq, Lk, d, 1.f, 0, 0) != ATTN_OK || B == 0 || Hq == 0 || Lq == 0) return 0;
  return staging(B, Hq, Hkv, Lq, Lk, d, with_backward != 0).total;
}

int attn_step_host(const void* q, const void* k, const void* v, const void* dO, void* o, float* lse, void* dq,
                   void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal,
                   int window, void* dev_buf, size_t dev_buf_bytes, void* stream) {
  int st = tea::validate_problem(B, Hq, Hkv, Lq, Lk, d, scale, causal, window);
  if (st != ATTN_OK) return st;
  if (B == 0 || Hq == 0 || Lq == 0) return ATTN_OK;
  const bool bwd = dO != nullptr;
  if (!q || !o || !lse || (Lk > 0 && (!k || !v)) || (bwd && (!dq || !dk || !dv))) return ATTN_ERR_INVALID_ARG;
  const Staging S = staging(B, Hq, Hkv, Lq, Lk, d, bwd);
  if (!dev_buf || (reinterpret_cast<uintptr_t>(dev_buf) & 255u) || dev_buf_bytes < S.total)
    return ATTN_ERR_INVALID_ARG;

  uint8_t* base = static_cast<uint8_t*>(dev_buf);
  const int G = Hq / Hkv;
  const int kc = kv_per_chunk(B, Hkv);
  CallResources R;
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&R.s_in, cudaStreamNonBlocking)) != cudaSuccess ||
      (e = cudaStreamCreateWithFlags(&R.s_comp, cudaStreamNonBlocking)) != cudaSuccess ||
      (e = cudaStreamCreateWithFlags(&R.s_out, cudaStreamNonBlocking)) != cudaSuccess)
    return tea::record_cuda_error("attn_step_host streams", e);
  cudaStream_t caller = static_cast<cudaStream_t>(stream);
  cudaEvent_t start;
  if ((e = R.event(&start)) != cudaSuccess || (e = cudaEventRecord(start, caller)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(R.s_in, start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(R.s_out, start, 0)) != cudaSuccess)
    return tea::record_cuda_error("attn_step_host start", e);

  // From here on, an error return waits for what was queued (see CallResources).
  R.quiesce = true;
  const int fail_at = g_fail_at.exchange(-1);
  int chunk = 0;
  for (int b = 0; b < B; b++) {
    for (int kv0 = 0; kv0 < Hkv; kv0 += kc, chunk++) {
      const int nkv = kv0 + kc <= Hkv ? kc : Hkv - kv0;
      const int hc = nkv * G;
      const size_t qe = ((size_t)b * Hq + (size_t)kv0 * G) * Lq;  // first query row of the chunk
      const size_t ke = ((size_t)b * Hkv + kv0) * Lk;             // first key row
      const size_t qb = (size_t)hc * Lq * d * 2, kb = (size_t)nkv * Lk * d * 2, lb = (size_t)hc * Lq * 4;
      auto in = [&](size_t dst, const void* src, size_t row, size_t bytes) {
        return cudaMemcpyAsync(base + dst + row * d * 2, static_cast<const uint8_t*>(src) + row * d * 2, bytes,
                               cudaMemcpyHostToDevice, R.s_in);
      };
      auto out = [&](void* dst, size_t src, size_t off, size_t bytes) {
        return cudaMemcpyAsync(static_cast<uint8_t*>(dst) + off, base + src + off, bytes, cudaMemcpyDeviceToHost,
                               R.s_out);
      };
      if (chunk == fail_at) return tea::record_cuda_error("attn_step_host copy in (self-test)", cudaErrorUnknown);
      if ((e = in(S.q, q, qe, qb)) != cudaSuccess ||
          (kb > 0 && ((e = in(S.k, k, ke, kb)) != cudaSuccess || (e = in(S.v, v, ke, kb)) != cudaSuccess)) ||
          (bwd && (e = in(S.dO, dO, qe, qb)) != cudaSuccess))
        return tea::record_cuda_error("attn_step_host copy in", e);
      cudaEvent_t ready, done;
      if ((e = R.event(&ready)) != cudaSuccess || (e = R.event(&done)) != cudaSuccess ||
          (e = cudaEventRecord(ready, R.s_in)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(R.s_comp, ready, 0)) != cudaSuccess)
        return tea::record_cuda_error("attn_step_host events", e);

      uint8_t* cq = base + S.q + qe * d * 2;
      uint8_t* ck = base + S.k + ke * d * 2;
      uint8_t* cv = base + S.v + ke * d * 2;
      uint8_t* co = base + S.o + qe * d * 2;
      const size_t cl_off = S.lse + (size_t)chunk * S.lse_chunk;
      float* cl = reinterpret_cast<float*>(base + cl_off);
      st = attn_fwd(cq, ck, cv, co, cl, 1, hc, nkv, Lq, Lk, d, scale, causal, window, R.s_comp);
      if (st != ATTN_OK) return st;
      if (bwd) {
        st = attn_bwd(cq, ck, cv, co, cl, base + S.dO + qe * d * 2, base + S.dq + qe * d * 2,
                      base + S.dk + ke * d * 2, base + S.dv + ke * d * 2, 1, hc, nkv, Lq, Lk, d, scale, causal,
                      window, base + S.ws, S.ws_bytes, R.s_comp);
        if (st != ATTN_OK) return st;
      }
      if ((e = cudaEventRecord(done, R.s_comp)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(R.s_out, done, 0)) != cudaSuccess)
        return tea::record_cuda_error("attn_step_host events", e);
      if ((e = out(o, S.o, qe * d * 2, qb)) != cudaSuccess || (e = cudaMemcpyAsync(lse + qe, base + cl_off, lb, cudaMemcpyDeviceToHost, R.s_out)) != cudaSuccess ||
          (bwd && ((e = out(dq, S.dq, qe * d * 2, qb)) != cudaSuccess ||
                   (kb > 0 && ((e = out(dk, S.dk, ke * d * 2, kb)) != cudaSuccess ||
                               (e = out(dv, S.dv, ke * d * 2, kb)) != cudaSuccess)))))
        return tea::record_cuda_error("attn_step_host copy out", e);
    }
  }
  cudaEvent_t end;
  if ((e = R.event(&end)) != cudaSuccess || (e = cudaEventRecord(end, R.s_out)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(caller, end, 0)) != cudaSuccess)
    return tea::record_cuda_error("attn_step_host end", e);
  R.quiesce = false;  // the caller's stream now orders everything after the call's work
  return ATTN_OK;
}

int attn_selftest_step_host_fail_at(int chunk) {
  if (chunk < -1) return ATTN_ERR_INVALID_ARG;
  g_fail_at.store(chunk);
  return ATTN_OK;
}

}  // extern "C"

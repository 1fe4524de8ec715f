/*
 * tiledattn.h - C ABI of the tiled exact attention library (sm_100a, B200).
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T + mask) V
 *
 * ("注意力优化：FlashAttention 与稀疏注意力", 核心公式: S = QK^T/sqrt(d_k), a row
 * softmax whose rows sum to 1, output row i = sum_j A_ij V_j, and disallowed
 * keys set to -inf before the softmax), tile by tile with an online softmax so
 * that the score matrix never reaches device memory ("缩放定律与高效注意力"
 * §3.2, tiling and the incremental max/sum; "高效注意力：FlashAttention 与线性
 * 注意力", 原理与机制: the running max and sum rescaled by e^{m_old - m_new}).
 * The backward pass recomputes the scores from the saved output and per-row
 * logsumexp ("缩放定律与高效注意力" §3.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are contiguous, row-major, [B, H, L, d]; Q/O/dO/dQ have H = Hq,
 *    K/V/dK/dV have H = Hkv.  bf16 tensors hold IEEE bfloat16 bit patterns.
 *  - GQA/MQA ("高效注意力" §3): Hq must be a multiple of Hkv; query head h
 *    reads K/V head h / (Hq / Hkv) (contiguous groups).
 *  - Masks: causal = 1 makes key j visible to query i only if j <= i (top-left
 *    alignment); causal = 2 only if j <= i + Lk - Lq (bottom-right alignment:
 *    the last query sits at the last key, as for new queries over a longer
 *    cache of earlier keys; the same as causal = 1 when Lq = Lk).  window =
 *    w > 0 further restricts it to a band ("高效注意力" §4, sliding-window
 *    attention): with causal to the w keys ending at the query's diagonal
 *    (i + off - w < j <= i + off, off = 0 or Lk - Lq); with causal = 0 to the
 *    two-sided band i - w < j < i + w (w - 1 keys on either side of i, and
 *    i).  window = 0 means no window.  causal outside {0, 1, 2} or window < 0
 *    is ATTN_ERR_INVALID_ARG.
 *  - A query row that sees no key gets O = 0 and LSE = -inf (and dQ = 0).
 *  - LSE is the natural logarithm of sum_j exp(scale * q_i . k_j) over visible j.
 *  - Supported head dimension: d = 64 or d = 128 (d_k = d_v = d).
 *  - Every device pointer must be 16-byte aligned and point to memory of the
 *    current CUDA device.  All buffers are owned by the caller; the library
 *    allocates nothing and keeps no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous on that stream.  Argument errors are detected and
 *    returned before anything is launched; launch failures return
 *    ATTN_ERR_CUDA.  No C++ exception crosses this interface.
 *  - Every device-side wait is bounded.  If a kernel gives up waiting, it
 *    records ATTN_ERR_TIMEOUT in a per-device error word, which
 *    attn_get_device_error() reports; its outputs are then undefined.
 *  - Empty problems (B, Hq, Lq = 0) are valid and launch nothing.  Lk = 0 is
 *    valid: every row sees no key.
 *  - The library looks up the device addresses of its own device-side objects
 *    (the error word, the attn_bwd_noalloc scratch array) once per device and
 *    keeps them: do not use it on a device across cudaDeviceReset(), which
 *    may move them.
 */
#ifndef TILEDATTN_H
#define TILEDATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad mask, Hq % Hkv != 0 */
  ATTN_ERR_UNSUPPORTED = 2, /* valid but not implemented (head dim other than 64/128, too large) */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  ATTN_ERR_TIMEOUT = 4      /* a kernel abandoned a bounded wait (see attn_get_device_error) */
} attn_status;

/*
 * Forward pass ("缩放定律与高效注意力" §3.2; output O and the per-row logsumexp
 * that §3.3 says the backward pass needs).
 *
 *  q    bf16 [B, Hq,  Lq, d]   input
 *  k    bf16 [B, Hkv, Lk, d]   input
 *  v    bf16 [B, Hkv, Lk, d]   input
 *  o    bf16 [B, Hq,  Lq, d]   output (rounded to nearest even from fp32)
 *  lse  fp32 [B, Hq,  Lq]      output, natural log
 *  scale  multiplies Q K^T (1/sqrt(d) for standard attention); must be finite
 *
 * Returns ATTN_OK or an attn_status error code.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
             int Lk, int d, float scale, int causal, int window, void* stream);

/*
 * Every mask option at once, for attn_fwd_ex / attn_bwd_ex.
 *  causal, window          as attn_fwd (causal 0 / 1 / 2, window 0 or w > 0)
 *  global_head, global_tail  >= 0: that many leading / trailing key positions
 *                          (of each sequence) are visible to every query on
 *                          top of the window, still subject to the causal
 *                          mask ("大模型高效注意力机制全解析" §5.1.2,
 *                          global_tokens [0, -1]: the first and last tokens
 *                          globally visible); 0 for none
 *  seqlens_q, seqlens_k    as attn_fwd_varlen (device int32 [B] or NULL)
 *  sparse_block            b >= 0: the block-sparse mask of
 *                          "大模型高效注意力机制全解析" §4.1.2 with b x b
 *                          blocks (0 for none): the query block starting at
 *                          s = b * floor(i / b) sees the key blocks starting
 *                          at every j in [s - b, s + b), i.e. keys
 *                          [max(0, s - b), min(Lk, s + 2b - 1)); intersected
 *                          with the causal and window masks (global keys stay
 *                          visible on top).  b <= 2^28.
 */
typedef struct {
  int causal;
  int window;
  int global_head;
  int global_tail;
  const int* seqlens_q;
  const int* seqlens_k;
  int sparse_block;
} attn_mask;

/*
 * Forward pass with any combination of the mask options above, optionally
 * split across the key range (n_split as attn_fwd_split, 1 = no split; the
 * workspace is only needed for n_split > 1).  Global tokens add the key
 * tiles of the global positions to each query tile's walk.
 */
ATTN_API int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int Lq, int Lk, int d, float scale, const attn_mask* mask, int n_split, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Backward pass with any combination of the mask options (workspace as attn_bwd). */
ATTN_API int attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                         float scale, const attn_mask* mask, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward pass over a padded batch of sequences of different lengths
 * ("大模型高效注意力机制全解析" §5.2.2: requests are padded into one batch and
 * each output cut back to its own length).  Tensors keep the padded [B, H, L,
 * d] layout of attn_fwd; sequence b is its own attention problem over its
 * first seqlens_q[b] queries and seqlens_k[b] keys (a bottom-right causal
 * diagonal is placed by those lengths).  Padded query rows get O = 0 and LSE =
 * -inf; padded keys are never visible.  Key tiles past a sequence's end are
 * skipped.
 *
 *  seqlens_q, seqlens_k  device int32 [B] (4-byte aligned), or NULL for "all
 *                        Lq" / "all Lk"; values are clamped to [0, Lq] and
 *                        [0, Lk].  Read by the kernels, not by the host.
 *  other arguments       as attn_fwd.
 */
ATTN_API int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* seqlens_q,
                             const int* seqlens_k, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                             int causal, int window, void* stream);

/*
 * Forward pass with the key range split across CTAs (for few query rows over
 * many keys, e.g. new queries over a long cache with causal = 2).  Each query
 * tile's visible key tiles are cut into n_split contiguous slices, each
 * computed by its own CTA into an fp32 partial (O normalised by the slice's
 * own sum, and the slice's LSE).  A second kernel then combines the slices
 * exactly, with weights exp(LSE_k - max_k LSE_k): the online-softmax merge of
 * "高效注意力：FlashAttention 与线性注意力" 原理与机制 applied to whole slices.
 * The result equals attn_fwd's up to rounding.
 *
 *  q, k, v, o, lse, sizes, scale, causal, window: as attn_fwd.
 *  n_split    1..64 slices (1: plain attn_fwd, the workspace is not used).
 *  workspace  caller-owned device memory, 256-byte aligned, at least
 *             attn_fwd_split_workspace_size(...) bytes; overwritten.
 *
 * Returns ATTN_OK or an attn_status error code (n_split out of range or a
 * short / misaligned workspace: ATTN_ERR_INVALID_ARG).
 */
ATTN_API int attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                            int Lq, int Lk, int d, float scale, int causal, int window, int n_split, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Workspace bytes attn_fwd_split needs: n_split x (fp32 O [B,Hq,Lq,d] + fp32
 * LSE [B,Hq,Lq]), each part padded to 256 bytes.  0 for n_split = 1, an empty
 * problem or invalid sizes. */
ATTN_API size_t attn_fwd_split_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d, int n_split);

/* A slice count for this problem on the current device; no slice shorter
 * than two 128-key tiles, at most 64; 1 when splitting would not help.
 * Host-only (no launch).
 * - Few query rows per kv group (the units pack them into one slot that both
 *   slots share: decoding): the most slices that still fit in one wave of one
 *   CTA per SM.  These CTAs stream K/V at the HBM rate; a second wave only
 *   adds fixed work and a tail.
 * - Otherwise: the count with the least estimated time when CTAs run in waves
 *   of one per SM and each costs its slice's key tiles plus about two tiles of
 *   fixed work. */
ATTN_API int attn_fwd_split_default(int B, int Hq, int Hkv, int Lq, int Lk, int d, int causal, int window);

/*
 * Bytes of device workspace attn_bwd needs for this shape: the per-row
 * D_i = dO_i . O_i (fp32 [B,Hq,Lq]) and an fp32 dQ accumulator [B,Hq,Lq,d].
 * Returns 0 for an empty problem or invalid sizes.
 */
ATTN_API size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d);

/*
 * Backward pass by recomputation ("缩放定律与高效注意力" §3.3: only O and the
 * per-row logsumexp are kept; Q, K, V are re-read and the scores rebuilt tile
 * by tile).  Gradients are the textbook softmax gradient:
 *   D_i = dO_i . O_i,  P = exp(scale*S - LSE),  dV = P^T dO,  dP = dO V^T,
 *   dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 *  q, k, v, o, lse   the forward's inputs and outputs (same shapes as above)
 *  dO   bf16 [B, Hq, Lq, d]   upstream gradient
 *  dq   bf16 [B, Hq, Lq, d]   output
 *  dk   bf16 [B, Hkv, Lk, d]  output, summed over the Hq/Hkv query heads of a group
 *  dv   bf16 [B, Hkv, Lk, d]  output, summed likewise
 *  workspace  device buffer of at least attn_bwd_workspace_size(...) bytes,
 *             256-byte aligned; its contents on entry do not matter
 */
ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
             void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window,
             void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_bwd over a padded batch (see attn_fwd_varlen): the same lengths as the
 * forward pass; padded query rows get dQ = 0 and padded keys dK = dV = 0.
 */
ATTN_API int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, void* dq, void* dk, void* dv, const int* seqlens_q, const int* seqlens_k,
                             int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three phases attn_bwd runs, for callers that schedule or time them
 * separately (same arguments and rules as attn_bwd; call them in this order
 * on one stream with the same workspace):
 *   attn_bwd_preprocess  D_i = dO_i . O_i into the workspace, zero the dQ accumulator
 *   attn_bwd_main        recompute P tile by tile; write dK, dV; accumulate dQ
 *   attn_bwd_finalize    dQ = scale * accumulator, rounded to bf16
 */
ATTN_API int attn_bwd_preprocess(const void* o, const void* dO, int B, int Hq, int Lq, int d, void* workspace,
                                 size_t workspace_bytes, void* stream);
ATTN_API int attn_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk,
                           void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window,
                           void* workspace, size_t workspace_bytes, void* stream);

/* attn_bwd_main over a padded batch (phase 2 of attn_bwd_varlen). */
ATTN_API int attn_bwd_main_varlen(const void* q, const void* k, const void* v, const float* lse, const void* dO,
                                  void* dk, void* dv, const int* seqlens_q, const int* seqlens_k, int B, int Hq,
                                  int Hkv, int Lq, int Lk, int d, float scale, int causal, int window,
                                  void* workspace, size_t workspace_bytes, void* stream);
ATTN_API int attn_bwd_finalize(void* dq, int B, int Hq, int Lq, int d, float scale, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * attn_bwd without a workspace argument, for callers that cannot allocate
 * device memory (for example a plugin inside a framework that owns every
 * device allocation, or a latency-critical path that must not call
 * cudaMalloc).  It allocates nothing: the workspace lives in a fixed 32 MiB
 * array of the library's own device memory, which every GPU that loads the
 * library holds until the process exits.  The pages have no counterpart;
 * this is a deployment convenience.
 *
 *  - Arguments, layouts and results are those of attn_bwd.
 *  - Problems whose attn_bwd_workspace_size exceeds 32 MiB (33554432 bytes)
 *    return ATTN_ERR_UNSUPPORTED before anything runs; at d = 128 that is
 *    about 65,000 query rows (B * Hq * Lq).
 *  - The first call on a device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - Every call on a device shares the one array.  Each call rewrites all of
 *    it that it reads (D and the zeroed dQ accumulator), but calls whose work
 *    overlaps on the GPU (different streams, or different host threads
 *    without ordering) race on it and give wrong results.
 */
ATTN_API int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk,
                              int d, float scale, int causal, int window, void* stream);

/*
 * Building blocks of ring (context-parallel) attention ("缩放定律与高效注意力"
 * §5.1, the table of three directions: for longer contexts, RingAttention
 * and LongFlashAttention run sequence parallelism on top of FlashAttention).
 * The sequence is cut into blocks held by different devices; each device
 * computes its queries against one K/V block at a time while the blocks are
 * passed around a ring, and the partial results are merged exactly with the
 * online-softmax rescale of "高效注意力：FlashAttention 与线性注意力", 原理与
 * 机制 (running max / sum, rescaled by e^{m_old - m_new}), applied to whole
 * key blocks through their logsumexp.  The exchange itself is the caller's
 * (the Python package drives it over torch.distributed); these calls are the
 * per-block compute.
 *
 * attn_fwd_accumulate: attention of q against the key block k, v (masks as
 * attn_fwd, relative to the two blocks' own row indices: causal = 1 is the
 * diagonal block of equal-length blocks, causal = 0 a block that lies wholly
 * before the queries), merged into running accumulators:
 *  o_acc    fp32 [B, Hq, Lq, d]  in/out: O over the key blocks so far,
 *                                normalised by its own softmax sum
 *  lse_acc  fp32 [B, Hq, Lq]     in/out: their natural-log logsumexp
 *                                (-inf: no visible key yet)
 *  init     1: the accumulators are written, not read (first block of these
 *           rows); 0: merged: with M = max(LSE_a, LSE_b), w = exp(LSE - M),
 *           O = (w_a O_a + w_b O_b) / (w_a + w_b), LSE = M + log(w_a + w_b).
 * Other arguments, layouts and errors as attn_fwd.  Calls on the same
 * accumulators must be ordered (one stream).
 *
 * attn_fwd_accumulate_finalize: o = bf16(o_acc) (round to nearest even),
 * lse = lse_acc; o bf16 [B, Hq, Lq, d], lse fp32 [B, Hq, Lq].
 *
 * attn_bwd_accumulate: the backward of one key block with the FINAL (merged)
 * lse of the queries and the workspace of attn_bwd_preprocess (D from the
 * final O, and the fp32 dQ accumulator, to which this block's dQ is added;
 * attn_bwd_finalize turns it into dQ after the last block).  This block's
 * dK (scaled) and dV are added into fp32 accumulators dk_acc, dv_acc
 * [B, Hkv, Lk, d] (init = 1: stored instead of added).  Other arguments as
 * attn_bwd_main.
 *
 * attn_accumulator_to_bf16: out[i] = bf16(acc[i]) for n elements (dK / dV
 * accumulators after the last block).  16-byte aligned pointers.
 */
ATTN_API int attn_fwd_accumulate(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, int B,
                                 int Hq, int Hkv, int Lq, int Lk, int d, float scale, int causal, int window, int init,
                                 void* stream);
ATTN_API int attn_fwd_accumulate_finalize(const float* o_acc, const float* lse_acc, void* o, float* lse, int B, int Hq,
                                          int Lq, int d, void* stream);
ATTN_API int attn_bwd_accumulate(const void* q, const void* k, const void* v, const float* lse, const void* dO,
                                 float* dk_acc, float* dv_acc, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                                 float scale, int causal, int window, int init, void* workspace,
                                 size_t workspace_bytes, void* stream);
ATTN_API int attn_accumulator_to_bf16(const float* acc, void* out, size_t n, void* stream);

/*
 * The attention step with HOST buffers: copies Q, K, V (and dO) in, runs
 * attn_fwd (and attn_bwd), and copies O and LSE (and dQ, dK, dV) out, all
 * ordered on `stream` like every other call (asynchronous; synchronise the
 * stream before reading the host outputs).  The computation is that of
 * attn_fwd / attn_bwd (the scaled-dot-product attention call of
 * "缩放定律与高效注意力" §3.5, and its recompute backward of §3.3); the pages
 * call it on tensors already on the device, this entry point serves a caller
 * whose data lives in host memory.
 *
 *  - q, k, v, dO, o, lse, dq, dk, dv: HOST pointers, same shapes and layouts
 *    as attn_fwd / attn_bwd.  Page-locked (pinned) host memory lets the copies
 *    run concurrently with the kernels; pageable memory gives the same
 *    results with the copies serialised.
 *  - dO == NULL: forward only (dq, dk, dv are ignored and may be NULL).
 *  - dev_buf: caller-owned device memory, 256-byte aligned, at least
 *    attn_step_host_buffer_size(...) bytes (with_backward = dO != NULL); it
 *    stages every tensor and the backward workspace.  The library allocates
 *    no device memory; it creates and releases three streams and a few events
 *    per call.
 *  - The problem is cut into chunks of whole kv-head groups of one sequence
 *    (about eight chunks): chunk c's inputs are copied in on one internal
 *    stream while chunk c-1 computes on a second and chunk c-2's outputs are
 *    copied out on a third.  Results are bit-identical to attn_fwd / attn_bwd
 *    on the whole problem.
 *  - Errors: shape, mask and scale checks as attn_fwd (before anything is
 *    enqueued); NULL host pointers or a short / misaligned dev_buf:
 *    ATTN_ERR_INVALID_ARG; a failing CUDA call: ATTN_ERR_CUDA.  Before an
 *    error is returned after chunks were already queued, the call waits for
 *    that work to finish, so no copy still reads or writes the caller's host
 *    buffers or dev_buf once it has returned; the outputs are then undefined.
 */
ATTN_API size_t attn_step_host_buffer_size(int B, int Hq, int Hkv, int Lq, int Lk, int d, int with_backward);
ATTN_API int attn_step_host(const void* q, const void* k, const void* v, const void* dO, void* o, float* lse,
                            void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                            int causal, int window, void* dev_buf, size_t dev_buf_bytes, void* stream);

/* Static, human-readable name of a status code. */
ATTN_API const char* attn_status_string(int status);

/*
 * Text of the last CUDA error that made a call on this thread return
 * ATTN_ERR_CUDA, prefixed with the failing step ("" if none).  The pointer
 * stays valid until the next call on this thread.
 */
ATTN_API const char* attn_last_cuda_error(void);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns ATTN_OK, ATTN_ERR_TIMEOUT if a kernel gave up a bounded wait
 * since the last call, or ATTN_ERR_CUDA if the synchronisation failed.
 * If `site` is not NULL it receives the internal wait-site id of a timeout.
 */
ATTN_API int attn_get_device_error(void* stream, int* site);

/*
 * Self-test of the bounded-wait mechanism: launches one CTA that waits on a
 * barrier nothing ever completes, with a limit of `limit_ns` nanoseconds.
 * The kernel gives up, records ATTN_ERR_TIMEOUT and exits normally; the
 * caller then sees it through attn_get_device_error().  Returns the launch
 * status.  No counterpart on the pages: it exists to test failure handling.
 */
ATTN_API int attn_selftest_wait_timeout(int64_t limit_ns, void* stream);

/*
 * Self-test of the backward kernel's abort path: attn_bwd (arguments as
 * there) in which the gradient warps withhold their arrival for step
 * `stall_step` of every CTA that has that many steps, so the MMA issuer's
 * bounded wait runs out after `limit_ns` (1 ns .. 10 s).  The CTA then lets
 * every copy, MMA and reduce it started finish, frees its tensor memory and
 * exits; attn_get_device_error() reports ATTN_ERR_TIMEOUT and the outputs are
 * undefined.  Nothing faults or hangs on the GPU, and the context stays
 * usable.  No counterpart on the pages: it exists to test failure handling.
 */
ATTN_API int attn_selftest_bwd_abort(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                     const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq,
                                     int Lk, int d, float scale, int causal, int window, int stall_step,
                                     int64_t limit_ns, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Self-test of attn_step_host's error path: the next attn_step_host call (on
 * any thread) behaves as if the copy in of chunk `chunk` had failed, after
 * the earlier chunks' copies and kernels were queued, and returns
 * ATTN_ERR_CUDA.  chunk = -1 cancels; chunk < -1 is ATTN_ERR_INVALID_ARG.
 * The failure is made on the host; nothing faults on the GPU.  No counterpart
 * on the pages: it exists to test failure handling.
 */
ATTN_API int attn_selftest_step_host_fail_at(int chunk);

#ifdef __cplusplus
}
#endif

#endif /* TILEDATTN_H */

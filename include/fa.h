/*
 * fa.h -- C ABI of libfa.so: exact scaled dot-product attention, computed tile by tile
 * with an online softmax so that the N x N score matrix never reaches device memory.
 *
 * What the calls compute
 *   Forward ("FlashAttention" page, introduction and "The bottleneck is memory, not
 *   multiplication"; "FlashAttention, simplified", "The trick"):
 *       S  = scale * Q K^T            (per batch b and head h, N x N)
 *       S_ij = -inf where causal and j > i   (query i sees keys 0..i)
 *       O  = softmax_rows(S) V
 *       LSE_i = log(sum_j exp(S_ij))  (natural log, of the scaled and masked logits)
 *   The result is the plain definition above; only the order of floating-point
 *   operations differs (tiles of 128 keys, running max and running sum, one final
 *   division).
 *   Backward ("What FlashAttention actually buys", "Why the distinction matters
 *   downstream": the backward recomputes the score tiles instead of storing them):
 *       P = exp(S - LSE), dV = P^T dO, dP = dO V^T, D_i = sum_k dO_ik O_ik,
 *       dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q.
 *
 * Layout and types
 *   Q, K, V, O, dO, dQ, dK, dV: [B, H, N, d] contiguous row-major (d fastest).  bf16 in
 *   the bf16 calls (__nv_bfloat16, passed as void*), float in the _f32 calls.
 *   LSE: [B, H, N] float32.  All pointers are device pointers.  The _qk calls take Nq
 *   query rows and Nk key rows, the _varlen calls padded batches with per-sequence
 *   lengths, the _packed calls [tokens, H, d] tensors delimited by start arrays; each
 *   declaration below gives its shapes.
 *   Arithmetic: bf16 inputs, float32 accumulation and softmax statistics; the bf16 calls
 *   round the probabilities (and dS in the backward) to bf16 before the second matrix
 *   product.  The _f32 calls compute in float32 throughout.
 *
 * Ownership and asynchrony
 *   The caller allocates and owns every buffer.  The library allocates no device memory
 *   and keeps no per-call state; it reads the device's SM count once per device.  (Its
 *   only device data of its own are an error word and the fixed scratch array of
 *   fa_bwd_noalloc, both part of the loaded module.)  Each
 *   call validates its arguments on the host, enqueues kernels on `stream` and returns;
 *   the results are ready when `stream` reaches that point.  A return of FA_OK says the
 *   launch was accepted; errors raised while the kernels run are reported by
 *   fa_check_device_error().
 *
 * Errors
 *   FA_ERR_INVALID_ARG  null or misaligned pointer (16-byte alignment is required),
 *                       negative size, B*H*N too large, non-finite or non-positive
 *                       scale, causal not 0/1, workspace too small, O aliasing an input.
 *   FA_ERR_UNSUPPORTED  head dimension other than 64 or 128.
 *   FA_ERR_CUDA         a CUDA runtime call failed (launch error, no device, ...).
 *   FA_ERR_TIMEOUT      a kernel gave up waiting on one of its own pipeline barriers
 *                       (reported by fa_check_device_error; the outputs are invalid).
 *   On any error the outputs are unspecified.  fa_last_error_message() gives detail for
 *   the calling thread's most recent failed call.
 *
 * N == 0 (or B*H == 0) is valid and does nothing; the pointers are then not checked
 * (empty tensors may have NULL data pointers).  The one exception is a backward call
 * with keys but no queries, which writes zero key gradients (see fa_bwd_qk).
 * Lengths above 2^31 - 256 rows are rejected.
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4
} fa_status;

/* Version of this ABI; bumped when a signature changes. */
FA_API int fa_abi_version(void);

/*
 * Forward pass, bf16 in and out ("FlashAttention, simplified", "The trick").
 *   Q, K, V  in : [B,H,N,d] bf16
 *   O        out: [B,H,N,d] bf16; must not overlap Q, K or V
 *   LSE      out: [B,H,N] float32 natural-log log-sum-exp per query row; may be NULL
 *   d in {64, 128}; scale > 0 and finite (usually 1/sqrt(d)); causal in {0, 1}
 * Kernel: persistent, one CTA per SM, tensor cores (tcgen05) with TMEM accumulators.
 */
FA_API fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE,
                 int B, int H, int N, int d, float scale, int causal, cudaStream_t stream);

/*
 * Forward pass with Nq queries and Nk keys per head (no counterpart on the pages, which
 * treat attention over N tokens; the reading used here: the queries are the last Nq of
 * the Nk tokens, e.g. a chunk of new tokens whose keys follow earlier ones).
 *   Q        in : [B,H,Nq,d] bf16
 *   K, V     in : [B,H,Nk,d] bf16
 *   O        out: [B,H,Nq,d] bf16; must not overlap Q, K or V
 *   LSE      out: [B,H,Nq] float32; may be NULL
 *   causal: query i sees keys j <= i + Nk - Nq (bottom-right alignment) and then needs
 *   Nq <= Nk (FA_ERR_INVALID_ARG otherwise); non-causal takes any Nq, Nk >= 1.
 *   fa_fwd(..., N, ...) is fa_fwd_qk(..., N, N, ...).  Same kernel, errors and
 *   asynchrony as fa_fwd.
 */
FA_API fa_status fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, float* LSE,
                           int B, int H, int Nq, int Nk, int d, float scale, int causal,
                           cudaStream_t stream);

/*
 * Forward pass over a padded batch of sequences of different lengths (no counterpart on
 * the pages; the queries of each sequence are aligned with the end of its keys as in
 * fa_fwd_qk).  Tensors are padded to common lengths:
 *   Q, O [B,H,Nq,d] bf16;  K, V [B,H,Nk,d] bf16;  LSE [B,H,Nq] float32 or NULL
 *   seqlens_q, seqlens_k: device int32 arrays [B], 4-byte aligned, required; sequence b
 *     uses its first seqlens_q[b] query rows and seqlens_k[b] key rows
 *     (0 <= seqlens_q[b] <= Nq, 0 <= seqlens_k[b] <= Nk, and causal needs
 *     seqlens_q[b] <= seqlens_k[b]).
 * Rows past a sequence's query length (in O and LSE) are not written.  A sequence with no
 * queries or no keys is skipped.  Padding rows of K and V must hold finite values (their
 * probabilities are zero, and 0 times a NaN is a NaN).  The lengths are read on the
 * device: one out of range makes the kernel skip that sequence and makes
 * fa_check_device_error report FA_ERR_INVALID_ARG.  Otherwise as fa_fwd_qk.
 */
FA_API fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, void* O,
                               float* LSE, const int* seqlens_q, const int* seqlens_k, int B,
                               int H, int Nq, int Nk, int d, float scale, int causal,
                               cudaStream_t stream);

/*
 * Forward pass over a packed batch of sequences of different lengths (no counterpart on
 * the pages; queries aligned with the end of their sequence's keys as in fa_fwd_qk).
 * The tokens of all sequences are stored one after another, with no padding:
 *   Q, O [total_q, H, d] bf16;  K, V [total_k, H, d] bf16;  LSE [H, total_q] float32
 *     or NULL
 *   cu_seqlens_q, cu_seqlens_k: device int32 arrays [B+1], 4-byte aligned, required;
 *     sequence b has queries cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and keys
 *     cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 (non-decreasing, ending at total_q and
 *     total_k)
 *   max_seqlen_q, max_seqlen_k: at least the longest sequence's query and key counts
 *     (they size the work grid); causal needs max_seqlen_q <= max_seqlen_k and each
 *     sequence's queries <= its keys.
 * A sequence with no queries or no keys is skipped (its rows are not written).  The
 * start arrays are read on the device: a sequence out of range is skipped and reported
 * by fa_check_device_error as FA_ERR_INVALID_ARG.  Otherwise as fa_fwd_qk.
 */
FA_API fa_status fa_fwd_packed(const void* Q, const void* K, const void* V, void* O,
                               float* LSE, const int* cu_seqlens_q, const int* cu_seqlens_k,
                               int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q,
                               int total_k, int d, float scale, int causal,
                               cudaStream_t stream);

/*
 * Forward pass with float32 inputs and outputs, computed in float32 on the CUDA cores
 * (same definition and arguments as fa_fwd).
 */
FA_API fa_status fa_fwd_f32(const float* Q, const float* K, const float* V, float* O, float* LSE,
                     int B, int H, int N, int d, float scale, int causal,
                     cudaStream_t stream);

/*
 * The float32 forward with Nq queries and Nk keys per head, over a padded batch, and
 * over a packed batch: the same definitions, arguments, layouts, length rules and
 * errors as fa_fwd_qk, fa_fwd_varlen and fa_fwd_packed, with float32 tensors (Q, K, V,
 * O) and float32 arithmetic on the CUDA cores.  Any sm_100 device.
 */
FA_API fa_status fa_fwd_f32_qk(const float* Q, const float* K, const float* V, float* O,
                               float* LSE, int B, int H, int Nq, int Nk, int d, float scale,
                               int causal, cudaStream_t stream);
FA_API fa_status fa_fwd_f32_varlen(const float* Q, const float* K, const float* V, float* O,
                                   float* LSE, const int* seqlens_q, const int* seqlens_k,
                                   int B, int H, int Nq, int Nk, int d, float scale,
                                   int causal, cudaStream_t stream);
FA_API fa_status fa_fwd_f32_packed(const float* Q, const float* K, const float* V, float* O,
                                   float* LSE, const int* cu_seqlens_q,
                                   const int* cu_seqlens_k, int B, int H, int max_seqlen_q,
                                   int max_seqlen_k, int total_q, int total_k, int d,
                                   float scale, int causal, cudaStream_t stream);

/*
 * Bytes of scratch that fa_bwd (and fa_bwd_f32) needs for given sizes: two float32 per query row
 * (D_i = sum_k dO_ik O_ik and LSE_i * log2(e)), rows padded to a multiple of 128,
 * rounded up to 256 bytes: 8 * B * H * ceil(N/128) * 128.  Grows as B*H*N, never as N^2.
 */
FA_API size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass, bf16 ("What FlashAttention actually buys", "Why the distinction
 * matters downstream": the score tiles are recomputed from Q, K and the saved LSE).
 *   Q, K, V, O, dO in : [B,H,N,d] bf16 (O is the forward output)
 *   LSE            in : [B,H,N] float32 from fa_fwd with the same scale and causal
 *   dQ, dK, dV     out: [B,H,N,d] bf16; must not overlap the inputs
 *   workspace         : caller-owned device scratch of at least
 *                       fa_bwd_workspace_bytes(B,H,N,d) bytes, 16-byte aligned; its
 *                       contents on entry do not matter and are overwritten
 * Three kernels on `stream`: D = rowsum(dO * O); dK and dV per key block; dQ per query
 * block.  No atomics: the result is the same bits on every run.
 */
FA_API fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O,
                 const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                 int B, int H, int N, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward pass with Nq queries and Nk keys per head, the gradient of fa_fwd_qk.
 *   Q, O, dO in : [B,H,Nq,d] bf16;   K, V in : [B,H,Nk,d] bf16
 *   LSE      in : [B,H,Nq] float32 from fa_fwd_qk with the same scale and causal
 *   dQ       out: [B,H,Nq,d] bf16;   dK, dV out: [B,H,Nk,d] bf16
 *   workspace   : fa_bwd_workspace_bytes(B,H,Nq,d) bytes (two floats per query row)
 * Same kernels, rules and errors as fa_bwd (causal needs Nq <= Nk).  With Nq == 0 and
 * Nk > 0 no query sees any key: dK and dV are set to zero (dK and dV must then be valid,
 * 16-byte aligned and not overlap; the other pointers are not used and may be NULL).
 */
FA_API fa_status fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O,
                           const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                           int B, int H, int Nq, int Nk, int d, float scale, int causal,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward pass over a padded batch (the gradient of fa_fwd_varlen, same lengths).
 *   Q, O, dO, dQ [B,H,Nq,d] bf16;  K, V, dK, dV [B,H,Nk,d] bf16;  LSE [B,H,Nq] float32
 *   workspace: fa_bwd_workspace_bytes(B,H,Nq,d) bytes
 * Rows past a sequence's lengths (dQ past seqlens_q[b], dK and dV past seqlens_k[b]) are
 * not written.  A sequence with keys but no queries (seqlens_q[b] == 0) gets zeros in its
 * dK and dV rows below seqlens_k[b] (no query sees those keys), also when Nq == 0 (then
 * only dK, dV and the length arrays are used).  A sequence with queries but no keys is
 * skipped.  Padding rows of Q, K, V, O and dO must hold finite values.  Lengths as for
 * fa_fwd_varlen; otherwise as fa_bwd_qk.
 */
FA_API fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* LSE, void* dQ, void* dK,
                               void* dV, const int* seqlens_q, const int* seqlens_k, int B,
                               int H, int Nq, int Nk, int d, float scale, int causal,
                               void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Backward pass over a packed batch (the gradient of fa_fwd_packed, same start arrays).
 *   Q, O, dO, dQ [total_q, H, d] bf16;  K, V, dK, dV [total_k, H, d] bf16;
 *   LSE [H, total_q] float32
 *   workspace: fa_bwd_workspace_bytes(B, H, max_seqlen_q, d) bytes
 * A sequence with keys but no queries gets zeros in its dK and dV rows, also when the
 * call has no query tokens at all (total_q == 0 or max_seqlen_q == 0; then only dK, dV
 * and the start arrays are used).  Otherwise as fa_bwd_varlen.
 */
FA_API fa_status fa_bwd_packed(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* LSE, void* dQ, void* dK,
                               void* dV, const int* cu_seqlens_q, const int* cu_seqlens_k,
                               int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q,
                               int total_k, int d, float scale, int causal, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward pass, float32: the same computation as fa_bwd with float32 inputs, outputs
 * and arithmetic (on the CUDA cores; no tensor cores, no bf16 rounding of P or dS).
 *   Q, K, V, O, dO in : [B,H,N,d] float32
 *   LSE            in : [B,H,N] float32 from fa_fwd_f32 with the same scale and causal
 *   dQ, dK, dV     out: [B,H,N,d] float32; must not overlap the inputs or each other
 *   workspace         : as for fa_bwd (fa_bwd_workspace_bytes(B,H,N,d) bytes, 16-byte
 *                       aligned); the first 4*B*H*N bytes receive D
 * Three kernels on `stream` (D; dK and dV per 32 key rows; dQ per 32 query rows), no
 * atomics.  Errors as for fa_bwd; any sm_100 device.
 */
FA_API fa_status fa_bwd_f32(const float* Q, const float* K, const float* V, const float* O,
                            const float* dO, const float* LSE, float* dQ, float* dK,
                            float* dV, int B, int H, int N, int d, float scale, int causal,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * The float32 backward with Nq queries and Nk keys per head, over a padded batch, and
 * over a packed batch: the gradients of fa_fwd_f32_qk, fa_fwd_f32_varlen and
 * fa_fwd_f32_packed, with the arguments, layouts, workspace sizes and rules of
 * fa_bwd_qk, fa_bwd_varlen and fa_bwd_packed and float32 tensors.  D goes to the first
 * 4*B*H*Nq (packed: 4*B*H*max_seqlen_q) bytes of the workspace.  Rows past a sequence's
 * lengths are not written; keys without queries get zero gradients, as in the bf16
 * calls.  Otherwise as fa_bwd_f32.
 */
FA_API fa_status fa_bwd_f32_qk(const float* Q, const float* K, const float* V, const float* O,
                               const float* dO, const float* LSE, float* dQ, float* dK,
                               float* dV, int B, int H, int Nq, int Nk, int d, float scale,
                               int causal, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);
FA_API fa_status fa_bwd_f32_varlen(const float* Q, const float* K, const float* V,
                                   const float* O, const float* dO, const float* LSE,
                                   float* dQ, float* dK, float* dV, const int* seqlens_q,
                                   const int* seqlens_k, int B, int H, int Nq, int Nk, int d,
                                   float scale, int causal, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream);
FA_API fa_status fa_bwd_f32_packed(const float* Q, const float* K, const float* V,
                                   const float* O, const float* dO, const float* LSE,
                                   float* dQ, float* dK, float* dV, const int* cu_seqlens_q,
                                   const int* cu_seqlens_k, int B, int H, int max_seqlen_q,
                                   int max_seqlen_k, int total_q, int total_k, int d,
                                   float scale, int causal, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/*
 * Merge a partial attention result into an accumulator ("FlashAttention, simplified",
 * "The trick": the rescale-and-add step of the online softmax, applied to two results
 * over disjoint key sets, as context-parallel attention needs when each GPU holds a
 * block of the keys).  With m = max(LSE_acc, LSE_part) and w = exp(LSE - m):
 *   O_acc <- (w_acc O_acc + w_part O_part) / (w_acc + w_part)
 *   LSE_acc <- m + log(w_acc + w_part)
 *   O_acc    in/out: [B,H,N,d] float32 (rows whose LSE_acc is -inf are empty; their
 *                    values are ignored)
 *   LSE_acc  in/out: [B,H,N] float32 natural-log normalisers (-inf: no keys yet)
 *   O_part   in    : [B,H,N,d] bf16, e.g. fa_fwd / fa_fwd_qk over one key block
 *   LSE_part in    : [B,H,N] float32 from the same call (-inf: an empty block)
 *   O_out    out   : [B,H,N,d] bf16, the merged O rounded once; may be NULL
 * A row empty on both sides stays empty (O 0, LSE -inf).  Pointers 16-byte aligned (LSE
 * arrays 4-byte); the accumulator must not overlap the partial result.  One kernel on
 * `stream`, one warp per row.
 */
FA_API fa_status fa_merge(float* O_acc, float* LSE_acc, const void* O_part,
                          const float* LSE_part, void* O_out, int B, int H, int N, int d,
                          cudaStream_t stream);

/*
 * Accumulate a bf16 partial result into float32: acc[i] += part[i] for i < n, and
 * out[i] = bf16(acc[i]) when out is not NULL.  The context-parallel backward sums the
 * gradient contributions of several key blocks with it (each block's dQ on the query's
 * GPU, each block's dK and dV as the block travels around the ring).
 *   acc  in/out: n float32;  part in: n bf16;  out: n bf16 or NULL
 * n a multiple of 8; pointers 16-byte aligned and not overlapping; one kernel on
 * `stream`.  n == 0 is a no-op.
 */
FA_API fa_status fa_accumulate(float* acc, const void* part, void* out, size_t n,
                               cudaStream_t stream);

/*
 * fa_bwd for callers that cannot allocate device memory (no counterpart on the pages:
 * it is a property of this library, not of the method).  Same arguments and result as
 * fa_bwd, without the workspace: the scratch is a fixed array inside the library,
 * fa_bwd_noalloc_max_scratch_bytes() bytes (8 MiB) of device memory that every GPU which
 * loads the library keeps until the process exits.
 *   Who needs it: a caller with no allocator to draw on (a plugin host that passes only
 *   tensors), code inside a framework step whose memory plan is fixed, or a loop that
 *   must not enter cudaMalloc because it can synchronise the device.
 *   Limit: fa_bwd_workspace_bytes(B,H,N,d) must not exceed that size, i.e.
 *   B*H*ceil(N/128)*128 <= 2^20 rows; larger problems get FA_ERR_INVALID_ARG.
 *   Set-up: the first call on a device looks up the array's device address and caches
 *   it (no allocation); make that first call before any stream capture.
 *   Sharing: all calls use the same array.  Each call rewrites what it reads, so no
 *   clearing is needed, but calls whose kernels overlap on the GPU race on the array:
 *   serialise them (one stream, or synchronise between streams and threads).
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
FA_API fa_status fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                                const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                                int B, int H, int N, int d, float scale, int causal,
                                cudaStream_t stream);

/* Size of the fixed scratch array behind fa_bwd_noalloc, in bytes. */
FA_API size_t fa_bwd_noalloc_max_scratch_bytes(void);

/*
 * Kernel-boundary timing, for profilers.  While a list of events is set on the calling
 * thread, every forward and backward call records events[0] on its stream just before
 * its first kernel and events[k] just after its k-th kernel; the forward calls launch
 * one kernel, the backward calls three (D preparation, dK/dV, dQ).  Boundaries
 * beyond n - 1 are not recorded.  The events are caller-created cudaEvent_t (timing
 * enabled) and stay caller-owned.  fa_trace_events(NULL, 0) stops recording.
 * Returns FA_ERR_INVALID_ARG if n < 0, n > 8, or events is NULL with n > 0.
 */
FA_API fa_status fa_trace_events(cudaEvent_t* events, int n);

/* Static text for a status code ("FA_OK", ...). */
FA_API const char* fa_status_string(fa_status status);

/* Detail of the calling thread's last failed call (empty string if none). */
FA_API const char* fa_last_error_message(void);

/*
 * Check of the failure path (no counterpart on the pages): launches one warp that waits
 * on an mbarrier nothing arrives on, in the same bounded loop as the kernels' pipeline
 * waits but giving up after limit_cycles SM cycles (0 .. 2^34; e.g. 2e7, about 10 ms).
 * It then sets the timeout bit of the library's error word and returns, so the next
 * fa_check_device_error reports FA_ERR_TIMEOUT and clears it; the CUDA context stays
 * usable.  Asynchronous on `stream`.
 */
FA_API fa_status fa_selftest_timeout(long long limit_cycles, cudaStream_t stream);

/*
 * Synchronises `stream`, then reports and clears the device-side error word that the
 * kernels set when a pipeline wait exceeds its time limit (FA_ERR_TIMEOUT) or when a
 * kernel finds its shared memory misaligned and skips its work (FA_ERR_CUDA), or
 * FA_ERR_CUDA if the stream itself reports an error.
 */
FA_API fa_status fa_check_device_error(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */

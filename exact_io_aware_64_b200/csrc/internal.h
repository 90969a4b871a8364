// internal.h -- launch interfaces shared between the API layer (fa_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>
#include <cstddef>

namespace fa {

// Problem shared by every kernel: [B*H, N, d] query-side tensors (Q, O, dO, dQ, LSE)
// and [B*H, Nk, d] key-side tensors (K, V, dK, dV), contiguous.  Nk == N except for
// the Nq != Nk entry points, whose queries are the last N of the Nk tokens.
struct Problem {
  int BH;
  int N;
  int Nk;
  int d;
  float scale;
  int causal;
  unsigned int* err;  // device address of the library's error word
  // padded batches: per-sequence lengths [B] on the device (both null otherwise); H
  // heads per sequence, so head bh belongs to sequence bh / H
  const int* seqlens_q;
  const int* seqlens_k;
  int H;
  // packed layout ([tokens, H, d] tensors, LSE [H, tokens]): per-sequence start tokens
  // [B+1] on the device (both null otherwise) and the token totals; N and Nk are then
  // the longest sequence's query and key counts
  const int* cu_q;
  const int* cu_k;
  int total_q;
  int total_k;
  // optional kernel-boundary events (fa_trace_events): trace[0] before the first kernel,
  // trace[k] after the k-th; n_trace entries
  cudaEvent_t* trace;
  int n_trace;
};

// Record trace event k of `p` on `stream` if the caller asked for it.
inline cudaError_t trace_mark(const Problem& p, int k, cudaStream_t stream) {
  if (p.trace == nullptr || k >= p.n_trace) return cudaSuccess;
  return cudaEventRecord(p.trace[k], stream);
}

// Forward, bf16, tcgen05.  Tensor maps describe Q, K, V and O as 3-D [BH][N][d] bf16
// (or packed [tokens][H][d]) with the 128-byte swizzle, boxes of 64 x 128 x 1 for Q, K
// and V and 64 x 32 x 1 for O, which is written through it (bulk tensor stores of 32
// valid rows at a time) and row by row where a warp's rows are ragged.
cudaError_t launch_fwd_sm100(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmO, void* O, float* LSE,
                             const Problem& p, int num_sms, cudaStream_t stream);

// Forward, float32 on the CUDA cores.
cudaError_t launch_fwd_f32(const float* Q, const float* K, const float* V, float* O,
                           float* LSE, const Problem& p, cudaStream_t stream);

// Backward, bf16: -D = -rowsum(dO * O) and -L2 = -LSE * log2(e) into the workspace,
// then dK/dV, then dQ.  Workspace layout: -D as [BH][Npad] float, then -L2 as [BH][Npad]
// float, Npad = bwd_padded_rows(N).  tmL2 / tmD describe those two arrays as 3-D
// [1][BH][Npad] float tensors with 128 x 1 x 1 boxes.  tmdK / tmdV describe dK and dV
// like K and V but with 64 x 32 x 1 boxes: the dK/dV kernel writes them through these.
long long bwd_padded_rows(long long N);
cudaError_t launch_bwd_sm100(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmdO,
                             const CUtensorMap& tmL2, const CUtensorMap& tmD,
                             const CUtensorMap& tmdK, const CUtensorMap& tmdV, const void* O,
                             const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                             float* workspace, const Problem& p, int num_sms,
                             cudaStream_t stream);

// Backward, float32 on the CUDA cores: D = rowsum(dO * O) into the workspace as
// [BH][N] float, then dK/dV, then dQ.
cudaError_t launch_bwd_f32(const float* Q, const float* K, const float* V, const float* O,
                           const float* dO, const float* LSE, float* dQ, float* dK, float* dV,
                           float* workspace, const Problem& p, cudaStream_t stream);

// Zeros in rows [0, lk) of dK and dV for every sequence with no queries (lq == 0);
// elem_bytes is 2 (bf16) or 4 (float32).  For calls with keys and no query rows at all,
// where the backward kernels have nothing to run over.
cudaError_t launch_zero_key_rows(void* dK, void* dV, const Problem& p, int elem_bytes,
                                 int num_sms, cudaStream_t stream);

// Merge of a partial attention result (O_part bf16, LSE_part) into a float32 accumulator
// (O_acc, LSE_acc), optionally writing the merged O as bf16 to O_out; [BH][N] rows.
cudaError_t launch_merge(float* O_acc, float* LSE_acc, const void* O_part,
                         const float* LSE_part, void* O_out, const Problem& p,
                         cudaStream_t stream);

// acc[i] += part[i] (float32 += bf16) for n elements, n a multiple of 8; out[i] =
// bf16(acc[i]) when out is not null.
cudaError_t launch_accumulate(float* acc, const void* part, void* out, long long n,
                              const Problem& p, cudaStream_t stream);

// One warp waiting on an mbarrier nothing arrives on, giving up after limit_cycles with
// the kernels' timeout error (a check of the failure path).
cudaError_t launch_timeout_probe(long long limit_cycles, const Problem& p,
                                 cudaStream_t stream);

}  // namespace fa

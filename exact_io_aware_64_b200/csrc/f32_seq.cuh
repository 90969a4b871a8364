// f32_seq.cuh -- one (batch, head)'s sequence as the float32 kernels address it.
//
// The float32 kernels take the same problems as the tensor-core path:
//   dense   Q, O, dO, dQ [BH][Nq][d];  K, V, dK, dV [BH][Nk][d];  LSE [BH][Nq]
//           (Nq != Nk allowed: the queries are the last Nq of the Nk tokens)
//   padded  the same tensors; sequence b = bh / H uses its first seqlens_q[b] query rows
//           and seqlens_k[b] key rows
//   packed  Q, O, dO, dQ [total_q][H][d];  K, V, dK, dV [total_k][H][d];  LSE [H][total_q];
//           sequence b holds tokens cu_q[b] .. cu_q[b+1]-1 (queries) and cu_k[b] ..
//           cu_k[b+1]-1 (keys)
// In every layout query row i of a sequence with lq queries and lk keys sits at token
// position i + lk - lq, so under the causal mask it sees keys j <= i + lk - lq.
#pragma once

#include <cstddef>

#include "internal.h"
#include "sm100.cuh"  // the library's device error bits

namespace fa {

struct F32Seq {
  int lq;       // query rows of this sequence (0: nothing to do)
  int lk;       // key rows
  int off;      // lk - lq: query row i sees keys j <= i + off under the causal mask
  size_t q0;    // element offset of query row 0 in Q, O, dO, dQ
  size_t k0;    // element offset of key row 0 in K, V, dK, dV
  size_t rs;    // elements from one row to the next (d, or H * d when packed)
  size_t lse0;  // index of query row 0 in LSE
  size_t d0;    // index of query row 0 in the [BH][Nq] row statistic D
};

// Head bh's sequence.  Lengths out of range (negative, above Nq / Nk, outside the token
// totals, or more queries than keys under the causal mask) set kErrBadLength in the
// library's error word (when `report`) and give an empty sequence, which every kernel
// skips.
__device__ __forceinline__ F32Seq f32_seq(const Problem& p, int bh, int D, bool report) {
  F32Seq s;
  int lq = p.N, lk = p.Nk, tq = 0, tk = 0;
  bool bad = false;
  const int b = bh / p.H;
  if (p.cu_q != nullptr) {
    tq = p.cu_q[b];
    tk = p.cu_k[b];
    lq = p.cu_q[b + 1] - tq;
    lk = p.cu_k[b + 1] - tk;
    bad = tq < 0 || tk < 0 || lq < 0 || lk < 0 || tq > p.total_q - lq ||
          tk > p.total_k - lk;
  } else if (p.seqlens_q != nullptr) {
    lq = p.seqlens_q[b];
    lk = p.seqlens_k[b];
  }
  if (bad || lq < 0 || lq > p.N || lk < 0 || lk > p.Nk || (p.causal && lq > lk)) {
    if (report) atomicOr(p.err, sm100::kErrBadLength);
    lq = 0;
    lk = 0;
  }
  s.lq = lq;
  s.lk = lk;
  s.off = lk - lq;
  if (p.cu_q != nullptr) {
    const int h = bh % p.H;
    s.q0 = (static_cast<size_t>(tq) * p.H + h) * D;
    s.k0 = (static_cast<size_t>(tk) * p.H + h) * D;
    s.rs = static_cast<size_t>(p.H) * D;
    s.lse0 = static_cast<size_t>(h) * p.total_q + tq;
  } else {
    s.q0 = static_cast<size_t>(bh) * p.N * D;
    s.k0 = static_cast<size_t>(bh) * p.Nk * D;
    s.rs = D;
    s.lse0 = static_cast<size_t>(bh) * p.N;
  }
  s.d0 = static_cast<size_t>(bh) * p.N;
  return s;
}

}  // namespace fa

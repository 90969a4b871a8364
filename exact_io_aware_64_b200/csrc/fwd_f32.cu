// fwd_f32.cu -- forward attention in float32 on the CUDA cores.
//
// Same tiled online softmax as the tensor-core path ("FlashAttention, simplified", "The
// trick"): per query row a running max m, running sum l and accumulator acc; each block
// of 32 keys is scored, the max updated, acc and l rescaled by exp(m - m_new), and O =
// acc / l at the end.  Every step is float32 (no TF32, no bf16 rounding).
//
// Mapping: a CTA of 128 threads owns 32 query rows of one (batch, head); four threads
// share a row, each holding every fourth element of q and acc, and combine their partial
// dot products with two shuffles.  The key and value blocks are staged in shared memory.
// Blocks are numbered flat over (head, row block), so B*H is not limited by the grid's y
// extent.  Each head's sequence (its lengths, the causal offset and where its rows live
// in the dense, padded or packed layout) comes from f32_seq.
#include <cmath>
#include <cstdint>

#include "f32_seq.cuh"
#include "internal.h"

namespace fa {
namespace {

constexpr int kRows = 32;     // query rows per CTA
constexpr int kKeys = 32;     // keys per shared-memory block
constexpr int kThreads = 128; // 4 threads per row

template <int D>
__global__ void __launch_bounds__(kThreads)
    fwd_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                   const float* __restrict__ V, float* __restrict__ O,
                   float* __restrict__ LSE, const Problem p, int tiles) {
  constexpr int E = D / 4;  // elements of q / acc per thread
  __shared__ float Ks[kKeys][D];
  __shared__ float Vs[kKeys][D];

  const int bh = blockIdx.x / tiles;
  const int tile = blockIdx.x % tiles;
  const F32Seq sq = f32_seq(p, bh, D, threadIdx.x == 0);
  // a whole CTA past its sequence's queries, or a sequence with no keys: nothing to do
  if (tile * kRows >= sq.lq || sq.lk == 0) return;
  const int r = threadIdx.x / 4;  // row within the CTA
  const int part = threadIdx.x % 4;
  const int row = tile * kRows + r;
  const bool valid = row < sq.lq;
  const float* qrow = Q + sq.q0 + static_cast<size_t>(row) * sq.rs;

  float q[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = valid ? qrow[4 * e + part] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const int last_row = min(sq.lq - 1, (tile + 1) * kRows - 1);
  const int key_end = p.causal ? min(sq.lk, last_row + sq.off + 1) : sq.lk;
  for (int k0 = 0; k0 < key_end; k0 += kKeys) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeys * D; i += kThreads) {
      const int kr = i / D, c = i % D;
      const int key = k0 + kr;
      const bool in = key < sq.lk;
      const size_t at = sq.k0 + static_cast<size_t>(key) * sq.rs + c;
      Ks[kr][c] = in ? K[at] : 0.f;
      Vs[kr][c] = in ? V[at] : 0.f;
    }
    __syncthreads();
    float s[kKeys];
    float tile_max = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float part_dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) part_dot = fmaf(q[e], Ks[j][4 * e + part], part_dot);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 1);
      part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 2);
      const int key = k0 + j;
      const bool visible = key < sq.lk && (!p.causal || key <= row + sq.off);
      s[j] = visible ? part_dot * p.scale : -INFINITY;
      tile_max = fmaxf(tile_max, s[j]);
    }
    const float m_new = fmaxf(m, tile_max);
    if (m_new == -INFINITY) continue;  // nothing visible yet for this row
    const float alpha = expf(m - m_new);
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      s[j] = expf(s[j] - m_new);
      psum += s[j];
    }
    l = alpha * l + psum;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float a = alpha * acc[e];
#pragma unroll
      for (int j = 0; j < kKeys; ++j) a = fmaf(s[j], Vs[j][4 * e + part], a);
      acc[e] = a;
    }
    m = m_new;
  }
  if (!valid) return;
  const float inv_l = 1.f / l;
  float* orow = O + sq.q0 + static_cast<size_t>(row) * sq.rs;
#pragma unroll
  for (int e = 0; e < E; ++e) orow[4 * e + part] = acc[e] * inv_l;
  if (LSE != nullptr && part == 0) LSE[sq.lse0 + row] = m + logf(l);
}

template <int D>
cudaError_t launch_d(const float* Q, const float* K, const float* V, float* O, float* LSE,
                     const Problem& p, cudaStream_t stream) {
  const int tiles = (p.N + kRows - 1) / kRows;
  const unsigned grid = static_cast<unsigned>(tiles) * static_cast<unsigned>(p.BH);
  cudaError_t e = trace_mark(p, 0, stream);
  if (e != cudaSuccess) return e;
  fwd_f32_kernel<D><<<grid, kThreads, 0, stream>>>(Q, K, V, O, LSE, p, tiles);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_mark(p, 1, stream);
}

}  // namespace

cudaError_t launch_fwd_f32(const float* Q, const float* K, const float* V, float* O,
                           float* LSE, const Problem& p, cudaStream_t stream) {
  if (p.d == 64) return launch_d<64>(Q, K, V, O, LSE, p, stream);
  return launch_d<128>(Q, K, V, O, LSE, p, stream);
}

}  // namespace fa

// bwd_f32.cu -- backward attention in float32 on the CUDA cores.
//
// The gradient of softmax attention, recomputing every score from Q, K and the saved
// per-row log-sum-exp instead of reading a stored probability matrix ("What
// FlashAttention actually buys", "Why the distinction matters downstream"):
//   p_ij = exp(scale * q_i . k_j - LSE_i)      (0 where the causal mask hides j)
//   D_i  = sum_k dO_ik O_ik
//   dV_j = sum_i p_ij dO_i
//   dS_ij = p_ij (dO_i . v_j - D_i)
//   dK_j = scale * sum_i dS_ij q_i,   dQ_i = scale * sum_j dS_ij k_j
// Every step is float32.  Three kernels: D per row, then dK/dV per block of key rows
// (queries streamed through shared memory), then dQ per block of query rows (keys and
// values streamed).  No atomics: each output row is summed by one thread group in a
// fixed order, so the result is the same on every run.
//
// Mapping: a CTA owns 32 rows of one (batch, head); kTpr threads share a row, each
// holding every kTpr-th element (16 per thread at both head sizes) and combining partial
// dot products with shuffles.  Blocks are numbered flat over (head, row block), so B*H is
// not limited by the grid's y extent.  Each head's sequence (its lengths, the causal
// offset and where its rows live in the dense, padded or packed layout) comes from
// f32_seq; rows past a sequence's lengths are neither read nor written.
#include <cmath>
#include <cstdint>

#include "f32_seq.cuh"
#include "internal.h"

namespace fa {
namespace {

constexpr int kRows = 32;   // rows owned by a CTA, and rows per streamed block
constexpr int kChunk = 4;   // streamed rows scored together before accumulating

template <int D>
struct F32Shape {
  static constexpr int kTpr = D / 16;            // threads per row: 4 (d=64) or 8 (d=128)
  static constexpr int kE = D / kTpr;            // elements per thread: 16
  static constexpr int kThreads = kRows * kTpr;  // 128 or 256
};

template <int TPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Copy rows r0 .. r0+31 of one sequence (rows `rs` elements apart from `src`, zeros from
// row n on) into shared memory, 16 bytes per load.
template <int D, int THREADS>
__device__ __forceinline__ void stage_rows(float (*dst)[D], const float* __restrict__ src,
                                           size_t rs, int r0, int n) {
  constexpr int kVec = D / 4;  // float4 per row
#pragma unroll
  for (int i = threadIdx.x; i < kRows * kVec; i += THREADS) {
    const int rr = i / kVec, c = (i % kVec) * 4;
    const int row = r0 + rr;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < n) x = *reinterpret_cast<const float4*>(src + static_cast<size_t>(row) * rs + c);
    *reinterpret_cast<float4*>(&dst[rr][c]) = x;
  }
}

// D_i = sum_k dO_ik O_ik, one warp per row of the [BH][Nq] row grid; stored at the same
// index of the workspace.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_f32_prep_kernel(const float* __restrict__ O, const float* __restrict__ dO,
                        float* __restrict__ Dout, const Problem p) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= static_cast<long long>(p.BH) * p.N) return;
  const int bh = static_cast<int>(row / p.N);
  const int r = static_cast<int>(row % p.N);
  const F32Seq sq = f32_seq(p, bh, D, lane == 0);
  if (r >= sq.lq) return;
  const float* o = O + sq.q0 + static_cast<size_t>(r) * sq.rs;
  const float* g = dO + sq.q0 + static_cast<size_t>(r) * sq.rs;
  float acc = 0.f;
#pragma unroll
  for (int c = lane; c < D; c += 32) acc = fmaf(o[c], g[c], acc);
  acc = row_sum<32>(acc);
  if (lane == 0) Dout[sq.d0 + r] = acc;
}

// dK, dV for 32 key rows; query rows stream through shared memory.
template <int D>
__global__ void __launch_bounds__(F32Shape<D>::kThreads)
    bwd_f32_dkdv_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                        const float* __restrict__ V, const float* __restrict__ dO,
                        const float* __restrict__ LSE, const float* __restrict__ Drow,
                        float* __restrict__ dK, float* __restrict__ dV, const Problem p,
                        int tiles) {
  using S = F32Shape<D>;
  constexpr int TPR = S::kTpr, E = S::kE;
  __shared__ __align__(16) float Qs[kRows][D];
  __shared__ __align__(16) float dOs[kRows][D];
  __shared__ float Ls[kRows];
  __shared__ float Ds[kRows];

  const int bh = blockIdx.x / tiles;
  const int tile = blockIdx.x % tiles;
  const F32Seq sq = f32_seq(p, bh, D, threadIdx.x == 0);
  if (tile * kRows >= sq.lk) return;  // past the sequence's keys
  const int r = threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const int key = tile * kRows + r;
  const bool valid = key < sq.lk;
  if (sq.lq == 0) {
    // keys without queries: no query sees them, so their gradients are exactly zero
    if (valid)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const size_t at = sq.k0 + static_cast<size_t>(key) * sq.rs + TPR * e + part;
        dK[at] = 0.f;
        dV[at] = 0.f;
      }
    return;
  }

  float k[E], v[E], dk[E], dv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const size_t at = sq.k0 + static_cast<size_t>(key) * sq.rs + TPR * e + part;
    k[e] = valid ? K[at] : 0.f;
    v[e] = valid ? V[at] : 0.f;
    dk[e] = 0.f;
    dv[e] = 0.f;
  }

  // causal: query q sees key j when j <= q + off, so queries before this block's first
  // key minus off see none of its keys
  const int q_begin = p.causal ? max(0, tile * kRows - sq.off) : 0;
  for (int q0 = q_begin; q0 < sq.lq; q0 += kRows) {
    __syncthreads();
    stage_rows<D, S::kThreads>(Qs, Q + sq.q0, sq.rs, q0, sq.lq);
    stage_rows<D, S::kThreads>(dOs, dO + sq.q0, sq.rs, q0, sq.lq);
    if (threadIdx.x < kRows) {
      const int q = q0 + threadIdx.x;
      Ls[threadIdx.x] = q < sq.lq ? LSE[sq.lse0 + q] : 0.f;
      Ds[threadIdx.x] = q < sq.lq ? Drow[sq.d0 + q] : 0.f;
    }
    __syncthreads();
    // queries in chunks of kChunk: scores and dS first, then the two accumulations
#pragma unroll 1
    for (int j0 = 0; j0 < kRows; j0 += kChunk) {
      float pr[kChunk], ds[kChunk];
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj) {
        const int j = j0 + jj;
        float s_part = 0.f, dp_part = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s_part = fmaf(k[e], Qs[j][TPR * e + part], s_part);
          dp_part = fmaf(v[e], dOs[j][TPR * e + part], dp_part);
        }
        const float s = row_sum<TPR>(s_part);
        const float dp = row_sum<TPR>(dp_part);
        const int q = q0 + j;
        const bool visible = valid && q < sq.lq && (!p.causal || key <= q + sq.off);
        pr[jj] = visible ? expf(s * p.scale - Ls[j]) : 0.f;
        ds[jj] = pr[jj] * (dp - Ds[j]);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float a = dv[e], b = dk[e];
#pragma unroll
        for (int jj = 0; jj < kChunk; ++jj) {
          a = fmaf(pr[jj], dOs[j0 + jj][TPR * e + part], a);
          b = fmaf(ds[jj], Qs[j0 + jj][TPR * e + part], b);
        }
        dv[e] = a;
        dk[e] = b;
      }
    }
  }
  if (!valid) return;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const size_t at = sq.k0 + static_cast<size_t>(key) * sq.rs + TPR * e + part;
    dK[at] = dk[e] * p.scale;
    dV[at] = dv[e];
  }
}

// dQ for 32 query rows; key and value rows stream through shared memory.
template <int D>
__global__ void __launch_bounds__(F32Shape<D>::kThreads)
    bwd_f32_dq_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                      const float* __restrict__ V, const float* __restrict__ dO,
                      const float* __restrict__ LSE, const float* __restrict__ Drow,
                      float* __restrict__ dQ, const Problem p, int tiles) {
  using S = F32Shape<D>;
  constexpr int TPR = S::kTpr, E = S::kE;
  __shared__ __align__(16) float Ks[kRows][D];
  __shared__ __align__(16) float Vs[kRows][D];

  const int bh = blockIdx.x / tiles;
  const int tile = blockIdx.x % tiles;
  const F32Seq sq = f32_seq(p, bh, D, threadIdx.x == 0);
  // past the sequence's queries, or no keys (then its query rows are not written)
  if (tile * kRows >= sq.lq || sq.lk == 0) return;
  const int r = threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const int row = tile * kRows + r;
  const bool valid = row < sq.lq;

  float q[E], g[E], dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const size_t at = sq.q0 + static_cast<size_t>(row) * sq.rs + TPR * e + part;
    q[e] = valid ? Q[at] : 0.f;
    g[e] = valid ? dO[at] : 0.f;
    dq[e] = 0.f;
  }
  const float lse = valid ? LSE[sq.lse0 + row] : 0.f;
  const float drow = valid ? Drow[sq.d0 + row] : 0.f;

  const int last_row = min(sq.lq - 1, (tile + 1) * kRows - 1);
  const int key_end = p.causal ? min(sq.lk, last_row + sq.off + 1) : sq.lk;
  for (int k0 = 0; k0 < key_end; k0 += kRows) {
    __syncthreads();
    stage_rows<D, S::kThreads>(Ks, K + sq.k0, sq.rs, k0, sq.lk);
    stage_rows<D, S::kThreads>(Vs, V + sq.k0, sq.rs, k0, sq.lk);
    __syncthreads();
#pragma unroll 1
    for (int j0 = 0; j0 < kRows; j0 += kChunk) {
      float ds[kChunk];
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj) {
        const int j = j0 + jj;
        float s_part = 0.f, dp_part = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s_part = fmaf(q[e], Ks[j][TPR * e + part], s_part);
          dp_part = fmaf(g[e], Vs[j][TPR * e + part], dp_part);
        }
        const float s = row_sum<TPR>(s_part);
        const float dp = row_sum<TPR>(dp_part);
        const int key = k0 + j;
        const bool visible = valid && key < sq.lk && (!p.causal || key <= row + sq.off);
        const float pr = visible ? expf(s * p.scale - lse) : 0.f;
        ds[jj] = pr * (dp - drow);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float a = dq[e];
#pragma unroll
        for (int jj = 0; jj < kChunk; ++jj) a = fmaf(ds[jj], Ks[j0 + jj][TPR * e + part], a);
        dq[e] = a;
      }
    }
  }
  if (!valid) return;
#pragma unroll
  for (int e = 0; e < E; ++e)
    dQ[sq.q0 + static_cast<size_t>(row) * sq.rs + TPR * e + part] = dq[e] * p.scale;
}

template <int D>
cudaError_t launch_d(const float* Q, const float* K, const float* V, const float* dO,
                     const float* O, const float* LSE, float* dQ, float* dK, float* dV,
                     float* Drow, const Problem& p, cudaStream_t stream) {
  using S = F32Shape<D>;
  const long long rows = static_cast<long long>(p.BH) * p.N;
  const int q_tiles = (p.N + kRows - 1) / kRows;
  const int k_tiles = (p.Nk + kRows - 1) / kRows;
  cudaError_t e = trace_mark(p, 0, stream);
  if (e != cudaSuccess) return e;
  bwd_f32_prep_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      O, dO, Drow, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = trace_mark(p, 1, stream)) != cudaSuccess) return e;
  bwd_f32_dkdv_kernel<D>
      <<<static_cast<unsigned>(k_tiles) * static_cast<unsigned>(p.BH), S::kThreads, 0,
         stream>>>(Q, K, V, dO, LSE, Drow, dK, dV, p, k_tiles);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = trace_mark(p, 2, stream)) != cudaSuccess) return e;
  bwd_f32_dq_kernel<D>
      <<<static_cast<unsigned>(q_tiles) * static_cast<unsigned>(p.BH), S::kThreads, 0,
         stream>>>(Q, K, V, dO, LSE, Drow, dQ, p, q_tiles);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_mark(p, 3, stream);
}

}  // namespace

cudaError_t launch_bwd_f32(const float* Q, const float* K, const float* V, const float* O,
                           const float* dO, const float* LSE, float* dQ, float* dK, float* dV,
                           float* workspace, const Problem& p, cudaStream_t stream) {
  if (p.d == 64) return launch_d<64>(Q, K, V, dO, O, LSE, dQ, dK, dV, workspace, p, stream);
  return launch_d<128>(Q, K, V, dO, O, LSE, dQ, dK, dV, workspace, p, stream);
}

}  // namespace fa

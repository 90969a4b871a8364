// zero_rows.cu -- the key gradients of calls that have keys but no query rows.
//
// dK_j = scale * sum_i dS_ij q_i and dV_j = sum_i P_ij dO_i sum over the queries that see
// key j; with no queries at all both sums are empty and the gradients are exactly zero.
// The tensor-core and float32 backward kernels write those zeros themselves for a
// sequence of a batch that has no queries; this kernel does it when the whole call has
// none (Nq == 0, or no query tokens in the packed layout), where there is no query tile
// to run the backward kernels over.  It writes rows [0, lk) of every sequence's dK and
// dV and nothing past them, in any of the three layouts (dense, padded, packed).
#include <cstdint>

#include "f32_seq.cuh"
#include "internal.h"

namespace fa {
namespace {

constexpr int kThreads = 256;

// One thread per 16 bytes of a key row, grid-stride over the B*H*Nk row grid.
__global__ void __launch_bounds__(kThreads)
    zero_key_rows_kernel(uint8_t* dK, uint8_t* dV, const Problem p, int elem_bytes) {
  const int chunks = p.d * elem_bytes / 16;  // 16-byte pieces of one row
  const long long total = static_cast<long long>(p.BH) * p.Nk * chunks;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += stride) {
    const long long row = t / chunks;
    const int c = static_cast<int>(t % chunks);
    const int bh = static_cast<int>(row / p.Nk);
    const int r = static_cast<int>(row % p.Nk);
    // lengths out of range are reported once per head and the head is left alone
    const F32Seq sq = f32_seq(p, bh, p.d, r == 0 && c == 0);
    if (sq.lq != 0 || r >= sq.lk) continue;
    const size_t at = (sq.k0 + static_cast<size_t>(r) * sq.rs) * elem_bytes + 16u * c;
    *reinterpret_cast<uint4*>(dK + at) = make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(dV + at) = make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

cudaError_t launch_zero_key_rows(void* dK, void* dV, const Problem& p, int elem_bytes,
                                 int num_sms, cudaStream_t stream) {
  const long long total = static_cast<long long>(p.BH) * p.Nk * (p.d * elem_bytes / 16);
  if (total == 0) return cudaSuccess;
  long long blocks = (total + kThreads - 1) / kThreads;
  const long long cap = static_cast<long long>(num_sms > 0 ? num_sms : 1) * 8;
  if (blocks > cap) blocks = cap;
  zero_key_rows_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<uint8_t*>(dK), static_cast<uint8_t*>(dV), p, elem_bytes);
  return cudaGetLastError();
}

}  // namespace fa

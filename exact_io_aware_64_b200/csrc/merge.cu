// merge.cu -- combine attention results computed over disjoint sets of keys.
//
// A partial result over a key set A is O_A (rows of softmax-weighted values over A) and
// LSE_A (the log of each row's normaliser over A).  Over A and B together the normaliser
// is exp(LSE_A) + exp(LSE_B), so with m = max(LSE_A, LSE_B) and w = exp(LSE - m):
//   O = (w_A O_A + w_B O_B) / (w_A + w_B),   LSE = m + log(w_A + w_B).
// This is the rescale-and-add step of the online softmax ("FlashAttention, simplified",
// "The trick") applied to two whole partial results, as context-parallel attention does
// when each GPU holds a block of the keys.  An empty set has LSE = -inf and weight 0.
//
// Mapping: one warp per query row, each lane holding d / 32 consecutive elements; the
// accumulator is float32 so that a chain of merges rounds to bf16 only once, at the end.
//
// The same file holds the float32 accumulation of gradients over key blocks that the
// context-parallel backward needs (acc += part, with a final bf16 copy).
#include <cmath>
#include <cstdint>

#include <cuda_bf16.h>

#include "internal.h"

namespace fa {
namespace {

constexpr int kRowsPerBlock = 8;  // warps per CTA

template <int D>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
    merge_kernel(float* __restrict__ Oacc, float* __restrict__ Lacc,
                 const __nv_bfloat16* __restrict__ Opart, const float* __restrict__ Lpart,
                 __nv_bfloat16* __restrict__ Oout, long long rows) {
  constexpr int E = D / 32;  // elements per lane: 2 or 4
  const long long row = static_cast<long long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const float la = Lacc[row], lb = Lpart[row];
  const float m = fmaxf(la, lb);
  float wa = 0.f, wb = 0.f, inv = 0.f, lnew = -INFINITY;
  if (m != -INFINITY) {
    wa = expf(la - m);
    wb = expf(lb - m);
    const float s = wa + wb;
    inv = 1.f / s;
    lnew = m + logf(s);
  }
  const size_t off = static_cast<size_t>(row) * D + lane * E;
  float a[E], b[E], o[E];
  if constexpr (E == 4) {
    const float4 va = *reinterpret_cast<const float4*>(Oacc + off);
    a[0] = va.x, a[1] = va.y, a[2] = va.z, a[3] = va.w;
    const uint2 vb = *reinterpret_cast<const uint2*>(Opart + off);
    const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vb.x));
    const float2 b23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vb.y));
    b[0] = b01.x, b[1] = b01.y, b[2] = b23.x, b[3] = b23.y;
  } else {
    const float2 va = *reinterpret_cast<const float2*>(Oacc + off);
    a[0] = va.x, a[1] = va.y;
    const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Opart + off));
    b[0] = b01.x, b[1] = b01.y;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    // an empty side contributes nothing, whatever its stored values
    const float ta = wa > 0.f ? wa * a[e] : 0.f;
    const float tb = wb > 0.f ? wb * b[e] : 0.f;
    o[e] = (ta + tb) * inv;
  }
  if constexpr (E == 4) {
    *reinterpret_cast<float4*>(Oacc + off) = make_float4(o[0], o[1], o[2], o[3]);
    if (Oout != nullptr) {
      const __nv_bfloat162 p01 = __floats2bfloat162_rn(o[0], o[1]);
      const __nv_bfloat162 p23 = __floats2bfloat162_rn(o[2], o[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&p01);
      pk.y = *reinterpret_cast<const uint32_t*>(&p23);
      *reinterpret_cast<uint2*>(Oout + off) = pk;
    }
  } else {
    *reinterpret_cast<float2*>(Oacc + off) = make_float2(o[0], o[1]);
    if (Oout != nullptr)
      *reinterpret_cast<__nv_bfloat162*>(Oout + off) = __floats2bfloat162_rn(o[0], o[1]);
  }
  if (lane == 0) Lacc[row] = lnew;
}

// acc[i] += part[i] for n elements (float32 += bf16), 8 per thread with 16-byte loads of
// the bf16 operand; out[i] = bf16(acc[i]) when out is given.  n is a multiple of 8.
__global__ void __launch_bounds__(256)
    accumulate_kernel(float* __restrict__ acc, const __nv_bfloat16* __restrict__ part,
                      __nv_bfloat16* __restrict__ out, long long n8) {
  const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n8) return;
  const uint4 pv = reinterpret_cast<const uint4*>(part)[i];
  float4* a4 = reinterpret_cast<float4*>(acc) + 2 * i;
  float4 a0 = a4[0], a1 = a4[1];
  const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&pv);
  const float2 f0 = __bfloat1622float2(p2[0]), f1 = __bfloat1622float2(p2[1]);
  const float2 f2 = __bfloat1622float2(p2[2]), f3 = __bfloat1622float2(p2[3]);
  a0.x += f0.x, a0.y += f0.y, a0.z += f1.x, a0.w += f1.y;
  a1.x += f2.x, a1.y += f2.y, a1.z += f3.x, a1.w += f3.y;
  a4[0] = a0;
  a4[1] = a1;
  if (out != nullptr) {
    uint4 o;
    const __nv_bfloat162 o0 = __floats2bfloat162_rn(a0.x, a0.y), o1 = __floats2bfloat162_rn(a0.z, a0.w);
    const __nv_bfloat162 o2 = __floats2bfloat162_rn(a1.x, a1.y), o3 = __floats2bfloat162_rn(a1.z, a1.w);
    o.x = *reinterpret_cast<const uint32_t*>(&o0);
    o.y = *reinterpret_cast<const uint32_t*>(&o1);
    o.z = *reinterpret_cast<const uint32_t*>(&o2);
    o.w = *reinterpret_cast<const uint32_t*>(&o3);
    reinterpret_cast<uint4*>(out)[i] = o;
  }
}

template <int D>
cudaError_t launch_d(float* Oacc, float* Lacc, const void* Opart, const float* Lpart,
                     void* Oout, const Problem& p, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.BH) * p.N;
  cudaError_t e = trace_mark(p, 0, stream);
  if (e != cudaSuccess) return e;
  merge_kernel<D><<<static_cast<unsigned>((rows + kRowsPerBlock - 1) / kRowsPerBlock),
                    kRowsPerBlock * 32, 0, stream>>>(
      Oacc, Lacc, static_cast<const __nv_bfloat16*>(Opart), Lpart,
      static_cast<__nv_bfloat16*>(Oout), rows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_mark(p, 1, stream);
}

}  // namespace

cudaError_t launch_accumulate(float* acc, const void* part, void* out, long long n,
                              const Problem& p, cudaStream_t stream) {
  const long long n8 = n / 8;
  cudaError_t e = trace_mark(p, 0, stream);
  if (e != cudaSuccess) return e;
  accumulate_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(
      acc, static_cast<const __nv_bfloat16*>(part), static_cast<__nv_bfloat16*>(out), n8);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_mark(p, 1, stream);
}

cudaError_t launch_merge(float* Oacc, float* Lacc, const void* Opart, const float* Lpart,
                         void* Oout, const Problem& p, cudaStream_t stream) {
  if (p.d == 64) return launch_d<64>(Oacc, Lacc, Opart, Lpart, Oout, p, stream);
  return launch_d<128>(Oacc, Lacc, Opart, Lpart, Oout, p, stream);
}

}  // namespace fa

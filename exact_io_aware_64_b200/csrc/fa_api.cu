// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor-map
// construction, kernel launches, status reporting.
//
// Everything here runs on the host.  Validation happens before any CUDA call, so a bad
// argument is reported without touching the device.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime_api.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "internal.h"

// Set by kernels when a pipeline wait runs out of time (see sm100.cuh).
__device__ unsigned int g_fa_device_error;

namespace {

thread_local char g_last_error[512] = "";
constexpr int kMaxTrace = 8;
thread_local cudaEvent_t g_trace[kMaxTrace] = {};
thread_local int g_n_trace = 0;

fa_status fail(fa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

fa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------------ per-device facts
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
  unsigned int* err = nullptr;  // device address of g_fa_device_error
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

fa_status device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_fa_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "querying the device");
    d.ready = true;
  }
  *out = d;
  return FA_OK;
}

fa_status require_sm100(const DeviceInfo& d) {
  if (d.cc_major != 10 || d.cc_minor != 0)
    return fail(FA_ERR_UNSUPPORTED,
                "the kernels are built for sm_100a (B200); this device is sm_%d%d",
                d.cc_major, d.cc_minor);
  return FA_OK;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [BH][N][d] bf16 viewed as a 3-D tensor; boxes of 64 elements x `rows` rows x 1 head
// with the 128-byte swizzle that the tensor-core shared-memory descriptors expect (128
// rows for the operand tiles, 32 for the forward's per-warp output stores).  Rows past N
// inside a head read as zeros.
fa_status make_tmap(CUtensorMap* tm, const void* ptr, int BH, int N, int d, int rows = 128) {
  auto fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FA_OK;
}

// Packed [tokens][H][d] bf16 viewed as a 3-D tensor {d, H, tokens}; boxes of 64
// elements x 1 head x `rows` tokens, which land in shared memory exactly like the boxes
// above (`rows` rows of 128 bytes, 128-byte swizzle).  Tokens past the end read as zeros.
fa_status make_tmap_packed(CUtensorMap* tm, const void* ptr, int tokens, int H, int d,
                           int rows = 128) {
  auto fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FA_OK;
}

// [BH][rows] float32 (a per-row statistic padded to whole tiles) viewed as a 3-D tensor
// [1][BH][rows] with boxes of 128 rows, no swizzle.
fa_status make_row_tmap(CUtensorMap* tm, const float* ptr, int BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH), 1};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(rows) * 4,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(BH) * 4};
  cuuint32_t box[3] = {128, 1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FA_OK;
}

// ------------------------------------------------------------------ validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a + a_bytes) and [b, b + b_bytes) share a byte
bool overlaps(const void* a, size_t a_bytes, const void* b, size_t b_bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + b_bytes && y < x + a_bytes;
}

// Longest sequence any call accepts: every length rounded up to whole 256-row units
// still fits a 32-bit int.
constexpr int kMaxRows = 0x7fffffff - 255;

// Checks shared by every call: Nq query rows and Nk key rows per head (Nk == Nq for
// the entry points without the _qk suffix).  Sets *noop when there is nothing to
// compute.
fa_status check_common(int B, int H, int Nq, int Nk, int d, float scale, int causal,
                       bool* noop) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0)
    return fail(FA_ERR_INVALID_ARG, "sizes must be non-negative (B=%d H=%d Nq=%d Nk=%d)", B,
                H, Nq, Nk);
  if (d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "head dimension d=%d is not supported (64 or 128)", d);
  if (!(std::isfinite(scale) && scale > 0.f))
    return fail(FA_ERR_INVALID_ARG, "scale must be finite and positive");
  if (causal != 0 && causal != 1) return fail(FA_ERR_INVALID_ARG, "causal must be 0 or 1");
  const long long bh = static_cast<long long>(B) * H;
  // work units and row indices are 32-bit on the device, and lengths are rounded up to
  // whole 256-row units in 32-bit arithmetic there
  for (const int n : {Nq, Nk}) {
    if (n > kMaxRows)
      return fail(FA_ERR_INVALID_ARG, "N = %d rows is too large (at most %d)", n, kMaxRows);
    const long long units = (static_cast<long long>(n) + 255) / 256;
    if (bh > 0 && n > 0 && (bh > (1ll << 31) / units || bh * n >= (1ll << 31)))
      return fail(FA_ERR_INVALID_ARG, "B*H*N = %lld rows is too large", bh * n);
  }
  *noop = (bh == 0 || Nq == 0);
  if (*noop) return FA_OK;
  if (Nk == 0) return fail(FA_ERR_INVALID_ARG, "queries need at least one key (Nk=0)");
  if (causal && Nq > Nk)
    return fail(FA_ERR_INVALID_ARG,
                "causal attention needs Nq <= Nk: the queries are the last Nq of the Nk "
                "tokens (Nq=%d Nk=%d)", Nq, Nk);
  return FA_OK;
}

fa_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(FA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(FA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return FA_OK;
}

#define FA_TRY(x)                      \
  do {                                 \
    fa_status _s = (x);                \
    if (_s != FA_OK) return _s;        \
  } while (0)

// Argument checks of the forward calls (elem = bytes per element of the tensors).
fa_status check_fwd_args(const void* Q, const void* K, const void* V, const void* O,
                         const float* LSE, int B, int H, int Nq, int Nk, int d, float scale,
                         int causal, size_t elem, bool* noop) {
  FA_TRY(check_common(B, H, Nq, Nk, d, scale, causal, noop));
  if (*noop) return FA_OK;
  FA_TRY(check_ptr(Q, "Q"));
  FA_TRY(check_ptr(K, "K"));
  FA_TRY(check_ptr(V, "V"));
  FA_TRY(check_ptr(O, "O"));
  if (LSE != nullptr && (reinterpret_cast<uintptr_t>(LSE) & 3u))
    return fail(FA_ERR_INVALID_ARG, "LSE is not 4-byte aligned");
  const size_t qb = static_cast<size_t>(B) * H * Nq * d * elem;
  const size_t kb = static_cast<size_t>(B) * H * Nk * d * elem;
  if (overlaps(O, qb, Q, qb) || overlaps(O, qb, K, kb) || overlaps(O, qb, V, kb))
    return fail(FA_ERR_INVALID_ARG, "O overlaps an input");
  return FA_OK;
}

// Argument checks of the backward calls (elem = bytes per element of the tensors).
// Q, O, dO, dQ have Nq rows per head; K, V, dK, dV have Nk.
fa_status check_bwd_args(const void* Q, const void* K, const void* V, const void* O,
                         const void* dO, const float* LSE, const void* dQ, const void* dK,
                         const void* dV, int B, int H, int Nq, int Nk, int d, float scale,
                         int causal, const void* workspace, size_t workspace_bytes,
                         size_t elem, bool* noop) {
  FA_TRY(check_common(B, H, Nq, Nk, d, scale, causal, noop));
  if (*noop) return FA_OK;
  FA_TRY(check_ptr(Q, "Q"));
  FA_TRY(check_ptr(K, "K"));
  FA_TRY(check_ptr(V, "V"));
  FA_TRY(check_ptr(O, "O"));
  FA_TRY(check_ptr(dO, "dO"));
  FA_TRY(check_ptr(LSE, "LSE"));
  FA_TRY(check_ptr(dQ, "dQ"));
  FA_TRY(check_ptr(dK, "dK"));
  FA_TRY(check_ptr(dV, "dV"));
  const size_t need = fa_bwd_workspace_bytes(B, H, Nq, d);
  if (need > 0) {
    FA_TRY(check_ptr(workspace, "workspace"));
    if (workspace_bytes < need)
      return fail(FA_ERR_INVALID_ARG, "workspace has %zu bytes, %zu needed", workspace_bytes,
                  need);
  }
  const size_t qb = static_cast<size_t>(B) * H * Nq * d * elem;
  const size_t kb = static_cast<size_t>(B) * H * Nk * d * elem;
  struct Buf {
    const void* p;
    size_t n;
  };
  const Buf ins[5] = {{Q, qb}, {K, kb}, {V, kb}, {O, qb}, {dO, qb}};
  const Buf outs[3] = {{dQ, qb}, {dK, kb}, {dV, kb}};
  for (const Buf& o : outs) {
    for (const Buf& in : ins)
      if (overlaps(o.p, o.n, in.p, in.n))
        return fail(FA_ERR_INVALID_ARG, "a gradient overlaps an input");
    if (need > 0 && overlaps(o.p, o.n, workspace, need))
      return fail(FA_ERR_INVALID_ARG, "a gradient overlaps the workspace");
  }
  if (overlaps(dQ, qb, dK, kb) || overlaps(dQ, qb, dV, kb) || overlaps(dK, kb, dV, kb))
    return fail(FA_ERR_INVALID_ARG, "gradients overlap each other");
  return FA_OK;
}

fa::Problem make_problem(int B, int H, int Nq, int Nk, int d, float scale, int causal,
                         const DeviceInfo& dev, const int* seqlens_q = nullptr,
                         const int* seqlens_k = nullptr, const int* cu_q = nullptr,
                         const int* cu_k = nullptr, int total_q = 0, int total_k = 0) {
  fa::Problem p{};
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.BH = B * H;
  p.N = Nq;
  p.Nk = Nk;
  p.d = d;
  p.scale = scale;
  p.causal = causal;
  p.err = dev.err;
  p.seqlens_q = seqlens_q;
  p.seqlens_k = seqlens_k;
  p.H = H;
  p.trace = g_n_trace ? g_trace : nullptr;
  p.n_trace = g_n_trace;
  return p;
}

// Per-sequence length arrays of the padded-batch calls: both given, 4-byte aligned.
fa_status check_seqlens(const int* seqlens_q, const int* seqlens_k) {
  if (seqlens_q == nullptr || seqlens_k == nullptr)
    return fail(FA_ERR_INVALID_ARG, "seqlens_q and seqlens_k are required");
  if ((reinterpret_cast<uintptr_t>(seqlens_q) | reinterpret_cast<uintptr_t>(seqlens_k)) & 3u)
    return fail(FA_ERR_INVALID_ARG, "seqlens_q and seqlens_k must be 4-byte aligned");
  return FA_OK;
}

// A backward call with keys but no query rows (Nq == 0, or no query tokens in the
// packed layout): no query sees any key, so dK and dV are exactly zero in every key row
// of every sequence; rows past a sequence's key length stay unwritten as elsewhere.
// Its arguments are checked (check_key_grads) before the device is queried.
fa_status check_key_grads(const void* dK, const void* dV, size_t key_bytes) {
  FA_TRY(check_ptr(dK, "dK"));
  FA_TRY(check_ptr(dV, "dV"));
  if (overlaps(dK, key_bytes, dV, key_bytes))
    return fail(FA_ERR_INVALID_ARG, "gradients overlap each other");
  return FA_OK;
}

fa_status zero_key_grads(void* dK, void* dV, const fa::Problem& p, size_t elem,
                         const DeviceInfo& dev, cudaStream_t stream) {
  cudaError_t e = fa::launch_zero_key_rows(dK, dV, p, static_cast<int>(elem), dev.num_sms,
                                           stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the key-gradient zero fill");
  return FA_OK;
}

fa_status fwd_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                   int H, int Nq, int Nk, int d, float scale, int causal, cudaStream_t stream,
                   const int* seqlens_q = nullptr, const int* seqlens_k = nullptr) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_fwd_args(Q, K, V, O, LSE, B, H, Nq, Nk, d, scale, causal, 2, &noop));
  if (noop) return FA_OK;  // empty problem: the pointers are never used (may be NULL)
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  FA_TRY(require_sm100(dev));
  const int BH = B * H;
  CUtensorMap tmQ, tmK, tmV, tmO;
  FA_TRY(make_tmap(&tmQ, Q, BH, Nq, d));
  FA_TRY(make_tmap(&tmK, K, BH, Nk, d));
  FA_TRY(make_tmap(&tmV, V, BH, Nk, d));
  FA_TRY(make_tmap(&tmO, O, BH, Nq, d, 32));
  const fa::Problem p = make_problem(B, H, Nq, Nk, d, scale, causal, dev, seqlens_q, seqlens_k);
  cudaError_t e = fa::launch_fwd_sm100(tmQ, tmK, tmV, tmO, O, LSE, p, dev.num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the forward kernel");
  return FA_OK;
}

fa_status bwd_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                   const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int Nq, int Nk,
                   int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream, const int* seqlens_q = nullptr,
                   const int* seqlens_k = nullptr) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Nq, Nk, d, scale, causal,
                        workspace, workspace_bytes, 2, &noop));
  if (noop) {
    // no work, and then no pointer is used (they may be NULL) -- unless there are keys
    // without queries, whose gradients are zeros to be written
    if (static_cast<long long>(B) * H == 0 || Nk == 0) return FA_OK;
    FA_TRY(check_key_grads(dK, dV, static_cast<size_t>(B) * H * Nk * d * 2));
    DeviceInfo dev;
    FA_TRY(device_info(&dev));
    const fa::Problem p = make_problem(B, H, Nq, Nk, d, scale, causal, dev, seqlens_q,
                                       seqlens_k);
    return zero_key_grads(dK, dV, p, 2, dev, stream);
  }
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  FA_TRY(require_sm100(dev));
  const int BH = B * H;
  CUtensorMap tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV;
  FA_TRY(make_tmap(&tmQ, Q, BH, Nq, d));
  FA_TRY(make_tmap(&tmK, K, BH, Nk, d));
  FA_TRY(make_tmap(&tmV, V, BH, Nk, d));
  FA_TRY(make_tmap(&tmdO, dO, BH, Nq, d));
  FA_TRY(make_tmap(&tmdK, dK, BH, Nk, d, 32));
  FA_TRY(make_tmap(&tmdV, dV, BH, Nk, d, 32));
  const int Npad = static_cast<int>(fa::bwd_padded_rows(Nq));  // Nq <= kMaxRows
  float* ws = static_cast<float*>(workspace);
  FA_TRY(make_row_tmap(&tmD, ws, BH, Npad));
  FA_TRY(make_row_tmap(&tmL2, ws + static_cast<size_t>(BH) * Npad, BH, Npad));
  const fa::Problem p = make_problem(B, H, Nq, Nk, d, scale, causal, dev, seqlens_q, seqlens_k);
  cudaError_t e = fa::launch_bwd_sm100(tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV, O, dO, LSE,
                                       dQ, dK, dV, ws, p, dev.num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the backward kernels");
  return FA_OK;
}

// The start-token arrays of the packed-layout calls: both given, 4-byte aligned.
fa_status check_cu(const int* cu_q, const int* cu_k) {
  if (cu_q == nullptr || cu_k == nullptr)
    return fail(FA_ERR_INVALID_ARG, "cu_seqlens_q and cu_seqlens_k are required");
  if ((reinterpret_cast<uintptr_t>(cu_q) | reinterpret_cast<uintptr_t>(cu_k)) & 3u)
    return fail(FA_ERR_INVALID_ARG, "cu_seqlens_q and cu_seqlens_k must be 4-byte aligned");
  return FA_OK;
}

// Checks of the packed-layout calls: lengths, totals and the start-token arrays.
fa_status check_packed(const int* cu_q, const int* cu_k, int B, int H, int max_q, int max_k,
                       int total_q, int total_k, int d, float scale, int causal, bool* noop) {
  FA_TRY(check_common(B, H, max_q, max_k, d, scale, causal, noop));
  if (total_q < 0 || total_k < 0)
    return fail(FA_ERR_INVALID_ARG, "token totals must be non-negative");
  const long long h = H;
  if (h * total_q >= (1ll << 31) || h * total_k >= (1ll << 31))
    return fail(FA_ERR_INVALID_ARG, "H * tokens is too large");
  if (*noop || total_q == 0) {
    *noop = true;
    return FA_OK;
  }
  return check_cu(cu_q, cu_k);
}

// Pointer and overlap checks of the packed-layout forward calls (elem = bytes per
// element of Q, K, V, O).
fa_status check_packed_fwd_ptrs(const void* Q, const void* K, const void* V, const void* O,
                                const float* LSE, int H, int d, int total_q, int total_k,
                                size_t elem) {
  FA_TRY(check_ptr(Q, "Q"));
  FA_TRY(check_ptr(K, "K"));
  FA_TRY(check_ptr(V, "V"));
  FA_TRY(check_ptr(O, "O"));
  if (LSE != nullptr && (reinterpret_cast<uintptr_t>(LSE) & 3u))
    return fail(FA_ERR_INVALID_ARG, "LSE is not 4-byte aligned");
  const size_t qb = static_cast<size_t>(total_q) * H * d * elem;
  const size_t kb = static_cast<size_t>(total_k) * H * d * elem;
  if (overlaps(O, qb, Q, qb) || overlaps(O, qb, K, kb) || overlaps(O, qb, V, kb))
    return fail(FA_ERR_INVALID_ARG, "O overlaps an input");
  return FA_OK;
}

// Pointer, workspace and overlap checks of the packed-layout backward calls.
fa_status check_packed_bwd_ptrs(const void* Q, const void* K, const void* V, const void* O,
                                const void* dO, const float* LSE, const void* dQ,
                                const void* dK, const void* dV, int H, int d, int total_q,
                                int total_k, const void* workspace, size_t need,
                                size_t workspace_bytes, size_t elem) {
  FA_TRY(check_ptr(Q, "Q"));
  FA_TRY(check_ptr(K, "K"));
  FA_TRY(check_ptr(V, "V"));
  FA_TRY(check_ptr(O, "O"));
  FA_TRY(check_ptr(dO, "dO"));
  FA_TRY(check_ptr(LSE, "LSE"));
  FA_TRY(check_ptr(dQ, "dQ"));
  FA_TRY(check_ptr(dK, "dK"));
  FA_TRY(check_ptr(dV, "dV"));
  FA_TRY(check_ptr(workspace, "workspace"));
  if (workspace_bytes < need)
    return fail(FA_ERR_INVALID_ARG, "workspace has %zu bytes, %zu needed", workspace_bytes,
                need);
  const size_t qb = static_cast<size_t>(total_q) * H * d * elem;
  const size_t kb = static_cast<size_t>(total_k) * H * d * elem;
  struct Buf {
    const void* p;
    size_t n;
  };
  const Buf ins[5] = {{Q, qb}, {K, kb}, {V, kb}, {O, qb}, {dO, qb}};
  const Buf outs[3] = {{dQ, qb}, {dK, kb}, {dV, kb}};
  for (const Buf& o : outs) {
    for (const Buf& in : ins)
      if (overlaps(o.p, o.n, in.p, in.n))
        return fail(FA_ERR_INVALID_ARG, "a gradient overlaps an input");
    if (overlaps(o.p, o.n, workspace, need))
      return fail(FA_ERR_INVALID_ARG, "a gradient overlaps the workspace");
  }
  if (overlaps(dQ, qb, dK, kb) || overlaps(dQ, qb, dV, kb) || overlaps(dK, kb, dV, kb))
    return fail(FA_ERR_INVALID_ARG, "gradients overlap each other");
  return FA_OK;
}

// float32 forward, dense or padded layout (seqlens null: every row of every head).
fa_status fwd_f32_impl(const float* Q, const float* K, const float* V, float* O, float* LSE,
                       int B, int H, int Nq, int Nk, int d, float scale, int causal,
                       cudaStream_t stream, const int* seqlens_q = nullptr,
                       const int* seqlens_k = nullptr) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_fwd_args(Q, K, V, O, LSE, B, H, Nq, Nk, d, scale, causal, 4, &noop));
  if (noop) return FA_OK;  // empty problem: the pointers are never used (may be NULL)
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(B, H, Nq, Nk, d, scale, causal, dev, seqlens_q, seqlens_k);
  cudaError_t e = fa::launch_fwd_f32(Q, K, V, O, LSE, p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the float32 forward kernel");
  return FA_OK;
}

// float32 backward, dense or padded layout.
fa_status bwd_f32_impl(const float* Q, const float* K, const float* V, const float* O,
                       const float* dO, const float* LSE, float* dQ, float* dK, float* dV,
                       int B, int H, int Nq, int Nk, int d, float scale, int causal,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream,
                       const int* seqlens_q = nullptr, const int* seqlens_k = nullptr) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_bwd_args(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Nq, Nk, d, scale, causal,
                        workspace, workspace_bytes, 4, &noop));
  if (noop) {
    // as in bwd_impl: keys without queries get zero gradients
    if (static_cast<long long>(B) * H == 0 || Nk == 0) return FA_OK;
    FA_TRY(check_key_grads(dK, dV, static_cast<size_t>(B) * H * Nk * d * 4));
    DeviceInfo dev;
    FA_TRY(device_info(&dev));
    const fa::Problem p = make_problem(B, H, Nq, Nk, d, scale, causal, dev, seqlens_q,
                                       seqlens_k);
    return zero_key_grads(dK, dV, p, 4, dev, stream);
  }
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(B, H, Nq, Nk, d, scale, causal, dev, seqlens_q, seqlens_k);
  cudaError_t e = fa::launch_bwd_f32(Q, K, V, O, dO, LSE, dQ, dK, dV,
                                     static_cast<float*>(workspace), p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the float32 backward kernels");
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_abi_version(void) { return 1; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

const char* fa_last_error_message(void) { return g_last_error; }

fa_status fa_trace_events(cudaEvent_t* events, int n) {
  g_last_error[0] = '\0';
  if (n < 0 || n > kMaxTrace || (n > 0 && events == nullptr))
    return fail(FA_ERR_INVALID_ARG, "fa_trace_events: n=%d (0..%d, events non-NULL)", n,
                kMaxTrace);
  for (int k = 0; k < n; ++k) g_trace[k] = events[k];
  g_n_trace = n;
  return FA_OK;
}

fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
                 int N, int d, float scale, int causal, cudaStream_t stream) {
  return fwd_impl(Q, K, V, O, LSE, B, H, N, N, d, scale, causal, stream);
}

fa_status fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                    int H, int Nq, int Nk, int d, float scale, int causal,
                    cudaStream_t stream) {
  return fwd_impl(Q, K, V, O, LSE, B, H, Nq, Nk, d, scale, causal, stream);
}

fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                        const int* seqlens_q, const int* seqlens_k, int B, int H, int Nq,
                        int Nk, int d, float scale, int causal, cudaStream_t stream) {
  g_last_error[0] = '\0';
  if (B > 0 && H > 0 && Nq > 0) FA_TRY(check_seqlens(seqlens_q, seqlens_k));
  return fwd_impl(Q, K, V, O, LSE, B, H, Nq, Nk, d, scale, causal, stream, seqlens_q,
                  seqlens_k);
}

fa_status fa_fwd_packed(const void* Q, const void* K, const void* V, void* O, float* LSE,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                        int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int d,
                        float scale, int causal, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_packed(cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q,
                      total_k, d, scale, causal, &noop));
  if (noop) return FA_OK;
  FA_TRY(check_packed_fwd_ptrs(Q, K, V, O, LSE, H, d, total_q, total_k, 2));
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  FA_TRY(require_sm100(dev));
  CUtensorMap tmQ, tmK, tmV, tmO;
  FA_TRY(make_tmap_packed(&tmQ, Q, total_q, H, d));
  FA_TRY(make_tmap_packed(&tmK, K, total_k, H, d));
  FA_TRY(make_tmap_packed(&tmV, V, total_k, H, d));
  FA_TRY(make_tmap_packed(&tmO, O, total_q, H, d, 32));
  const fa::Problem p = make_problem(B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, dev,
                                     nullptr, nullptr, cu_seqlens_q, cu_seqlens_k, total_q,
                                     total_k);
  cudaError_t e = fa::launch_fwd_sm100(tmQ, tmK, tmV, tmO, O, LSE, p, dev.num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the forward kernel");
  return FA_OK;
}

fa_status fa_bwd_packed(const void* Q, const void* K, const void* V, const void* O,
                        const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                        int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int d,
                        float scale, int causal, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_packed(cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q,
                      total_k, d, scale, causal, &noop));
  if (noop) {
    // keys without queries get zero gradients (see bwd_impl)
    if (static_cast<long long>(B) * H == 0 || total_k == 0 || max_seqlen_k == 0) return FA_OK;
    FA_TRY(check_cu(cu_seqlens_q, cu_seqlens_k));
    FA_TRY(check_key_grads(dK, dV, static_cast<size_t>(total_k) * H * d * 2));
    DeviceInfo dev;
    FA_TRY(device_info(&dev));
    const fa::Problem p = make_problem(B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, dev,
                                       nullptr, nullptr, cu_seqlens_q, cu_seqlens_k, total_q,
                                       total_k);
    return zero_key_grads(dK, dV, p, 2, dev, stream);
  }
  const size_t need = fa_bwd_workspace_bytes(B, H, max_seqlen_q, d);
  FA_TRY(check_packed_bwd_ptrs(Q, K, V, O, dO, LSE, dQ, dK, dV, H, d, total_q, total_k,
                               workspace, need, workspace_bytes, 2));
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  FA_TRY(require_sm100(dev));
  const int BH = B * H;
  CUtensorMap tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV;
  FA_TRY(make_tmap_packed(&tmQ, Q, total_q, H, d));
  FA_TRY(make_tmap_packed(&tmK, K, total_k, H, d));
  FA_TRY(make_tmap_packed(&tmV, V, total_k, H, d));
  FA_TRY(make_tmap_packed(&tmdO, dO, total_q, H, d));
  FA_TRY(make_tmap_packed(&tmdK, dK, total_k, H, d, 32));
  FA_TRY(make_tmap_packed(&tmdV, dV, total_k, H, d, 32));
  const int Npad = static_cast<int>(fa::bwd_padded_rows(max_seqlen_q));
  float* ws = static_cast<float*>(workspace);
  FA_TRY(make_row_tmap(&tmD, ws, BH, Npad));
  FA_TRY(make_row_tmap(&tmL2, ws + static_cast<size_t>(BH) * Npad, BH, Npad));
  const fa::Problem p = make_problem(B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, dev,
                                     nullptr, nullptr, cu_seqlens_q, cu_seqlens_k, total_q,
                                     total_k);
  cudaError_t e = fa::launch_bwd_sm100(tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV, O, dO, LSE,
                                       dQ, dK, dV, ws, p, dev.num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the backward kernels");
  return FA_OK;
}

fa_status fa_fwd_f32(const float* Q, const float* K, const float* V, float* O, float* LSE,
                     int B, int H, int N, int d, float scale, int causal,
                     cudaStream_t stream) {
  return fwd_f32_impl(Q, K, V, O, LSE, B, H, N, N, d, scale, causal, stream);
}

fa_status fa_fwd_f32_qk(const float* Q, const float* K, const float* V, float* O, float* LSE,
                        int B, int H, int Nq, int Nk, int d, float scale, int causal,
                        cudaStream_t stream) {
  return fwd_f32_impl(Q, K, V, O, LSE, B, H, Nq, Nk, d, scale, causal, stream);
}

fa_status fa_fwd_f32_varlen(const float* Q, const float* K, const float* V, float* O,
                            float* LSE, const int* seqlens_q, const int* seqlens_k, int B,
                            int H, int Nq, int Nk, int d, float scale, int causal,
                            cudaStream_t stream) {
  g_last_error[0] = '\0';
  if (B > 0 && H > 0 && Nq > 0) FA_TRY(check_seqlens(seqlens_q, seqlens_k));
  return fwd_f32_impl(Q, K, V, O, LSE, B, H, Nq, Nk, d, scale, causal, stream, seqlens_q,
                      seqlens_k);
}

fa_status fa_fwd_f32_packed(const float* Q, const float* K, const float* V, float* O,
                            float* LSE, const int* cu_seqlens_q, const int* cu_seqlens_k,
                            int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q,
                            int total_k, int d, float scale, int causal,
                            cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_packed(cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q,
                      total_k, d, scale, causal, &noop));
  if (noop) return FA_OK;
  FA_TRY(check_packed_fwd_ptrs(Q, K, V, O, LSE, H, d, total_q, total_k, 4));
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, dev,
                                     nullptr, nullptr, cu_seqlens_q, cu_seqlens_k, total_q,
                                     total_k);
  cudaError_t e = fa::launch_fwd_f32(Q, K, V, O, LSE, p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the float32 forward kernel");
  return FA_OK;
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  (void)d;
  if (B <= 0 || H <= 0 || N <= 0) return 0;
  // D and LSE*log2(e), one float each per query row, rows padded to whole 128-row tiles
  const size_t raw = 2 * static_cast<size_t>(B) * H *
                    static_cast<size_t>(fa::bwd_padded_rows(N)) * sizeof(float);
  return (raw + 255) / 256 * 256;
}

fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                 float scale, int causal, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, N, d, scale, causal, workspace,
                  workspace_bytes, stream);
}

fa_status fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int Nq,
                    int Nk, int d, float scale, int causal, void* workspace,
                    size_t workspace_bytes, cudaStream_t stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Nq, Nk, d, scale, causal, workspace,
                  workspace_bytes, stream);
}

fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O,
                        const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                        const int* seqlens_q, const int* seqlens_k, int B, int H, int Nq,
                        int Nk, int d, float scale, int causal, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  g_last_error[0] = '\0';
  if (B > 0 && H > 0 && (Nq > 0 || Nk > 0)) FA_TRY(check_seqlens(seqlens_q, seqlens_k));
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Nq, Nk, d, scale, causal, workspace,
                  workspace_bytes, stream, seqlens_q, seqlens_k);
}

fa_status fa_bwd_f32(const float* Q, const float* K, const float* V, const float* O,
                     const float* dO, const float* LSE, float* dQ, float* dK, float* dV, int B,
                     int H, int N, int d, float scale, int causal, void* workspace,
                     size_t workspace_bytes, cudaStream_t stream) {
  return bwd_f32_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, N, d, scale, causal,
                      workspace, workspace_bytes, stream);
}

fa_status fa_bwd_f32_qk(const float* Q, const float* K, const float* V, const float* O,
                        const float* dO, const float* LSE, float* dQ, float* dK, float* dV,
                        int B, int H, int Nq, int Nk, int d, float scale, int causal,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return bwd_f32_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Nq, Nk, d, scale, causal,
                      workspace, workspace_bytes, stream);
}

fa_status fa_bwd_f32_varlen(const float* Q, const float* K, const float* V, const float* O,
                            const float* dO, const float* LSE, float* dQ, float* dK,
                            float* dV, const int* seqlens_q, const int* seqlens_k, int B,
                            int H, int Nq, int Nk, int d, float scale, int causal,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  g_last_error[0] = '\0';
  if (B > 0 && H > 0 && (Nq > 0 || Nk > 0)) FA_TRY(check_seqlens(seqlens_q, seqlens_k));
  return bwd_f32_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Nq, Nk, d, scale, causal,
                      workspace, workspace_bytes, stream, seqlens_q, seqlens_k);
}

fa_status fa_bwd_f32_packed(const float* Q, const float* K, const float* V, const float* O,
                            const float* dO, const float* LSE, float* dQ, float* dK,
                            float* dV, const int* cu_seqlens_q, const int* cu_seqlens_k,
                            int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q,
                            int total_k, int d, float scale, int causal, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_packed(cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q,
                      total_k, d, scale, causal, &noop));
  if (noop) {
    // keys without queries get zero gradients (see bwd_impl)
    if (static_cast<long long>(B) * H == 0 || total_k == 0 || max_seqlen_k == 0) return FA_OK;
    FA_TRY(check_cu(cu_seqlens_q, cu_seqlens_k));
    FA_TRY(check_key_grads(dK, dV, static_cast<size_t>(total_k) * H * d * 4));
    DeviceInfo dev;
    FA_TRY(device_info(&dev));
    const fa::Problem p = make_problem(B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, dev,
                                       nullptr, nullptr, cu_seqlens_q, cu_seqlens_k, total_q,
                                       total_k);
    return zero_key_grads(dK, dV, p, 4, dev, stream);
  }
  const size_t need = fa_bwd_workspace_bytes(B, H, max_seqlen_q, d);
  FA_TRY(check_packed_bwd_ptrs(Q, K, V, O, dO, LSE, dQ, dK, dV, H, d, total_q, total_k,
                               workspace, need, workspace_bytes, 4));
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, dev,
                                     nullptr, nullptr, cu_seqlens_q, cu_seqlens_k, total_q,
                                     total_k);
  cudaError_t e = fa::launch_bwd_f32(Q, K, V, O, dO, LSE, dQ, dK, dV,
                                     static_cast<float*>(workspace), p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the float32 backward kernels");
  return FA_OK;
}

fa_status fa_merge(float* O_acc, float* LSE_acc, const void* O_part, const float* LSE_part,
                   void* O_out, int B, int H, int N, int d, cudaStream_t stream) {
  g_last_error[0] = '\0';
  bool noop = false;
  FA_TRY(check_common(B, H, N, N, d, 1.f, 0, &noop));
  if (noop) return FA_OK;  // empty problem: the pointers are never used (may be NULL)
  FA_TRY(check_ptr(O_acc, "O_acc"));
  FA_TRY(check_ptr(O_part, "O_part"));
  if (O_out != nullptr) FA_TRY(check_ptr(O_out, "O_out"));
  if (LSE_acc == nullptr || LSE_part == nullptr)
    return fail(FA_ERR_INVALID_ARG, "LSE_acc and LSE_part are required");
  if ((reinterpret_cast<uintptr_t>(LSE_acc) | reinterpret_cast<uintptr_t>(LSE_part)) & 3u)
    return fail(FA_ERR_INVALID_ARG, "LSE_acc and LSE_part must be 4-byte aligned");
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t acc_b = rows * d * 4, part_b = rows * d * 2, lse_b = rows * 4;
  if (overlaps(O_acc, acc_b, O_part, part_b) || overlaps(O_acc, acc_b, LSE_part, lse_b) ||
      overlaps(LSE_acc, lse_b, O_part, part_b) || overlaps(LSE_acc, lse_b, LSE_part, lse_b) ||
      overlaps(O_acc, acc_b, LSE_acc, lse_b))
    return fail(FA_ERR_INVALID_ARG, "the accumulator overlaps the partial result");
  if (O_out != nullptr &&
      (overlaps(O_out, part_b, O_acc, acc_b) || overlaps(O_out, part_b, LSE_acc, lse_b) ||
       overlaps(O_out, part_b, LSE_part, lse_b)))
    return fail(FA_ERR_INVALID_ARG, "O_out overlaps the accumulator");
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(B, H, N, N, d, 1.f, 0, dev);
  cudaError_t e = fa::launch_merge(O_acc, LSE_acc, O_part, LSE_part, O_out, p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the merge kernel");
  return FA_OK;
}

fa_status fa_accumulate(float* acc, const void* part, void* out, size_t n,
                        cudaStream_t stream) {
  g_last_error[0] = '\0';
  if (n == 0) return FA_OK;
  if (n % 8 != 0) return fail(FA_ERR_INVALID_ARG, "n=%zu is not a multiple of 8", n);
  if (n >= (size_t(1) << 40)) return fail(FA_ERR_INVALID_ARG, "n=%zu is too large", n);
  FA_TRY(check_ptr(acc, "acc"));
  FA_TRY(check_ptr(part, "part"));
  if (out != nullptr) FA_TRY(check_ptr(out, "out"));
  if (overlaps(acc, n * 4, part, n * 2) ||
      (out != nullptr && (overlaps(out, n * 2, acc, n * 4) || overlaps(out, n * 2, part, n * 2))))
    return fail(FA_ERR_INVALID_ARG, "acc, part and out must not overlap");
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(1, 1, 1, 1, 64, 1.f, 0, dev);
  cudaError_t e = fa::launch_accumulate(acc, part, out, static_cast<long long>(n), p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the accumulate kernel");
  return FA_OK;
}

fa_status fa_selftest_timeout(long long limit_cycles, cudaStream_t stream) {
  g_last_error[0] = '\0';
  if (limit_cycles < 0 || limit_cycles > (1ll << 34))
    return fail(FA_ERR_INVALID_ARG, "limit_cycles=%lld out of range (0 .. 2^34)", limit_cycles);
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  const fa::Problem p = make_problem(1, 1, 1, 1, 64, 1.f, 0, dev);
  cudaError_t e = fa::launch_timeout_probe(limit_cycles, p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launching the timeout probe");
  return FA_OK;
}

fa_status fa_check_device_error(cudaStream_t stream) {
  g_last_error[0] = '\0';
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  DeviceInfo dev;
  FA_TRY(device_info(&dev));
  unsigned int word = 0;
  e = cudaMemcpy(&word, dev.err, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpy(dev.err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    if (word & 4u)
      return fail(FA_ERR_INVALID_ARG,
                  "a per-sequence length was negative, above the padded length, or (causal) "
                  "had more queries than keys; that sequence was skipped (error word 0x%x)",
                  word);
    if (word & 2u)
      return fail(FA_ERR_CUDA,
                  "a kernel found its dynamic shared memory misaligned and did no work "
                  "(error word 0x%x)", word);
    return fail(FA_ERR_TIMEOUT, "a kernel pipeline wait timed out (error word 0x%x)", word);
  }
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.
//
// Some callers have no way to hand fa_bwd a workspace: a plugin whose host API gives it
// no allocator, code that runs inside a framework step whose memory plan is frozen, or
// a latency-sensitive loop that must not enter cudaMalloc (which can synchronise the
// device).  For them the library keeps its own scratch: the array below, a fixed
// kNoAllocScratchBytes of device memory that every GPU which loads libfa.so holds until
// the process exits.  The caller still provides every input and output.
//
// In host code `g_fa_bwd_scratch` names a host-side stand-in, not device memory, so it
// is never passed to a kernel directly.  The first fa_bwd_noalloc call on a device looks
// up the array's device address with cudaGetSymbolAddress while that device is current
// and caches it; that first call should therefore come before any stream capture.
//
// Every call shares the one array.  fa_bwd fully rewrites the part it uses (D and
// LSE*log2(e) for every padded row) before reading it, so nothing needs clearing between
// calls, but two calls whose kernels overlap on the GPU (different streams, or another
// thread) race on the array and give wrong gradients: serialise them.
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB: B*H*ceil(N/128)*128 <= 2^20
static __device__ __align__(256) unsigned char g_fa_bwd_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

fa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_fa_bwd_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_fa_bwd_scratch)");
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

size_t fa_bwd_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

fa_status fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                         const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                         int B, int H, int N, int d, float scale, int causal,
                         cudaStream_t stream) {
  g_last_error[0] = '\0';
  void* scratch = nullptr;
  bool noop = false;
  // sizes first: the scratch arithmetic below assumes validated sizes
  fa_status st = check_common(B, H, N, N, d, scale, causal, &noop);
  if (st != FA_OK || noop) return st;
  const size_t need = fa_bwd_workspace_bytes(B, H, N, d);
  if (need > kNoAllocScratchBytes)
    return fail(FA_ERR_INVALID_ARG,
                "fa_bwd_noalloc: B=%d H=%d N=%d needs %zu bytes of scratch, more than the "
                "library's fixed %zu (B*H*ceil(N/128)*128 must be at most %zu); use fa_bwd "
                "with a workspace",
                B, H, N, need, kNoAllocScratchBytes, kNoAllocScratchBytes / 8);
  st = noalloc_scratch(&scratch);
  if (st != FA_OK) return st;
  return fa_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, scratch,
                kNoAllocScratchBytes, stream);
}

}  // extern "C"

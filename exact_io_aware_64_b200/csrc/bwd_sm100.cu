// bwd_sm100.cu -- backward attention on the sm_100a tensor cores.
//
// Method ("What FlashAttention actually buys", "Why the distinction matters downstream":
// the backward recomputes score tiles instead of storing the N x N matrix).  With the
// forward's per-row log-sum-exp L, every probability tile is rebuilt on chip as
// P = exp(scale Q K^T - L); the gradients are the textbook ones
//     dV = P^T dO,  dP = dO V^T,  D_i = sum_k dO_ik O_ik,  dS = P * (dP - D),
//     dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels, no atomics (bitwise reproducible):
//   1. bwd_prep: -D = -rowsum(dO * O) and -L2 = -L * log2(e), both stored padded to
//      whole 128-row tiles in the caller's workspace (rows past N: 0 and -inf, so their
//      probabilities are exactly 0) so that TMA can stream them.  They are stored
//      negated because the element-wise steps add them (packed fused multiply-adds).
//   2. bwd_dkdv: one work unit per (batch*head, 128-row key tile j).  K_j and V_j stay in
//      shared memory while the query tiles i stream past; the tile products are taken
//      transposed so that the key row is the TMEM lane:
//          S^T = K_j Q_i^T,  dP^T = V_j dO_i^T             (SS MMAs into TMEM)
//          P^T = exp2(S^T * scale*log2e - L2_i)            (one thread per key row)
//          dS^T = P^T * (dP^T - D_i)
//          dV_j += P^T dO_i,  dK_j += dS^T Q_i             (TS MMAs, P^T/dS^T from TMEM)
//      TMEM: dV | dK | S^T (P^T over its first 64 columns) | dP^T (dS^T likewise).
//      K_j and V_j are released after the unit's last dP^T product, so the next unit's
//      load overlaps this unit's last products.  At the end of a unit the element-wise
//      warps of group 0 write dV and those of group 1 write dK, each warp its 32 rows,
//      through a 4 KB shared-memory staging box and a bulk tensor store (whole lines
//      instead of a row per lane).
//   3. bwd_dq: one work unit per (batch*head, 128-row query tile i); key and value tiles
//      stream past through separate rings (3 slots for K, which the last product of a
//      tile still reads, 2 for V):  S = Q_i K_j^T, dP = dO_i V_j^T, P, dS as above,
//      dQ_i += dS K_j.
//      TMEM: dQ | S | dP (dS over it) | Q_i | dO_i.  The element-wise warps copy the
//      unit's Q_i and dO_i into tensor memory once, so the S and dP products read only
//      K_j or V_j from shared memory: one SS product alone already uses the whole
//      shared-memory bandwidth, and the TMA writes of the incoming tiles share it.
//
// Both tensor-core kernels are persistent (one CTA per SM) with 384 threads: warps 0-7
// are two element-wise warpgroups that split every 128 x 128 tile by columns (group g
// owns columns 64g..64g+63; thread = TMEM lane = tile row), warp 8 issues TMA loads,
// warp 9 issues the MMAs from one thread, warps 10-11 only give up their registers.  Each group writes its bf16 half-row of P or
// dS over the first 32 columns of its own 64-column half, so the two groups never touch
// each other's TMEM, and the MMA reads the bf16 operand as two 32-column pieces.  The MMA order is chosen so the
// tensor core works on one product while the element-wise warps build the next operand
// (dK/dV: S^T(i) dP^T(i) | dV(i) S^T(i+1) | dK(i) dP^T(i+1) | ..., with dV(i) issued in
// two halves as the two halves of each group's P^T(i) are written;
//  dQ: S(j) dP(j) | S(j+1) dQ(j) dP(j+1) | S(j+2) dQ(j+1) dP(j+2) | ...).
// Causal work units are ordered heaviest first.
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

constexpr int kTile = 128;        // rows per query / key tile
constexpr int kGroups = 2;        // element-wise warpgroups, splitting a tile's columns
constexpr int kCols = kTile / kGroups;
constexpr int kEw = kGroups * 128;  // element-wise threads
constexpr int kThreads = kEw + 128;  // + a control warpgroup: TMA warp, MMA warp, 2 idle
constexpr int kWarpTMA = kEw / 32;
constexpr int kWarpMMA = kWarpTMA + 1;
// 12 warps put 3 on each SM sub-partition, so the launch grants 168 registers a thread
// (3 x 32 x 168 <= 16384 per sub-partition).  The control warpgroup drops to 104 and the
// element-wise warpgroups rise to 200: 2 x 128 x 200 + 128 x 104 = 384 x 168.
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 104;
constexpr int kRegsEw = 200;
static_assert(kGroups * 128 * kRegsEw + 128 * kRegsControl <= kThreads * kRegsLaunch,
              "register split exceeds the launch pool");

// TMEM column of the k-th 16-wide K step of a bf16 operand written as two 32-column
// pieces at `base` and `base + 64` (one per element-wise group).
__device__ __forceinline__ uint32_t split_operand_col(uint32_t base, int kk) {
  return base + (kk / 4) * 64 + (kk % 4) * 8;
}
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
  unsigned int* err;
  const int* seqlens_q;  // [B] per-sequence query rows, or null (all Nq)
  const int* seqlens_k;  // [B] per-sequence key rows, or null (all Nk)
  const int* cu_q;       // packed layout: [B+1] first query token of each sequence, or null
  const int* cu_k;       // packed layout: [B+1] first key token of each sequence
  int total_q;           // packed layout: query tokens of all sequences
  int total_k;
  int H;
  __nv_bfloat16* dQ;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  const float* Dpad;   // [BH][Npad]: -D
  const float* L2pad;  // [BH][Npad]: -LSE * log2(e)
  int BH;
  int Nq;           // query rows per head (Q, O, dO, dQ, LSE); padded length with seqlens
  int Nk;           // key rows per head (K, V, dK, dV); padded length with seqlens
  int Npad;         // Nq rounded up to whole tiles
  int n_qt;         // ceil(Nq / 128)
  int n_kt;         // ceil(Nk / 128)
  int total_units;  // this kernel's units: BH * n_kt (dK/dV) or BH * n_qt (dQ)
  int causal;
  int dq_aligned32;  // dQ starts on a 32-byte boundary (its rows then allow 32-byte stores)
  float scale;
  float scale_log2;
};

// Head bh's sequence: its query and key row counts (Nq, Nk, or its entries of
// seqlens_q / seqlens_k, or the differences of cu_q / cu_k) and, in the packed layout,
// its first query and key tokens (0 otherwise).  A sequence out of range sets
// kErrBadLength and is skipped: (0, 0).
__device__ __forceinline__ void seq_info(const BwdArgs& a, int bh, int& lq, int& lk, int& tq0,
                                         int& tk0) {
  lq = a.Nq;
  lk = a.Nk;
  tq0 = 0;
  tk0 = 0;
  bool bad = false;
  if (a.cu_q != nullptr) {
    const int b = bh / a.H;
    tq0 = a.cu_q[b];
    tk0 = a.cu_k[b];
    lq = a.cu_q[b + 1] - tq0;
    lk = a.cu_k[b + 1] - tk0;
    bad = tq0 < 0 || tq0 + lq > a.total_q || tk0 < 0 || tk0 + lk > a.total_k;
  } else if (a.seqlens_q != nullptr) {
    const int b = bh / a.H;
    lq = a.seqlens_q[b];
    lk = a.seqlens_k[b];
  } else {
    return;
  }
  if (bad || lq < 0 || lq > a.Nq || lk < 0 || lk > a.Nk || (a.causal && lq > lk)) {
    atomicOr(a.err, kErrBadLength);
    lq = 0;
    lk = 0;
  }
}

// Element offset of row `row` of head bh in a query-side ([BH][Nq][d] or packed
// [tokens][H][d]) tensor, t0 the sequence's first token in the packed layout.
__device__ __forceinline__ size_t q_row_offset(const BwdArgs& a, int bh, int t0, int row,
                                               int D) {
  return a.cu_q != nullptr ? (static_cast<size_t>(t0 + row) * a.H + bh % a.H) * D
                           : (static_cast<size_t>(bh) * a.Nq + row) * D;
}
__device__ __forceinline__ size_t k_row_offset(const BwdArgs& a, int bh, int t0, int row,
                                               int D) {
  return a.cu_q != nullptr ? (static_cast<size_t>(t0 + row) * a.H + bh % a.H) * D
                           : (static_cast<size_t>(bh) * a.Nk + row) * D;
}
// Index of row `row` of head bh in LSE ([BH][Nq], or [H][total_q] when packed).
__device__ __forceinline__ size_t lse_index(const BwdArgs& a, int bh, int t0, int row) {
  return a.cu_q != nullptr ? static_cast<size_t>(bh % a.H) * a.total_q + t0 + row
                           : static_cast<size_t>(bh) * a.Nq + row;
}

// ------------------------------------------------------------------ 1. preparation
// Stores the negated row statistics the element-wise steps add:
//   ND[bh][r] = -sum_k dO[bh][r][k] * O[bh][r][k],   NL2[bh][r] = -LSE[bh][r] * log2(e).
// Padded rows r in [N, Npad): ND = 0, NL2 = -inf (their probabilities are exactly 0).
// Bandwidth bound: each thread issues its 16-byte loads of O and dO for all of its
// kPrepRowsPerThread rows before using any (all in flight together), the D / 8 threads
// of a row combine their partial sums with shuffles, and a block's rows lie in one head
// (no per-row division).
constexpr int kPrepThreads = 256;
constexpr int kPrepRowsPerThread = 4;

template <int D>
__global__ void __launch_bounds__(kPrepThreads) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ LSE, float* __restrict__ Dout, float* __restrict__ L2out,
    const BwdArgs a) {
  const int Npad = a.Npad;
  constexpr int kPer = D / 8;                         // threads per row (8 bf16 each)
  constexpr int kRowsPerPass = kPrepThreads / kPer;   // rows covered by one pass
  constexpr int kRowsPerBlock = kRowsPerPass * kPrepRowsPerThread;
  static_assert(128 % kRowsPerBlock == 0, "a block's rows must lie in one head");
  const int part = threadIdx.x % kPer;
  // Npad is a multiple of 128, so a block's rows lie in one head
  const long long blk_row0 = static_cast<long long>(blockIdx.x) * kRowsPerBlock;
  const int bh = static_cast<int>(blk_row0 / Npad);
  if (bh >= a.BH) return;
  const int rb = static_cast<int>(blk_row0 - static_cast<long long>(bh) * Npad) + threadIdx.x / kPer;
  int lq, lk, tq0, tk0;
  seq_info(a, bh, lq, lk, tq0, tk0);
  // every load of the thread's rows first, so that they are all in flight together
  uint4 va[kPrepRowsPerThread], vb[kPrepRowsPerThread];
#pragma unroll
  for (int k = 0; k < kPrepRowsPerThread; ++k) {
    const int r = rb + k * kRowsPerPass;
    if (r < lq) {
      const size_t off = q_row_offset(a, bh, tq0, r, D) + part * 8;
      va[k] = *reinterpret_cast<const uint4*>(O + off);
      vb[k] = *reinterpret_cast<const uint4*>(dO + off);
    } else {
      va[k] = make_uint4(0u, 0u, 0u, 0u);
      vb[k] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int k = 0; k < kPrepRowsPerThread; ++k) {
    float acc = 0.f;
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&va[k]);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&vb[k]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(pa[e]);
      const float2 fb = __bfloat1622float2(pb[e]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
#pragma unroll
    for (int o = kPer / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const int r = rb + k * kRowsPerPass;
    if (part == 0) {
      const size_t row = static_cast<size_t>(bh) * Npad + r;
      Dout[row] = -acc;
      L2out[row] = r < lq ? -LSE[lse_index(a, bh, tq0, r)] * kLog2e : -INFINITY;
    }
  }
}

// Convert 32 fp32 accumulator columns (times `mul`) to bf16 and store them to a row.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t* v, float mul) {
  uint32_t pk[16];
#pragma unroll
  for (int k = 0; k < 16; ++k)
    pk[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * mul, __uint_as_float(v[2 * k + 1]) * mul);
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int k = 0; k < 4; ++k) d[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
}

// The same for 64 columns with 32-byte stores (dst 32-byte aligned).
__device__ __forceinline__ void store_row64_v8(__nv_bfloat16* dst, const uint32_t* v, float mul) {
  uint32_t pk[32];
#pragma unroll
  for (int k = 0; k < 32; ++k)
    pk[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * mul, __uint_as_float(v[2 * k + 1]) * mul);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 16 * k),
                 "r"(pk[8 * k]), "r"(pk[8 * k + 1]), "r"(pk[8 * k + 2]), "r"(pk[8 * k + 3]),
                 "r"(pk[8 * k + 4]), "r"(pk[8 * k + 5]), "r"(pk[8 * k + 6]), "r"(pk[8 * k + 7])
                 : "memory");
}

// ------------------------------------------------------------------ 2. dK, dV
template <int D>
struct DkdvLayout {
  // K_j and V_j stay for the whole unit.  Query tiles stream through two rings: Q_i
  // (2 slots; its last reader is the dK product) and dO_i together with the tile's
  // LSE*log2(e) and D rows (2 slots; read by dP^T, dV and the element-wise warps).
  // (A third Q slot measured no faster; its 32 KB hold the epilogue's staging boxes
  // instead: 4 KB per element-wise warp, through which dK and dV leave by bulk tensor
  // stores.)  At d = 128 the layout uses 226 KB of the 227 KB (232448 B) a CTA may have,
  // so it leaves no slack for aligning the base: the kernel checks that the dynamic
  // shared memory starts on a 1024-byte boundary (the 128-byte swizzle atoms need it)
  // and reports kErrSmemAlign instead of running if it does not.
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kBoxBytes = 128 * 128;
  // (d = 64 tiles are half the size: three slots in each ring there)
  static constexpr int kQStages = (D == 64) ? 3 : 2;
  static constexpr int kDOStages = (D == 64) ? 3 : 2;
  static constexpr int kK = 0;
  static constexpr int kV = kTileBytes;
  static constexpr int kQ0 = 2 * kTileBytes;
  static constexpr int kDO0 = kQ0 + kQStages * kTileBytes;
  static constexpr int kDOSlotBytes = kTileBytes + 1024;  // dO tile, L2 row, D row
  static constexpr int kSlotL = kTileBytes;
  static constexpr int kSlotD = kTileBytes + 512;
  static constexpr int kOst = kDO0 + kDOStages * kDOSlotBytes;  // [kEw / 32] x 4 KB
  static constexpr int kBar = kOst + (kEw / 32) * 4096;
  static constexpr int kBarKVFull = 0, kBarKVEmpty = 1;
  static constexpr int kBarQFull = 2;                            // [kQStages]
  static constexpr int kBarQEmpty = kBarQFull + kQStages;        // [kQStages]
  static constexpr int kBarDOFull = kBarQEmpty + kQStages;       // [kDOStages]
  static constexpr int kBarDOEmpty = kBarDOFull + kDOStages;     // [kDOStages]
  static constexpr int kBarSFull = kBarDOEmpty + kDOStages;
  static constexpr int kBarDPFull = kBarSFull + 1;
  static constexpr int kBarPReady = kBarSFull + 2;
  static constexpr int kBarDSReady = kBarSFull + 3;
  static constexpr int kBarAccFull = kBarSFull + 4;
  static constexpr int kBarAccFree = kBarSFull + 5;
  static constexpr int kBarDrain = kBarSFull + 6;
  static constexpr int kBarPReadyB = kBarSFull + 7;  // second half of each group's P^T
  static constexpr int kNumBars = kBarPReadyB + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kAlloc = kMisc + 16;
  static_assert(kAlloc <= 232448, "shared memory over the 227 KB per-block limit");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmL2, const __grid_constant__ CUtensorMap tmD,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const BwdArgs args) {
  using L = DkdvLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {  // see DkdvLayout: the layout has no room to realign
    if (threadIdx.x == 0) atomicOr(args.err, kErrSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  // a wait for a whole converged warp: every lane gets the same answer
  auto wait_warp = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, args.err));
  };
  // TMA coordinates of row `row` of head bh's queries (t0 = tq0) or keys (t0 = tk0):
  // (row, head) in the [BH][N][d] maps, (head, first token + row) in the packed maps
  const bool packed = args.cu_q != nullptr;
  auto tma_y = [&](int bh, int row) { return packed ? bh % args.H : row; };
  auto tma_z = [&](int bh, int t0, int row) { return packed ? t0 + row : bh; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::kBarKVFull), 1);
    mbar_init(bar(L::kBarKVEmpty), 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar(L::kBarQFull + s), 1);
      mbar_init(bar(L::kBarQEmpty + s), 1);
    }
    for (int s = 0; s < L::kDOStages; ++s) {
      mbar_init(bar(L::kBarDOFull + s), 1);
      mbar_init(bar(L::kBarDOEmpty + s), 1 + kEw / 32);  // MMA commit + element-wise warps
    }
    mbar_init(bar(L::kBarSFull), 1);
    mbar_init(bar(L::kBarDPFull), 1);
    mbar_init(bar(L::kBarPReady), kEw / 32);
    mbar_init(bar(L::kBarPReadyB), kEw / 32);
    mbar_init(bar(L::kBarDSReady), kEw / 32);
    mbar_init(bar(L::kBarAccFull), 1);
    mbar_init(bar(L::kBarAccFree), kEw / 32);
    mbar_init(bar(L::kBarDrain), 1);
    fence_mbar_init();
  }
  if (warp == kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tdV = tmem, tdK = tmem + D, tS = tmem + 2 * D, tdP = tmem + 2 * D + 128;

  // unit w: key tile j of head bh, meeting query tiles i0 .. i0 + m - 1 of its sequence
  // (m = 0: the tile lies past the sequence's keys, or the sequence has no queries)
  auto unit = [&](int w, int& bh, int& j, int& i0, int& m, int& lk, int& off, int& tq0,
                  int& tk0, int& lq) {
    if (args.causal) {
      j = w / args.BH;  // key tile 0 meets every query tile: heaviest first
      bh = w % args.BH;
    } else {
      bh = w / args.n_kt;
      j = w % args.n_kt;
    }
    seq_info(args, bh, lq, lk, tq0, tk0);
    off = lk - lq;  // position of query row 0 among the keys
    i0 = 0;
    if (j * kTile >= lk || lq == 0) {
      m = 0;
      return;
    }
    // causal: first query tile with a row whose position reaches key j*128
    if (args.causal && j * kTile > off) i0 = (j * kTile - off) / kTile;
    m = (lq + kTile - 1) / kTile - i0;
  };
  auto qslot = [&](int s) -> uint32_t { return base + L::kQ0 + s * L::kTileBytes; };
  auto doslot = [&](int s) -> uint32_t { return base + L::kDO0 + s * L::kDOSlotBytes; };

  if (warp >= kWarpTMA) regs_dec<kRegsControl>();
  if (warp == kWarpTMA) {
    // the whole warp runs the loop; one elected lane issues each copy
    int qs = 0, ds = 0, units = 0, kv_loads = 0;
    uint32_t qph = 0, dph = 0;
    int q_issued[L::kQStages] = {}, d_issued[L::kDOStages] = {};
    uint32_t q_phase[L::kQStages] = {}, d_phase[L::kDOStages] = {};
    bool ok = true;
    int live = 0;  // 1 when the unit just processed had work: units counts only those
    for (int r = 0, w = snake_unit(0); ok && w < args.total_units;
         w = snake_unit(++r), units += live) {
      int bh, j, i0, m, lk, off, tq0, tk0, lq;
      unit(w, bh, j, i0, m, lk, off, tq0, tk0, lq);
      live = m > 0;
      if (!live) continue;
      if (units > 0) ok = wait_warp(bar(L::kBarKVEmpty), (units - 1) & 1);
      if (!ok) break;
      mbar_arrive_expect_tx_elect(bar(L::kBarKVFull), 2 * L::kTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d_elect(base + L::kK + c * L::kBoxBytes, &tmK, bar(L::kBarKVFull), c * 64,
                          tma_y(bh, j * kTile), tma_z(bh, tk0, j * kTile));
        tma_load_3d_elect(base + L::kV + c * L::kBoxBytes, &tmV, bar(L::kBarKVFull), c * 64,
                          tma_y(bh, j * kTile), tma_z(bh, tk0, j * kTile));
      }
      ++kv_loads;
      for (int i = i0; ok && i < i0 + m; ++i) {
        ok = wait_warp(bar(L::kBarQEmpty + qs), qph ^ 1);
        if (!ok) break;
        mbar_arrive_expect_tx_elect(bar(L::kBarQFull + qs), L::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d_elect(qslot(qs) + c * L::kBoxBytes, &tmQ, bar(L::kBarQFull + qs), c * 64,
                            tma_y(bh, i * kTile), tma_z(bh, tq0, i * kTile));
        q_issued[qs] = 1;
        q_phase[qs] = qph;
        if (++qs == L::kQStages) qs = 0, qph ^= 1;
        ok = wait_warp(bar(L::kBarDOEmpty + ds), dph ^ 1);
        if (!ok) break;
        const uint32_t fb = bar(L::kBarDOFull + ds);
        mbar_arrive_expect_tx_elect(fb, L::kTileBytes + 1024);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d_elect(doslot(ds) + c * L::kBoxBytes, &tmdO, fb, c * 64,
                            tma_y(bh, i * kTile), tma_z(bh, tq0, i * kTile));
        tma_load_3d_elect(doslot(ds) + L::kSlotL, &tmL2, fb, i * kTile, bh, 0);
        tma_load_3d_elect(doslot(ds) + L::kSlotD, &tmD, fb, i * kTile, bh, 0);
        d_issued[ds] = 1;
        d_phase[ds] = dph;
        if (++ds == L::kDOStages) ds = 0, dph ^= 1;
      }
    }
    if (!ok) {
      // let the loads already issued land before the CTA exits
      for (int s = 0; s < L::kQStages; ++s)
        if (q_issued[s]) mbar_wait_drain(bar(L::kBarQFull + s), q_phase[s], args.err);
      for (int s = 0; s < L::kDOStages; ++s)
        if (d_issued[s]) mbar_wait_drain(bar(L::kBarDOFull + s), d_phase[s], args.err);
      if (kv_loads > 0) mbar_wait_drain(bar(L::kBarKVFull), (kv_loads - 1) & 1, args.err);
    }
  } else if (warp == kWarpMMA) {
    // the whole warp runs the loop so descriptors stay warp-uniform; one elected lane
    // issues each tcgen05 instruction
    constexpr uint32_t idSS = idesc_bf16_f32(kTile, false);
    constexpr uint32_t idTS = idesc_bf16_f32(D, true);
    const uint64_t dK0 = desc_kmajor(base + L::kK);
    const uint64_t dV0 = desc_kmajor(base + L::kV);
    int qc = 0, dc = 0, units = 0, p_cnt = 0, ds_cnt = 0;
    uint32_t qcph = 0, dcph = 0;
    bool ok = true;
    // S^T = K Q^T or dP^T = V dO^T: both operands K-major, K extent = D.  The K-step
    // loops are fully unrolled so that the single issuing thread keeps up with the
    // tensor pipe (64 cycles per 128 x 128 x 16 MMA).
    auto issue_ss = [&](uint32_t dtm, uint64_t da, uint32_t b_saddr, uint32_t done_bar) {
      const uint64_t db = desc_kmajor(b_saddr);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk / 4) * L::kBoxBytes + (kk % 4) * 32) >> 4;
        mma_ss_elect(dtm, da + off, db + off, idSS, kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(done_bar);
    };
    // acc += A(TMEM, 128 x 128 bf16) * B(smem tile, 128 rows x D, MN-major)
    auto issue_ts = [&](uint32_t acc, uint32_t a_tmem, uint32_t b_saddr, bool accumulate) {
      const uint64_t db = desc_mnmajor(b_saddr, L::kBoxBytes);
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        mma_ts_elect(acc, split_operand_col(a_tmem, kk), db + static_cast<uint64_t>((kk * 2048) >> 4),
                     idTS, (accumulate || kk > 0) ? 1u : 0u);
    };
    // the same product over the K steps whose 16 queries lie in half h of each group's
    // 64 columns (h = 0: K steps 0, 1, 4, 5; h = 1: 2, 3, 6, 7); half 0 comes first, so the
    // product's first K step, which starts the accumulation of a unit, is in it
    auto issue_ts_half = [&](uint32_t acc, uint32_t a_tmem, uint32_t b_saddr, bool accumulate,
                             int h) {
      const uint64_t db = desc_mnmajor(b_saddr, L::kBoxBytes);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = (q / 2) * 4 + h * 2 + (q % 2);
        mma_ts_elect(acc, split_operand_col(a_tmem, kk), db + static_cast<uint64_t>((kk * 2048) >> 4),
                     idTS, (accumulate || kk > 0) ? 1u : 0u);
      }
    };
    // S^T(next query tile) from the next Q slot
    auto next_s = [&](int& slot) -> bool {
      if (!wait_warp(bar(L::kBarQFull + qc), qcph)) return false;
      slot = qc;
      if (++qc == L::kQStages) qc = 0, qcph ^= 1;
      tc_fence_after();
      issue_ss(tS, dK0, qslot(slot), bar(L::kBarSFull));
      return true;
    };
    // dP^T(next query tile) from the next dO slot
    auto next_dp = [&](int& slot) -> bool {
      if (!wait_warp(bar(L::kBarDOFull + dc), dcph)) return false;
      slot = dc;
      if (++dc == L::kDOStages) dc = 0, dcph ^= 1;
      tc_fence_after();
      issue_ss(tdP, dV0, doslot(slot), bar(L::kBarDPFull));
      return true;
    };
    int live = 0;
    for (int r = 0, w = snake_unit(0); ok && w < args.total_units;
         w = snake_unit(++r), units += live) {
      int bh, j, i0, m, lk, off, tq0, tk0, lq;
      unit(w, bh, j, i0, m, lk, off, tq0, tk0, lq);
      live = m > 0;
      if (!live) continue;
      ok = wait_warp(bar(L::kBarKVFull), units & 1);
      int curq = 0, curd = 0;
      if (ok) ok = next_s(curq);
      if (ok) ok = next_dp(curd);
      if (!ok) break;
      // K_j and V_j are read only by the S^T and dP^T products: once the unit's last
      // dP^T is issued, their slot is released (when it completes) and the next unit's
      // K and V load while this unit's last dV and dK products and the element-wise work
      // still run, instead of after them
      if (m == 1) mma_commit_elect(bar(L::kBarKVEmpty));
      for (int t = 0; t < m; ++t) {
        ok = wait_warp(bar(L::kBarPReady), p_cnt & 1);
        if (ok && t == 0 && units > 0) ok = wait_warp(bar(L::kBarAccFree), (units - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        // dV += P^T dO over the first half of every group's queries while the
        // element-wise warps still compute the second half (the dV product reads P^T;
        // starting it early shortens the S^T -> exponentials -> dV -> next S^T loop that
        // paces the kernel), then over the second half
        issue_ts_half(tdV, tS, doslot(curd), t > 0, 0);
        ok = wait_warp(bar(L::kBarPReadyB), p_cnt & 1);
        if (!ok) break;
        tc_fence_after();
        issue_ts_half(tdV, tS, doslot(curd), t > 0, 1);
        ++p_cnt;
        mma_commit_elect(bar(L::kBarDOEmpty + curd));
        int nq = -1, nd = -1;
        if (t + 1 < m) {
          ok = next_s(nq);
          if (!ok) break;
        }
        ok = wait_warp(bar(L::kBarDSReady), ds_cnt & 1);
        if (!ok) break;
        ++ds_cnt;
        tc_fence_after();
        issue_ts(tdK, tdP, qslot(curq), t > 0);  // dK += dS^T Q
        mma_commit_elect(bar(L::kBarQEmpty + curq));
        if (t + 1 < m) {
          ok = next_dp(nd);
          if (!ok) break;
          if (t + 2 == m) mma_commit_elect(bar(L::kBarKVEmpty));
          curq = nq;
          curd = nd;
        }
      }
      if (!ok) break;
      mma_commit_elect(bar(L::kBarAccFull));
    }
    mma_commit_elect(bar(L::kBarDrain));
    mbar_wait_drain(bar(L::kBarDrain), 0, args.err);
  } else if (warp < kWarpTMA) {
    regs_inc<kRegsEw>();
    const int g = warp / 4;            // column group
    const int col0 = g * kCols;        // first tile column of this group
    const int row = (warp % 4) * 32 + lane;  // key row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    int stage = 0, units = 0, s_cnt = 0, dp_cnt = 0;
    bool st_used = false;  // this warp's staging box has been handed to a bulk store
    uint32_t phase = 0;
    bool ok = true;
    int live = 0;
    for (int r = 0, w = snake_unit(0); ok && w < args.total_units;
         w = snake_unit(++r), units += live) {
      int bh, j, i0, m, lk, off, tq0, tk0, lq;
      unit(w, bh, j, i0, m, lk, off, tq0, tk0, lq);
      live = m > 0;
      if (!live) {
        // a sequence with keys but no queries: no query sees these keys, so their
        // gradients are exactly zero (group g writes its half of each row)
        const int kv_row = j * kTile + row;
        if (lq == 0 && kv_row < lk) {
          const size_t orow = k_row_offset(args, bh, tk0, kv_row, D) + g * (D / 2);
          uint4* zk = reinterpret_cast<uint4*>(args.dK + orow);
          uint4* zv = reinterpret_cast<uint4*>(args.dV + orow);
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            zk[c] = make_uint4(0u, 0u, 0u, 0u);
            zv[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        continue;
      }
      for (int i = i0; i < i0 + m; ++i) {
        // this tile's L2 and D rows sit in its dO slot
        const uint8_t* sb = smem + L::kDO0 + stage * L::kDOSlotBytes;
        const float* sL = reinterpret_cast<const float*>(sb + L::kSlotL) + col0;
        const float* sD = reinterpret_cast<const float*>(sb + L::kSlotD) + col0;
        ok = wait_warp(bar(L::kBarDOFull + stage), phase);
        if (ok) ok = wait_warp(bar(L::kBarSFull), s_cnt & 1);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        float p[kCols];
        {
          uint32_t r[kCols];
#pragma unroll
          for (int c = 0; c < kCols / 32; ++c)
            tmem_ld32(tS + lane_off + col0 + c * 32, &r[c * 32]);
          tmem_wait_ld();
          // causal: key j*128+row is hidden from query i*128+col when col < row + delta
          const int delta = (j - i) * kTile - off;
          const bool diag = args.causal && delta > -kTile;
          const uint64_t scale2 = f32x2(args.scale_log2, args.scale_log2);
          // the group's 64 columns in two halves of 32; each half's bf16 P^T is stored and
          // announced as soon as it is made
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
            for (int c = hf * (kCols / 2); c < (hf + 1) * (kCols / 2); c += 2) {
              // x = S^T * scale * log2e - L2 for two query columns in one packed FMA
              const uint64_t nl = *reinterpret_cast<const uint64_t*>(sL + c);
              const uint64_t x2 =
                  fma_x2(f32x2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), scale2, nl);
              float e0, e1;
              exp2_pair(x2, e0, e1);
              if (diag && col0 + c < row + delta) e0 = 0.f;
              if (diag && col0 + c + 1 < row + delta) e1 = 0.f;
              p[c] = e0;
              p[c + 1] = e1;
            }
            uint32_t pk[kCols / 4];
#pragma unroll
            for (int c = 0; c < kCols / 4; ++c)
              pk[c] = pack_bf16x2(p[hf * (kCols / 2) + 2 * c], p[hf * (kCols / 2) + 2 * c + 1]);
            tmem_st16(tS + lane_off + col0 + hf * (kCols / 4), pk);
            tmem_wait_st();
            warp_arrive(bar(hf == 0 ? L::kBarPReady : L::kBarPReadyB));
          }
        }
        ok = wait_warp(bar(L::kBarDPFull), dp_cnt & 1);
        if (!ok) break;
        ++dp_cnt;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tdP + lane_off + col0 + c * 32, r);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            // dS = P (dP - D) for two query columns: one packed add, one packed multiply
            const int c0 = c * 32 + 2 * k;
            const uint64_t nd = *reinterpret_cast<const uint64_t*>(sD + c0);
            float ds0, ds1;
            f32x2_split(mul_x2(f32x2(p[c0], p[c0 + 1]),
                               add_x2(f32x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), nd)),
                        ds0, ds1);
            pk[k] = pack_bf16x2(ds0, ds1);
          }
          // dS for columns c*32.. lands on columns this group has already read
          tmem_st16(tdP + lane_off + col0 + c * 16, pk);
        }
        tmem_wait_st();
        warp_arrive(bar(L::kBarDSReady));
        if (lane == 0) mbar_arrive(bar(L::kBarDOEmpty + stage));  // done with its L2, D rows
        if (++stage == L::kDOStages) stage = 0, phase ^= 1;
      }
      if (!ok) break;
      // epilogue: group 0 writes dV, group 1 scale * dK, each warp its 32 key rows.  A
      // warp whose rows all lie inside the sequence puts them, 64 columns at a time, into
      // its staging box in the 128-byte-swizzled layout (row r's 16-byte chunk k at
      // r * 128 + ((k ^ (r % 8)) * 16): 32 rows cover the 32 banks four times over) and
      // its lane 0 writes the box out with a bulk tensor store, whole lines at a time;
      // otherwise the valid rows are stored one per lane.
      ok = wait_warp(bar(L::kBarAccFull), units & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = g == 0 ? tdV : tdK;
      const float mul = g == 0 ? 1.f : args.scale;
      const int r0 = j * kTile + (warp % 4) * 32;  // the warp's first key row
      const bool whole = r0 + 32 <= lk;
      const uint32_t stg_a = base + L::kOst + warp * 4096;
      uint8_t* stg = smem + L::kOst + warp * 4096;
      __nv_bfloat16* grad = g == 0 ? args.dV : args.dK;
      const size_t orow = k_row_offset(args, bh, tk0, j * kTile + row, D);
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[64];
        tmem_ld32(tacc + lane_off + c * 64, v);
        tmem_ld32(tacc + lane_off + c * 64 + 32, v + 32);
        tmem_wait_ld();
        // the accumulators may be zeroed by the next unit once every warp has read them
        if (c == D / 64 - 1) warp_arrive(bar(L::kBarAccFree));
        if (whole) {
          if (st_used) {
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t* v8 = &v[8 * k];
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((k ^ (lane & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(v8[0]) * mul, __uint_as_float(v8[1]) * mul),
                pack_bf16x2(__uint_as_float(v8[2]) * mul, __uint_as_float(v8[3]) * mul),
                pack_bf16x2(__uint_as_float(v8[4]) * mul, __uint_as_float(v8[5]) * mul),
                pack_bf16x2(__uint_as_float(v8[6]) * mul, __uint_as_float(v8[7]) * mul));
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(g == 0 ? &tmdV : &tmdK, stg_a, c * 64, tma_y(bh, r0), tma_z(bh, tk0, r0));
            bulk_commit_group();
          }
          st_used = true;
        } else if (j * kTile + row < lk) {
          store_row32(grad + orow + c * 64, v, mul);
          store_row32(grad + orow + c * 64 + 32, v + 32, mul);
        }
      }
    }
    // the bulk stores this thread issued have completed before the CTA (and its shared
    // memory) goes away
    if (lane == 0) bulk_wait_group0();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ 3. dQ
template <int D>
struct DqLayout {
  // Q_i and dO_i arrive once per unit and are copied into tensor memory, where the S and
  // dP products read them (so those products read only K_j or V_j from shared memory);
  // their shared-memory slot is then free for the next unit's tiles.  K_j and V_j stream
  // through separate rings.
  // K_j is read until the dQ product of its tile, V_j only by the dP product, so K gets
  // one more slot: both are then loaded a tile and a half before they are needed.
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kTileBytes;
  static constexpr int kK0 = 2 * kTileBytes;
  static constexpr int kV0 = kK0 + kKStages * kTileBytes;
  static constexpr int kBar = kV0 + kVStages * kTileBytes;
  static constexpr int kBarQFull = 0, kBarQEmpty = 1;
  static constexpr int kBarKFull = 2;                          // [kKStages]
  static constexpr int kBarKEmpty = kBarKFull + kKStages;      // [kKStages]
  static constexpr int kBarVFull = kBarKEmpty + kKStages;      // [kVStages]
  static constexpr int kBarVEmpty = kBarVFull + kVStages;      // [kVStages]
  static constexpr int kBarSFull = kBarVEmpty + kVStages;
  static constexpr int kBarSFree = kBarSFull + 1;
  static constexpr int kBarDPFull = kBarSFull + 2;
  static constexpr int kBarDSReady = kBarSFull + 3;
  static constexpr int kBarAccFull = kBarSFull + 4;
  static constexpr int kBarAccFree = kBarSFull + 5;
  static constexpr int kBarDrain = kBarSFull + 6;
  static constexpr int kBarQTmem = kBarSFull + 7;   // this unit's Q, dO are in TMEM
  static constexpr int kNumBars = kBarQTmem + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "shared memory over the 227 KB per-block limit");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdArgs args) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    return mbar_wait(b, parity, abort_flag, args.err);
  };
  // the same for a whole converged warp: every lane gets the same answer
  auto wait_warp = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, args.err));
  };
  // TMA coordinates of row `row` of head bh's queries (t0 = tq0) or keys (t0 = tk0):
  // (row, head) in the [BH][N][d] maps, (head, first token + row) in the packed maps
  const bool packed = args.cu_q != nullptr;
  auto tma_y = [&](int bh, int row) { return packed ? bh % args.H : row; };
  auto tma_z = [&](int bh, int t0, int row) { return packed ? t0 + row : bh; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::kBarQFull), 1);
    mbar_init(bar(L::kBarQEmpty), kEw / 32);  // the element-wise warps, once copied
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    mbar_init(bar(L::kBarSFull), 1);
    mbar_init(bar(L::kBarSFree), kEw / 32);
    mbar_init(bar(L::kBarDPFull), 1);
    mbar_init(bar(L::kBarDSReady), kEw / 32);
    mbar_init(bar(L::kBarAccFull), 1);
    mbar_init(bar(L::kBarAccFree), kEw / 32);
    mbar_init(bar(L::kBarDrain), 1);
    mbar_init(bar(L::kBarQTmem), kEw / 32);
    fence_mbar_init();
  }
  if (warp == kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // dQ | S | dP (dS written over the columns each group has read, as bf16) | Q | dO.
  // Q and dO (bf16, one 32-bit column per pair of elements) are the A operands of the
  // S and dP products for the whole unit.
  const uint32_t tdQ = tmem, tS = tmem + 128, tdP = tmem + 256, tQt = tmem + 384,
                 tdOt = tmem + 384 + D / 2;

  // unit w: query tile i of head bh, meeting key tiles 0 .. m - 1 of its sequence
  // (m = 0: the tile lies past the sequence's queries, or the sequence has no keys)
  auto unit = [&](int w, int& bh, int& i, int& m, int& lq, int& lk, int& off, int& tq0,
                  int& tk0) {
    if (args.causal) {
      i = args.n_qt - 1 - w / args.BH;  // last query tile meets the most key tiles
      bh = w % args.BH;
    } else {
      bh = w / args.n_qt;
      i = w % args.n_qt;
    }
    seq_info(args, bh, lq, lk, tq0, tk0);
    off = lk - lq;
    if (i * kTile >= lq || lk == 0) {
      m = 0;
      return;
    }
    const int n_kv = (lk + kTile - 1) / kTile;
    // causal: key tiles up to the one holding the position of the tile's last row
    m = args.causal ? min((i * kTile + kTile - 1 + off) / kTile + 1, n_kv) : n_kv;
  };

  if (warp >= kWarpTMA) regs_dec<kRegsControl>();
  if (warp == kWarpTMA) {
    // the whole warp runs the loop; one elected lane issues each copy
    {
      int ks = 0, vs = 0, units = 0, q_loads = 0;
      uint32_t kph = 0, vph = 0;
      int k_issued[L::kKStages] = {}, v_issued[L::kVStages] = {};
      uint32_t k_phase[L::kKStages] = {}, v_phase[L::kVStages] = {};
      bool ok = true;
      int live = 0;  // 1 when the unit just processed had work: units counts only those
      for (int r = 0, w = snake_unit(0); ok && w < args.total_units;
         w = snake_unit(++r), units += live) {
        int bh, i, m, lq, lk, off, tq0, tk0;
        unit(w, bh, i, m, lq, lk, off, tq0, tk0);
        live = m > 0;
        if (!live) continue;
        if (units > 0) ok = wait_warp(bar(L::kBarQEmpty), (units - 1) & 1);
        if (!ok) break;
        mbar_arrive_expect_tx_elect(bar(L::kBarQFull), 2 * L::kTileBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d_elect(base + L::kQ + c * L::kBoxBytes, &tmQ, bar(L::kBarQFull), c * 64,
                            tma_y(bh, i * kTile), tma_z(bh, tq0, i * kTile));
          tma_load_3d_elect(base + L::kDO + c * L::kBoxBytes, &tmdO, bar(L::kBarQFull), c * 64,
                            tma_y(bh, i * kTile), tma_z(bh, tq0, i * kTile));
        }
        ++q_loads;
        for (int j = 0; ok && j < m; ++j) {
          ok = wait_warp(bar(L::kBarKEmpty + ks), kph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx_elect(bar(L::kBarKFull + ks), L::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d_elect(base + L::kK0 + ks * L::kTileBytes + c * L::kBoxBytes, &tmK,
                              bar(L::kBarKFull + ks), c * 64, tma_y(bh, j * kTile),
                              tma_z(bh, tk0, j * kTile));
          k_issued[ks] = 1;
          k_phase[ks] = kph;
          if (++ks == L::kKStages) ks = 0, kph ^= 1;
          ok = wait_warp(bar(L::kBarVEmpty + vs), vph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx_elect(bar(L::kBarVFull + vs), L::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d_elect(base + L::kV0 + vs * L::kTileBytes + c * L::kBoxBytes, &tmV,
                              bar(L::kBarVFull + vs), c * 64, tma_y(bh, j * kTile),
                              tma_z(bh, tk0, j * kTile));
          v_issued[vs] = 1;
          v_phase[vs] = vph;
          if (++vs == L::kVStages) vs = 0, vph ^= 1;
        }
      }
      if (!ok) {
        // let the loads already issued land before the CTA exits
        for (int s = 0; s < L::kKStages; ++s)
          if (k_issued[s]) mbar_wait_drain(bar(L::kBarKFull + s), k_phase[s], args.err);
        for (int s = 0; s < L::kVStages; ++s)
          if (v_issued[s]) mbar_wait_drain(bar(L::kBarVFull + s), v_phase[s], args.err);
        if (q_loads > 0) mbar_wait_drain(bar(L::kBarQFull), (q_loads - 1) & 1, args.err);
      }
    }
  } else if (warp == kWarpMMA) {
    // the whole warp runs the loop so descriptors stay warp-uniform; one elected lane
    // issues each tcgen05 instruction
    {
      constexpr uint32_t idS = idesc_bf16_f32(kTile, false);  // B K-major, N = 128 keys
      constexpr uint32_t idTS = idesc_bf16_f32(D, true);
      int kc = 0, vc = 0, units = 0, sfree_cnt = 0, ds_cnt = 0;
      uint32_t kcph = 0, vcph = 0;
      bool ok = true;
      auto kslot = [&](int s) { return base + L::kK0 + s * L::kTileBytes; };
      auto vslot = [&](int s) { return base + L::kV0 + s * L::kTileBytes; };
      // S = Q K^T or dP = dO V^T: A (this unit's Q or dO, K extent = D) from tensor
      // memory, B (K_j or V_j) K-major from shared memory
      auto issue_qk = [&](uint32_t dtm, uint32_t a_tmem, uint32_t b_saddr, uint32_t done_bar) {
        const uint64_t db = desc_kmajor(b_saddr);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * L::kBoxBytes + (kk % 4) * 32) >> 4;
          mma_ts_elect(dtm, a_tmem + kk * 8, db + off, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_elect(done_bar);
      };
      // dP = dO V^T into TMEM, then release V's slot once that product completes
      auto issue_dp = [&]() -> bool {
        if (!wait_warp(bar(L::kBarVFull + vc), vcph)) return false;
        tc_fence_after();
        issue_qk(tdP, tdOt, vslot(vc), bar(L::kBarDPFull));
        mma_commit_elect(bar(L::kBarVEmpty + vc));
        if (++vc == L::kVStages) vc = 0, vcph ^= 1;
        return true;
      };
      int live = 0;
      for (int r = 0, w = snake_unit(0); ok && w < args.total_units;
         w = snake_unit(++r), units += live) {
        int bh, i, m, lq, lk, off, tq0, tk0;
        unit(w, bh, i, m, lq, lk, off, tq0, tk0);
        live = m > 0;
        if (!live) continue;
        ok = wait_warp(bar(L::kBarQTmem), units & 1);
        if (ok) ok = wait_warp(bar(L::kBarKFull + kc), kcph);
        if (!ok) break;
        tc_fence_after();
        int cur = kc;
        if (++kc == L::kKStages) kc = 0, kcph ^= 1;
        issue_qk(tS, tQt, kslot(cur), bar(L::kBarSFull));
        ok = issue_dp();
        if (!ok) break;
        // per tile t: S(t+1) | dQ(t) | dP(t+1).  dS(t) lies over the dP region, so dP(t+1)
        // is issued after the dQ(t) product that reads it (the tensor pipe executes
        // products in issue order).
        for (int t = 0; t < m; ++t) {
          int nxt = -1;
          if (t + 1 < m) {
            // S(t+1) once the element-wise warps hold S(t) in registers
            ok = wait_warp(bar(L::kBarKFull + kc), kcph);
            if (ok) ok = wait_warp(bar(L::kBarSFree), sfree_cnt & 1);
            if (!ok) break;
            ++sfree_cnt;
            nxt = kc;
            if (++kc == L::kKStages) kc = 0, kcph ^= 1;
            tc_fence_after();
            issue_qk(tS, tQt, kslot(nxt), bar(L::kBarSFull));
          }
          ok = wait_warp(bar(L::kBarDSReady), ds_cnt & 1);
          if (ok && t == 0 && units > 0) ok = wait_warp(bar(L::kBarAccFree), (units - 1) & 1);
          if (!ok) break;
          ++ds_cnt;
          tc_fence_after();
          // dQ += dS K_j: A = dS (TMEM), B = K_j (128 key rows x D, MN-major)
          const uint64_t db = desc_mnmajor(kslot(cur), L::kBoxBytes);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts_elect(tdQ, split_operand_col(tdP, kk), db + static_cast<uint64_t>((kk * 2048) >> 4),
                         idTS, (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit_elect(bar(L::kBarKEmpty + cur));
          if (t + 1 < m) {
            ok = issue_dp();
            if (!ok) break;
          }
          if (nxt >= 0) cur = nxt;
        }
        if (!ok) break;
        // the unit's last S tile was read by the element-wise warps: consume that signal
        // before the next unit overwrites the region
        ok = wait_warp(bar(L::kBarSFree), sfree_cnt & 1);
        if (!ok) break;
        ++sfree_cnt;
        mma_commit_elect(bar(L::kBarAccFull));
      }
      mma_commit_elect(bar(L::kBarDrain));
      mbar_wait_drain(bar(L::kBarDrain), 0, args.err);
    }
  } else if (warp < kWarpTMA) {
    regs_inc<kRegsEw>();
    const int g = warp / 4;            // column group
    const int col0 = g * kCols;        // first tile column (key) of this group
    const int row = (warp % 4) * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    int units = 0, s_cnt = 0, dp_cnt = 0;
    bool ok = true;
    int live = 0;
    for (int r = 0, w = snake_unit(0); ok && w < args.total_units;
         w = snake_unit(++r), units += live) {
      int bh, i, m, lq, lk, off, tq0, tk0;
      unit(w, bh, i, m, lq, lk, off, tq0, tk0);
      live = m > 0;
      if (!live) continue;
      // This unit's Q and dO rows into tensor memory: thread = query row = TMEM lane;
      // group g copies the d-columns [g*D/2, (g+1)*D/2), one 32-bit column per pair of
      // bf16 elements.  The tiles sit in shared memory as 64-column boxes with the
      // 128-byte swizzle (16-byte chunk c of row r stored at chunk c ^ (r % 8)).  Every
      // product of the previous unit has completed (its dQ accumulator was drained), so
      // nothing still reads these TMEM columns.
      ok = wait_warp(bar(L::kBarQFull), units & 1);
      if (!ok) break;
      {
        constexpr int kChunks = D / 16;  // 16-byte chunks per group
        uint32_t vq[D / 4], vo[D / 4];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const int J = g * kChunks + c;  // chunk of the whole row
          const uint32_t at = (J / 8) * L::kBoxBytes + row * 128 + (((J % 8) ^ (row & 7)) * 16);
          const uint4 a = *reinterpret_cast<const uint4*>(smem + L::kQ + at);
          const uint4 b = *reinterpret_cast<const uint4*>(smem + L::kDO + at);
          vq[4 * c] = a.x, vq[4 * c + 1] = a.y, vq[4 * c + 2] = a.z, vq[4 * c + 3] = a.w;
          vo[4 * c] = b.x, vo[4 * c + 1] = b.y, vo[4 * c + 2] = b.z, vo[4 * c + 3] = b.w;
        }
        if constexpr (D == 128) {
          tmem_st32(tQt + lane_off + g * 32, vq);
          tmem_st32(tdOt + lane_off + g * 32, vo);
        } else {
          tmem_st16(tQt + lane_off + g * 16, vq);
          tmem_st16(tdOt + lane_off + g * 16, vo);
        }
        tmem_wait_st();
      }
      warp_arrive(bar(L::kBarQTmem));   // the S and dP products may read them
      warp_arrive(bar(L::kBarQEmpty));  // the next unit's tiles may be loaded
      const int q_row = i * kTile + row;
      const size_t prow = static_cast<size_t>(bh) * args.Npad + q_row;  // q_row < Npad
      const float nl2row = args.L2pad[prow];   // -LSE * log2(e) of this query row
      const float ndrow = args.Dpad[prow];     // -D of this query row
      for (int j = 0; j < m; ++j) {
        ok = wait_warp(bar(L::kBarSFull), s_cnt & 1);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        float p[kCols];
        {
          uint32_t r[kCols];
#pragma unroll
          for (int c = 0; c < kCols / 32; ++c)
            tmem_ld32(tS + lane_off + col0 + c * 32, &r[c * 32]);
          tmem_wait_ld();
          warp_arrive(bar(L::kBarSFree));
          const int kv0 = j * kTile + col0;
          // a ragged last key tile, or (causal) keys past the position of the tile's
          // first row
          const bool need_mask = (kv0 + kCols > lk) ||
                                 (args.causal && kv0 + kCols - 1 > i * kTile + off);
          const int lim = args.causal ? min(lk, q_row + off + 1) : lk;
          const uint64_t scale2 = f32x2(args.scale_log2, args.scale_log2);
          const uint64_t nl2 = f32x2(nl2row, nl2row);
#pragma unroll
          for (int c = 0; c < kCols; c += 2) {
            const uint64_t x2 =
                fma_x2(f32x2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), scale2, nl2);
            float e0, e1;
            exp2_pair(x2, e0, e1);
            if (need_mask && kv0 + c >= lim) e0 = 0.f;
            if (need_mask && kv0 + c + 1 >= lim) e1 = 0.f;
            p[c] = e0;
            p[c + 1] = e1;
          }
        }
        ok = wait_warp(bar(L::kBarDPFull), dp_cnt & 1);
        if (!ok) break;
        ++dp_cnt;
        tc_fence_after();
        uint32_t dpv[kCols];
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(tdP + lane_off + col0 + c * 32, &dpv[c * 32]);
        tmem_wait_ld();
        uint32_t pk[kCols / 2];
        const uint64_t nd2 = f32x2(ndrow, ndrow);
#pragma unroll
        for (int k = 0; k < kCols / 2; ++k) {
          // dS = P (dP - D), two key columns per packed add and multiply
          float ds0, ds1;
          f32x2_split(mul_x2(f32x2(p[2 * k], p[2 * k + 1]),
                             add_x2(f32x2(__uint_as_float(dpv[2 * k]), __uint_as_float(dpv[2 * k + 1])), nd2)),
                      ds0, ds1);
          pk[k] = pack_bf16x2(ds0, ds1);
        }
        // this group's 32-column piece of dS, over dP columns it has just read
        tmem_st32(tdP + lane_off + col0, pk);
        tmem_wait_st();
        warp_arrive(bar(L::kBarDSReady));
      }
      if (!ok) break;
      ok = wait_warp(bar(L::kBarAccFull), units & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const size_t orow = q_row_offset(args, bh, tq0, q_row, D) + g * (D / 2);
      // this group's half of the row: read whole, release the accumulator (the next
      // unit's first dQ product may start), then store it, 32 bytes per store where dQ
      // is aligned for that (half as many store instructions, each still touching a
      // line per row)
      uint32_t v[D / 2];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tmem_ld32(tdQ + lane_off + g * (D / 2) + c * 32, v + c * 32);
      tmem_wait_ld();
      warp_arrive(bar(L::kBarAccFree));
      if (q_row < lq) {
        if (D == 128 && args.dq_aligned32) {
          store_row64_v8(args.dQ + orow, v, args.scale);
        } else {
#pragma unroll
          for (int c = 0; c < D / 64; ++c) store_row32(args.dQ + orow + c * 32, v + c * 32, args.scale);
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
template <int D>
cudaError_t launch_d(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                     const CUtensorMap& tmdO, const CUtensorMap& tmL2, const CUtensorMap& tmD,
                     const CUtensorMap& tmdK, const CUtensorMap& tmdV, const void* O, const void* dO, const float* LSE, void* dQ, void* dK,
                     void* dV, float* ws, const Problem& p, int num_sms, cudaStream_t stream) {
  BwdArgs a;
  a.err = p.err;
  a.dQ = static_cast<__nv_bfloat16*>(dQ);
  a.dK = static_cast<__nv_bfloat16*>(dK);
  a.dV = static_cast<__nv_bfloat16*>(dV);
  a.BH = p.BH;
  a.seqlens_q = p.seqlens_q;
  a.seqlens_k = p.seqlens_k;
  a.cu_q = p.cu_q;
  a.cu_k = p.cu_k;
  a.total_q = p.total_q;
  a.total_k = p.total_k;
  a.H = p.H;
  a.Nq = p.N;
  a.Nk = p.Nk;
  a.n_qt = (p.N + kTile - 1) / kTile;
  a.n_kt = (p.Nk + kTile - 1) / kTile;
  a.Npad = a.n_qt * kTile;
  a.causal = p.causal;
  a.dq_aligned32 = (reinterpret_cast<uintptr_t>(dQ) & 31u) == 0;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  float* Dpad = ws;
  float* L2pad = ws + static_cast<size_t>(p.BH) * a.Npad;
  a.Dpad = Dpad;
  a.L2pad = L2pad;

  const long long rows = static_cast<long long>(p.BH) * a.Npad;
  const long long rows_per_block = static_cast<long long>(kPrepThreads / (D / 8)) * kPrepRowsPerThread;
  cudaError_t e = trace_mark(p, 0, stream);
  if (e != cudaSuccess) return e;
  bwd_prep_kernel<D><<<static_cast<unsigned>((rows + rows_per_block - 1) / rows_per_block),
                       kPrepThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), LSE, Dpad,
      L2pad, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = trace_mark(p, 1, stream)) != cudaSuccess) return e;

  BwdArgs a_kv = a, a_q = a;
  a_kv.total_units = p.BH * a.n_kt;
  a_q.total_units = p.BH * a.n_qt;
  const int grid_kv = a_kv.total_units < num_sms ? a_kv.total_units : num_sms;
  const int grid_q = a_q.total_units < num_sms ? a_q.total_units : num_sms;
  // the in-kernel register split assumes exactly kRegsLaunch registers a thread at launch
  cudaFuncAttributes fattr;
  e = cudaFuncGetAttributes(&fattr, bwd_dkdv_kernel<D>);
  if (e != cudaSuccess) return e;
  if (fattr.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncGetAttributes(&fattr, bwd_dq_kernel<D>);
  if (e != cudaSuccess) return e;
  if (fattr.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           DkdvLayout<D>::kAlloc);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<grid_kv, kThreads, DkdvLayout<D>::kAlloc, stream>>>(
      tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV, a_kv);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = trace_mark(p, 2, stream)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           DqLayout<D>::kAlloc);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<grid_q, kThreads, DqLayout<D>::kAlloc, stream>>>(tmQ, tmK, tmV, tmdO, a_q);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_mark(p, 3, stream);
}

}  // namespace

long long bwd_padded_rows(long long N) { return (N + kTile - 1) / kTile * kTile; }

cudaError_t launch_bwd_sm100(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmdO,
                             const CUtensorMap& tmL2, const CUtensorMap& tmD,
                             const CUtensorMap& tmdK, const CUtensorMap& tmdV, const void* O,
                             const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                             float* workspace, const Problem& p, int num_sms,
                             cudaStream_t stream) {
  if (p.d == 64)
    return launch_d<64>(tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV, O, dO, LSE, dQ, dK, dV,
                        workspace, p, num_sms, stream);
  return launch_d<128>(tmQ, tmK, tmV, tmdO, tmL2, tmD, tmdK, tmdV, O, dO, LSE, dQ, dK, dV,
                       workspace, p, num_sms, stream);
}

}  // namespace fa

// fwd_sm100.cu -- forward attention on the sm_100a tensor cores.
//
// Method ("FlashAttention, simplified", "The trick"; "FlashAttention" page, "The
// bottleneck is memory, not multiplication" and "A concrete example: 10,000 tokens"):
// for a block of queries, walk the key/value blocks, form the 128 x 128 score tile on
// chip, keep a running row max m and running sum l, rescale the accumulated output when
// the max grows, add exp(S - m) V, and divide by l once at the end.  The N x N scores
// never leave the SM.
//
// B200 mapping
//   * One persistent CTA per SM walks a static list of work units; a unit is two
//     128-row query tiles (Q0, Q1) of one (batch, head), so every K/V tile that TMA
//     brings in is used by 256 query rows.
//   * Warp roles (384 threads, three warpgroups): warps 0-3 own the softmax of Q0 (one
//     thread per row, TMEM lane = row), warps 4-7 the softmax of Q1, warp 8 issues TMA
//     loads, warp 9 issues tcgen05 MMAs from one thread, warps 10-11 only give up their
//     registers.  The launch grants 168 registers a thread (384 x 168 = 64512); the
//     control warpgroup drops to 88 (enough for fully unrolled MMA issue) and the two
//     softmax warpgroups rise to 208, which uses exactly that pool
//     (2 x 128 x 208 + 128 x 88 = 64512) and lets a softmax
//     thread hold its whole 128-entry score row in registers.
//   * TMEM (512 columns): S0 | S1 | O0 | O1.  The score tile S_t = Q_t K_j^T lands in
//     TMEM as fp32; the softmax threads read their row, write the probabilities as bf16
//     over the first 64 columns of the same S_t region, and the MMA O_t += P_t V_j
//     takes P straight from TMEM (A operand) and V from shared memory.
//   * The MMA issue order S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) ... lets the
//     tensor core work on one tile's products while the other tile's softmax runs.
//   * The running max is kept in log2 units.  The output is rescaled only when a row's
//     max grows by more than kRescaleThreshold (a factor 2^8); otherwise the older,
//     smaller reference max stays in force, which is exact because l and O always use
//     the same reference, and keeps every exponential below 2^8.
//   * K/V tiles stream through a ring of shared-memory slots guarded by mbarriers
//     (full: TMA transaction bytes; empty: tcgen05.commit from the MMA thread).
//   * O leaves through shared memory: each softmax warp writes its 32 rows, 64 columns
//     at a time, into a 4 KB staging box and its lane 0 issues a bulk tensor store of the
//     box, so HBM sees whole 128-byte lines and the warp goes on to its next unit while
//     the store drains.  A store of a row per lane would touch 32 lines per instruction;
//     at short sequences, where a unit is only a few key tiles long, those stores took
//     about a third of each unit.
//   * Queries and keys may differ in number (Nq <= Nk when causal): the queries are then
//     the last Nq tokens of the sequence, query row r at position r + Nk - Nq, and a
//     causal row sees keys up to its position (bottom-right alignment; Nq == Nk gives
//     the usual j <= i).  A query tile needs the key tiles up to the one holding its
//     last row's position; only tiles that cross a row's limit, and a ragged last key
//     tile, need element masks.  Rows past Nq (ragged last query tile) are computed on
//     zero-filled Q and never stored.
//   * Padded batches: with per-sequence lengths (seqlens_q[b], seqlens_k[b] <= Nq, Nk)
//     sequence b uses its first seqlens_q[b] query and seqlens_k[b] key rows, with the
//     same alignment rule; units past a sequence's queries have no work and every role
//     skips them.  Key rows past a sequence's length are masked like a ragged tail.
//   * Packed layout: tensors [tokens, H, d] with sequence b's tokens from cu_q[b] (keys
//     cu_k[b]); the tensor maps address (column, head, token), so a tile is 128 tokens of
//     one head from the sequence's first token on.  Tile rows past the sequence hold the
//     next sequence's tokens: masked as keys, not stored as queries.
#include <cfloat>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // key rows per tile
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsControl = 88;
constexpr int kRegsSoftmax = 208;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsLaunch,
              "register split exceeds the launch pool");
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;
// At d = 64 the S0 | S1 | O0 | O1 regions fill 384 of the 512 TMEM columns, which leaves
// room for the probabilities in regions of their own (P0 | P1, 64 columns each) instead
// of over their score tile.  S_t(j+1) can then be computed while the softmax of S_t(j)
// is still running: the tile's score product no longer waits for the P V product that
// reads the probabilities, and the softmax warps, which bound the kernel at d = 64
// (a 128 x 128 tile costs as many exponentials as at d = 128 for half the tensor work),
// find their next tile ready.
template <int D>
struct SeparateP {
  static constexpr bool value = (D == 64);
};

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = kBM * D * 2;  // one 128-row bf16 tile
  static constexpr int kBoxBytes = 128 * 128;     // one 128-row x 64-col box
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTileBytes;
  static constexpr int kRing = 2 * kTileBytes;
  // O staging for the bulk tensor stores of the epilogue: per softmax warp, one box of
  // its 32 rows x 64 columns (4 KB)
  static constexpr int kOst = kRing + kStages * kTileBytes;
  static constexpr int kBar = kOst + 2 * kBoxBytes;
  // barrier indices
  static constexpr int kBarQFull = 0;                 // [2]
  static constexpr int kBarQEmpty = 2;                // [2]
  static constexpr int kBarKVFull = 4;                // [kStages]
  static constexpr int kBarKVEmpty = 4 + kStages;     // [kStages]
  static constexpr int kBarSFull = 4 + 2 * kStages;   // [2]
  static constexpr int kBarPReady = 6 + 2 * kStages;  // [2]
  static constexpr int kBarODone = 8 + 2 * kStages;   // [2]
  static constexpr int kBarOFree = 10 + 2 * kStages;  // [2]
  static constexpr int kBarDrain = 12 + 2 * kStages;  // [1]
  static constexpr int kBarSFree = 13 + 2 * kStages;  // [2] (separate-P layout only)
  static constexpr int kNumBars = 15 + 2 * kStages;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 bytes
};

struct FwdArgs {
  unsigned int* err;  // library error word (wait timeouts)
  __nv_bfloat16* O;
  float* LSE;
  const int* seqlens_q;  // [B] per-sequence query rows, or null (all Nq)
  const int* seqlens_k;  // [B] per-sequence key rows, or null (all Nk)
  const int* cu_q;       // packed layout: [B+1] first query token of each sequence, or null
  const int* cu_k;       // packed layout: [B+1] first key token of each sequence
  int total_q;           // packed layout: query tokens of all sequences
  int total_k;
  int H;
  int BH;
  int Nq;           // query rows per head (padded length with seqlens)
  int Nk;           // key rows per head (padded length with seqlens)
  int causal;
  int n_units;      // units per (batch, head) = ceil(Nq / 256)
  int total_units;  // BH * n_units
  float scale_log2;  // scale * log2(e)
};

struct UnitInfo {
  int bh, u, n0, n1;  // n_t: key tiles of query tile t (0: no work)
  int lq, lk, off;    // the sequence's query rows, key rows, position of query row 0
  int h, tq0, tk0;    // head; packed layout: the sequence's first query and key token
};

__device__ __forceinline__ UnitInfo unit_info(int w, const FwdArgs& a) {
  UnitInfo r;
  if (a.causal) {
    // heaviest units (largest query index) first, all heads of one row-band together
    r.u = a.n_units - 1 - w / a.BH;
    r.bh = w % a.BH;
  } else {
    r.bh = w / a.n_units;
    r.u = w % a.n_units;
  }
  r.lq = a.Nq;
  r.lk = a.Nk;
  r.h = r.bh % a.H;
  r.tq0 = 0;
  r.tk0 = 0;
  if (a.cu_q != nullptr) {
    const int b = r.bh / a.H;
    r.tq0 = a.cu_q[b];
    r.tk0 = a.cu_k[b];
    r.lq = a.cu_q[b + 1] - r.tq0;
    r.lk = a.cu_k[b + 1] - r.tk0;
    if (r.tq0 < 0 || r.lq < 0 || r.lq > a.Nq || r.tq0 + r.lq > a.total_q || r.tk0 < 0 ||
        r.lk < 0 || r.lk > a.Nk || r.tk0 + r.lk > a.total_k || (a.causal && r.lq > r.lk)) {
      if (threadIdx.x == 0) atomicOr(a.err, kErrBadLength);
      r.lq = 0;  // the sequence is skipped
      r.lk = 0;
    }
  } else if (a.seqlens_q != nullptr) {
    const int b = r.bh / a.H;
    r.lq = a.seqlens_q[b];
    r.lk = a.seqlens_k[b];
    if (r.lq < 0 || r.lq > a.Nq || r.lk < 0 || r.lk > a.Nk || (a.causal && r.lq > r.lk)) {
      if (threadIdx.x == 0) atomicOr(a.err, kErrBadLength);
      r.lq = 0;  // the sequence is skipped
      r.lk = 0;
    }
  }
  r.off = r.lk - r.lq;
  const int n_kv = (r.lk + kBN - 1) / kBN;
  const int qt0 = 2 * r.u, qt1 = 2 * r.u + 1;
  const bool valid0 = r.lk > 0 && qt0 * kBM < r.lq;
  const bool valid1 = r.lk > 0 && qt1 * kBM < r.lq;
  // causal: key tiles up to the one holding the position of the tile's last row
  auto n_causal = [&](int qt) { return min((qt * kBM + kBM - 1 + r.off) / kBN + 1, n_kv); };
  r.n0 = valid0 ? (a.causal ? n_causal(qt0) : n_kv) : 0;
  r.n1 = valid1 ? (a.causal ? n_causal(qt1) : n_kv) : 0;
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmO, const FwdArgs args) {
  using L = FwdLayout<D>;
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
  // TMA coordinates of row `row` of a unit's queries (t0 = tq0) or keys (t0 = tk0):
  // (row, head) in the [BH][N][d] maps, (head, first token + row) in the packed maps
  const bool packed = args.cu_q != nullptr;
  auto tma_y = [&](const UnitInfo& ui, int row) { return packed ? ui.h : row; };
  auto tma_z = [&](const UnitInfo& ui, int t0, int row) { return packed ? t0 + row : ui.bh; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::kBarQFull + 0), 1);
    mbar_init(bar(L::kBarQFull + 1), 1);
    mbar_init(bar(L::kBarQEmpty + 0), 1);
    mbar_init(bar(L::kBarQEmpty + 1), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kBarKVFull + s), 1);
      mbar_init(bar(L::kBarKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kBarSFull + t), 1);
      mbar_init(bar(L::kBarPReady + t), kBM / 32);  // one arrival per softmax warp
      mbar_init(bar(L::kBarODone + t), 1);
      mbar_init(bar(L::kBarOFree + t), kBM / 32);
      mbar_init(bar(L::kBarSFree + t), kBM / 32);
    }
    mbar_init(bar(L::kBarDrain), 1);
    fence_mbar_init();
  }
  if (warp == kWarpTMA && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr bool kSepP = SeparateP<D>::value;
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
  // where the bf16 probabilities of tile t go: their own region, or over S_t
  const uint32_t tP[2] = {kSepP ? tmem + 256 + 2 * D : tS[0],
                          kSepP ? tmem + 256 + 2 * D + 64 : tS[1]};

  if (warp >= 8) regs_dec<kRegsControl>();
  if (warp == kWarpTMA) {
    // ------------------------------------------------------------ TMA producer
    // (the whole warp runs the loop; one elected lane issues each copy)
    {
      int stage = 0;
      uint32_t phase = 0;
      int q_uses[2] = {0, 0};
      bool ok = true;
      int issued[L::kStages];
      uint32_t issued_phase[L::kStages];
      for (int s = 0; s < L::kStages; ++s) issued[s] = 0, issued_phase[s] = 0;
      for (int r = 0, w = snake_unit(0); ok && w < args.total_units; w = snake_unit(++r)) {
        const UnitInfo ui = unit_info(w, args);
        if (ui.n0 == 0) continue;  // no query rows in this unit (every role skips it)
        for (int t = 0; t < 2 && ok; ++t) {
          if (t == 1 && ui.n1 == 0) break;
          if (q_uses[t] > 0)
            ok = wait_warp(bar(L::kBarQEmpty + t), (q_uses[t] - 1) & 1);
          if (!ok) break;
          const uint32_t qb = bar(L::kBarQFull + t);
          mbar_arrive_expect_tx_elect(qb, L::kTileBytes);
          const uint32_t dst = base + (t == 0 ? L::kQ0 : L::kQ1);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d_elect(dst + c * L::kBoxBytes, &tmQ, qb, c * 64,
                              tma_y(ui, (2 * ui.u + t) * kBM), tma_z(ui, ui.tq0, (2 * ui.u + t) * kBM));
          ++q_uses[t];
        }
        const int n = max(ui.n0, ui.n1);
        for (int j = 0; ok && j < n; ++j) {
          for (int kv = 0; kv < 2; ++kv) {  // K_j then V_j
            ok = wait_warp(bar(L::kBarKVEmpty + stage), phase ^ 1);
            if (!ok) break;
            const uint32_t fb = bar(L::kBarKVFull + stage);
            mbar_arrive_expect_tx_elect(fb, L::kTileBytes);
            const uint32_t dst = base + L::kRing + stage * L::kTileBytes;
            const CUtensorMap* tm = kv == 0 ? &tmK : &tmV;
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d_elect(dst + c * L::kBoxBytes, tm, fb, c * 64, tma_y(ui, j * kBN),
                                tma_z(ui, ui.tk0, j * kBN));
            issued[stage] = 1;
            issued_phase[stage] = phase;
            if (++stage == L::kStages) stage = 0, phase ^= 1;
          }
        }
      }
      if (!ok) {
        // wind down: let every load already issued land before the CTA exits
        for (int s = 0; s < L::kStages; ++s)
          if (issued[s]) mbar_wait_drain(bar(L::kBarKVFull + s), issued_phase[s], args.err);
        for (int t = 0; t < 2; ++t)
          if (q_uses[t] > 0)
            mbar_wait_drain(bar(L::kBarQFull + t), (q_uses[t] - 1) & 1, args.err);
      }
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------------ MMA issuer
    // (the whole warp runs the loop so descriptors stay warp-uniform; one elected lane
    // issues each tcgen05 instruction)
    {
      constexpr uint32_t idS = idesc_bf16_f32(kBN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(D, true);
      int stage = 0;
      uint32_t phase = 0;
      int uses[2] = {0, 0};
      int p_count[2] = {0, 0};
      bool ok = true;
      auto next_slot = [&](int& slot) -> bool {
        slot = stage;
        const bool r = wait_warp(bar(L::kBarKVFull + stage), phase);
        if (++stage == L::kStages) stage = 0, phase ^= 1;
        return r;
      };
      // Descriptors differ only in their start-address field (low 14 bits, address >> 4),
      // so each K step adds its byte offset >> 4 to a base descriptor.  The K-step loops
      // are fully unrolled: one thread issues every MMA, and with loop overhead between
      // the instructions it cannot keep the tensor pipe fed (a 128 x 128 x 16 MMA takes
      // only 64 cycles).
      const uint64_t dQ0 = desc_kmajor(base + L::kQ0);
      const uint64_t dQ1 = desc_kmajor(base + L::kQ1);
      const uint64_t dRingK = desc_kmajor(base + L::kRing);
      const uint64_t dRingV = desc_mnmajor(base + L::kRing, L::kBoxBytes);
      auto issue_s = [&](int t, int kslot) {
        const uint64_t da = t == 0 ? dQ0 : dQ1;
        const uint64_t db = dRingK + static_cast<uint64_t>((kslot * L::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * L::kBoxBytes + (kk % 4) * 32) >> 4;
          mma_ss_elect(tS[t], da + off, db + off, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit_elect(bar(L::kBarSFull + t));
      };
      auto issue_pv = [&](int t, int vslot, bool accumulate) {
        const uint64_t db = dRingV + static_cast<uint64_t>((vslot * L::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          mma_ts_elect(tO[t], tP[t] + kk * 8, db + static_cast<uint64_t>((kk * 2048) >> 4), idPV,
                 (accumulate || kk > 0) ? 1u : 0u);
        }
        mma_commit_elect(bar(L::kBarODone + t));
      };
      // warp-uniform non-blocking test of a barrier phase
      auto test_warp = [&](uint32_t b, uint32_t parity) -> bool {
        return __shfl_sync(0xffffffffu, mbar_test(b, parity) ? 1 : 0, 0) != 0;
      };
      if constexpr (kSepP) {
        // Separate P regions: the four products of a key tile j (S_t(j) for t = 0, 1 and
        // P_t V_j) are issued in whatever order their inputs become ready -- S_t(j) once
        // K_j has landed and the softmax warps hold S_t(j-1) in registers, P_t V_j once
        // they have written P_t(j) and V_j has landed.  K_j and V_j are released when
        // both tiles have issued their product with it.  The TMA warp loads the unit's
        // tiles in the order K_0 V_0 K_1 V_1 ..., so K_j sits at ring position
        // ring + 2j and V_j at ring + 2j + 1.
        int ring = 0;
        int s_tot[2] = {0, 0};
        for (int r = 0, w = snake_unit(0); ok && w < args.total_units; w = snake_unit(++r)) {
          const UnitInfo ui = unit_info(w, args);
          if (ui.n0 == 0) continue;  // no query rows in this unit
          const int nt[2] = {ui.n0, ui.n1};
          const int n = max(ui.n0, ui.n1);
          for (int t = 0; t < 2 && ok; ++t)
            if (nt[t] > 0) ok = wait_warp(bar(L::kBarQFull + t), uses[t] & 1);
          if (!ok) break;
          int sI[2] = {0, 0}, pI[2] = {0, 0};
          long long t0 = clock64();
          uint32_t idle = 0;
          while (sI[0] < nt[0] || sI[1] < nt[1] || pI[0] < nt[0] || pI[1] < nt[1]) {
            bool progress = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int o = 1 - t;
              if (sI[t] < nt[t]) {
                const int j = sI[t];
                const int pos = ring + 2 * j;
                const int st = pos % L::kStages;
                if ((s_tot[t] == 0 || test_warp(bar(L::kBarSFree + t), (s_tot[t] - 1) & 1)) &&
                    test_warp(bar(L::kBarKVFull + st), (pos / L::kStages) & 1)) {
                  tc_fence_after();
                  issue_s(t, st);
                  if (j + 1 == nt[t]) mma_commit_elect(bar(L::kBarQEmpty + t));
                  ++s_tot[t];
                  ++sI[t];
                  if (nt[o] <= j || sI[o] > j) mma_commit_elect(bar(L::kBarKVEmpty + st));
                  progress = true;
                }
              }
              if (pI[t] < nt[t]) {
                const int j = pI[t];
                const int pos = ring + 2 * j + 1;
                const int st = pos % L::kStages;
                if (test_warp(bar(L::kBarPReady + t), p_count[t] & 1) &&
                    (j > 0 || uses[t] == 0 ||
                     test_warp(bar(L::kBarOFree + t), (uses[t] - 1) & 1)) &&
                    test_warp(bar(L::kBarKVFull + st), (pos / L::kStages) & 1)) {
                  tc_fence_after();
                  issue_pv(t, st, j > 0);
                  ++p_count[t];
                  ++pI[t];
                  if (nt[o] <= j || pI[o] > j) mma_commit_elect(bar(L::kBarKVEmpty + st));
                  progress = true;
                }
              }
            }
            if (progress) {
              idle = 0;
              continue;
            }
            // nothing was ready: give up after the same limit as every other wait
            if (++idle == 1) t0 = clock64();
            if (idle % kSpinCheck == 0) {
              int code = 0;  // 1: another warp aborted, 2: this wait timed out
              if (lane == 0)
                code = *abort_flag ? 1 : (clock64() - t0 > kWaitLimitCycles ? 2 : 0);
              code = __shfl_sync(0xffffffffu, code, 0);
              if (code == 2 && lane == 0) {
                atomicOr(args.err, kErrWaitTimeout);
                *abort_flag = 1;
              }
              if (code != 0) {
                ok = false;
                break;
              }
            }
          }
          ring += 2 * n;
          for (int t = 0; t < 2; ++t)
            if (nt[t] > 0) ++uses[t];
        }
      } else {
      for (int r = 0, w = snake_unit(0); ok && w < args.total_units; w = snake_unit(++r)) {
        const UnitInfo ui = unit_info(w, args);
        if (ui.n0 == 0) continue;  // no query rows in this unit
        const int nt[2] = {ui.n0, ui.n1};
        const int n = max(ui.n0, ui.n1);
        for (int t = 0; t < 2 && ok; ++t)
          if (nt[t] > 0) ok = wait_warp(bar(L::kBarQFull + t), uses[t] & 1);
        if (!ok) break;
        int kslot;
        ok = next_slot(kslot);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          if (nt[t] > 0) {
            issue_s(t, kslot);
            if (nt[t] == 1) mma_commit_elect(bar(L::kBarQEmpty + t));
          }
        }
        mma_commit_elect(bar(L::kBarKVEmpty + kslot));
        for (int j = 0; ok && j < n; ++j) {
          int vslot, knext = -1;
          ok = next_slot(vslot);
          if (!ok) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j >= nt[t]) continue;
            if (j == 0 && uses[t] > 0)
              ok = wait_warp(bar(L::kBarOFree + t), (uses[t] - 1) & 1);
            if (ok) ok = wait_warp(bar(L::kBarPReady + t), p_count[t] & 1);
            if (!ok) break;
            ++p_count[t];
            tc_fence_after();
            issue_pv(t, vslot, j > 0);
            if (j + 1 < nt[t]) {
              // the next key tile is needed only now, not before the P V product above
              if (knext < 0) ok = next_slot(knext);
              if (!ok) break;
              tc_fence_after();
              issue_s(t, knext);
              if (j + 2 == nt[t]) mma_commit_elect(bar(L::kBarQEmpty + t));
            }
          }
          if (!ok) break;
          mma_commit_elect(bar(L::kBarKVEmpty + vslot));
          if (knext >= 0) mma_commit_elect(bar(L::kBarKVEmpty + knext));
        }
        for (int t = 0; t < 2; ++t)
          if (nt[t] > 0) ++uses[t];
      }
      }
      // drain: every MMA issued has completed before TMEM is released
      mma_commit_elect(bar(L::kBarDrain));
      mbar_wait_drain(bar(L::kBarDrain), 0, args.err);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax, tile t
    regs_inc<kRegsSoftmax>();
    const int t = warp / 4;
    const int row = (warp % 4) * 32 + lane;        // row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tSrow = tS[t] + lane_off;
    const uint32_t tOrow = tO[t] + lane_off;
    const uint32_t tProw = tP[t] + lane_off;
    int s_count = 0, o_count = 0;
    bool st_used = false;  // this warp's O staging box has been handed to a bulk store
    bool ok = true;
    for (int r = 0, w = snake_unit(0); ok && w < args.total_units; w = snake_unit(++r)) {
      const UnitInfo ui = unit_info(w, args);
      const int n_t = t == 0 ? ui.n0 : ui.n1;
      if (n_t == 0) continue;
      const int qt = 2 * ui.u + t;
      const int q_row = qt * kBM + row;
      float m = -INFINITY;  // running max, log2 units (scaled logits * log2 e)
      float l = 0.f;
      for (int j = 0; j < n_t; ++j) {
        ok = wait_warp(bar(L::kBarSFull + t), s_count & 1);
        if (!ok) break;
        ++s_count;
        tc_fence_after();
        uint32_t sr[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tSrow + c * 32, &sr[c * 32]);
        tmem_wait_ld();
        // with P in its own region, S_t's columns are free as soon as they are read
        if constexpr (kSepP) warp_arrive(bar(L::kBarSFree + t));
        float s[kBN];
#pragma unroll
        for (int c = 0; c < kBN; ++c) s[c] = __uint_as_float(sr[c]);
        const int kv0 = j * kBN;
        // a ragged last key tile, or (causal) a tile whose last key lies past the
        // position of the tile's first row
        const bool need_mask = (kv0 + kBN > ui.lk) ||
                               (args.causal && kv0 + kBN - 1 > qt * kBM + ui.off);
        if (need_mask) {
          const int lim = args.causal ? min(ui.lk, q_row + ui.off + 1) : ui.lk;
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (kv0 + c >= lim) s[c] = -INFINITY;
        }
        // row max as 8 independent chains of 3-input max folded at the end (a single
        // chain of 128 dependent max operations would sit on the critical path)
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = s[k];
#pragma unroll
        for (int c = 8; c < kBN; c += 2) mx8[(c / 2) % 8] = max3(mx8[(c / 2) % 8], s[c], s[c + 1]);
        const float mx = max3(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5]),
                              fmaxf(mx8[6], mx8[7]));
        const float m_tile = mx * args.scale_log2;
        float alpha = 1.f;
        bool rescale = false;
        if (m_tile > m + kRescaleThreshold || m == -INFINITY) {
          const float m_new = fmaxf(m, m_tile);
          alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
          m = m_new;
          rescale = true;
        }
        // O_t holds the sum through key tile j-1 once that P V product completes; then it
        // is scaled by alpha (only when some row's reference max moved)
        auto rescale_o = [&]() {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tOrow + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k)
              v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
            tmem_st32(tOrow + c * 32, v);
          }
        };
        if (!kSepP && __any_sync(0xffffffffu, rescale && j > 0)) {
          ok = wait_warp(bar(L::kBarODone + t), (o_count + j - 1) & 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          rescale_o();
        }
        l *= alpha;
        const float mref = (m == -INFINITY) ? 0.f : m;
        // p = 2^(s * scale * log2e - m): the scale-and-subtract and the row sum run on
        // packed float pairs (one instruction per two entries), the exponentials on MUFU
        uint32_t pk[kBN / 2];
        const uint64_t scale2 = f32x2(args.scale_log2, args.scale_log2);
        const uint64_t negm2 = f32x2(-mref, -mref);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < kBN / 2; ++c) {
          const uint64_t x2 = fma_x2(f32x2(s[2 * c], s[2 * c + 1]), scale2, negm2);
          float p0, p1;
          exp2_pair(x2, p0, p1);
          ls2[c % 4] = add_x2(ls2[c % 4], f32x2(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
        float ls[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) f32x2_split(ls2[k], ls[2 * k], ls[2 * k + 1]);
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        if constexpr (kSepP) {
          // P_t's region is free, and O_t complete through key tile j-1, once P_t V_{j-1}
          // has completed; by now it normally has (it was issued a whole tile ago)
          if (j > 0) {
            ok = wait_warp(bar(L::kBarODone + t), (o_count + j - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, rescale)) rescale_o();
          }
        }
        tmem_st32(tProw, &pk[0]);
        tmem_st32(tProw + 32, &pk[32]);
        tmem_wait_st();
        warp_arrive(bar(L::kBarPReady + t));
      }
      if (!ok) break;
      // epilogue: O = acc / l, LSE = (m + log2 l) * ln 2
      ok = wait_warp(bar(L::kBarODone + t), (o_count + n_t - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      o_count += n_t;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int bh = ui.bh;
      __nv_bfloat16* orow =
          args.O + (packed ? (static_cast<size_t>(ui.tq0 + q_row) * args.H + ui.h) * D
                           : (static_cast<size_t>(bh) * args.Nq + q_row) * D);
      // take the whole O row into registers first, so the MMA warp may start the next
      // unit's first P V product while this row is being converted and stored
      uint32_t ov[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tOrow + c * 32, &ov[c * 32]);
      tmem_wait_ld();
      warp_arrive(bar(L::kBarOFree + t));
      if ((qt * kBM + (warp % 4) * 32 + 32) <= ui.lq) {
        // all 32 rows of this warp are valid: each row goes, 64 columns at a time, into
        // the warp's staging box in the 128-byte-swizzled layout of the tensor map (row
        // r's 16-byte chunk k at r * 128 + ((k ^ (r % 8)) * 16), so the warp writes all
        // 32 banks four times over), and one bulk tensor store per box writes it to HBM
        // in whole lines.  The warp's lane 0 issues the stores and, before the box is
        // written again, waits until the previous store has read it.
        const uint32_t stg_a = base + L::kOst + (t * 4 + warp % 4) * (32 * 128);
        uint8_t* stg = smem + (stg_a - base);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          if (st_used) {
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t* o8 = &ov[c * 64 + 8 * k];
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((k ^ (lane & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(o8[0]) * inv_l, __uint_as_float(o8[1]) * inv_l),
                pack_bf16x2(__uint_as_float(o8[2]) * inv_l, __uint_as_float(o8[3]) * inv_l),
                pack_bf16x2(__uint_as_float(o8[4]) * inv_l, __uint_as_float(o8[5]) * inv_l),
                pack_bf16x2(__uint_as_float(o8[6]) * inv_l, __uint_as_float(o8[7]) * inv_l));
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            const int r0 = qt * kBM + (warp % 4) * 32;
            tma_store_3d(&tmO, stg_a, c * 64, tma_y(ui, r0), tma_z(ui, ui.tq0, r0));
            bulk_commit_group();
          }
          st_used = true;
        }
      } else if (q_row < ui.lq) {
        // some of the warp's rows belong to no query (or, packed, to the next sequence):
        // row by row, valid rows only
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            pk[k] = pack_bf16x2(__uint_as_float(ov[c * 32 + 2 * k]) * inv_l,
                                __uint_as_float(ov[c * 32 + 2 * k + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (args.LSE != nullptr && q_row < ui.lq)
        args.LSE[packed ? static_cast<size_t>(ui.h) * args.total_q + ui.tq0 + q_row
                        : static_cast<size_t>(bh) * args.Nq + q_row] =
            (m + __log2f(l)) * 0.69314718055994531f;
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

template <int D>
cudaError_t launch_d(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                     const CUtensorMap& tmO, void* O, float* LSE, const Problem& p, int num_sms,
                     cudaStream_t stream) {
  using L = FwdLayout<D>;
  FwdArgs a;
  a.err = p.err;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
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
  a.causal = p.causal;
  a.n_units = (p.N + 2 * kBM - 1) / (2 * kBM);
  a.total_units = p.BH * a.n_units;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  // The register split inside the kernel assumes exactly kRegsLaunch registers a thread
  // at launch; with fewer, the softmax warpgroups' increase could never be granted.
  cudaFuncAttributes fattr;
  cudaError_t e = cudaFuncGetAttributes(&fattr, fwd_sm100_kernel<D>);
  if (e != cudaSuccess) return e;
  if (fattr.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L::kAlloc);
  if (e != cudaSuccess) return e;
  const int grid = a.total_units < num_sms ? a.total_units : num_sms;
  if ((e = trace_mark(p, 0, stream)) != cudaSuccess) return e;
  fwd_sm100_kernel<D><<<grid, kThreads, L::kAlloc, stream>>>(tmQ, tmK, tmV, tmO, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_mark(p, 1, stream);
}

}  // namespace

cudaError_t launch_fwd_sm100(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmO, void* O, float* LSE,
                             const Problem& p, int num_sms, cudaStream_t stream) {
  if (p.d == 64) return launch_d<64>(tmQ, tmK, tmV, tmO, O, LSE, p, num_sms, stream);
  return launch_d<128>(tmQ, tmK, tmV, tmO, O, LSE, p, num_sms, stream);
}

}  // namespace fa

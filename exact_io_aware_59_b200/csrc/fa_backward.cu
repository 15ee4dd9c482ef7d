// fa_backward.cu -- exact attention backward (dQ, dK, dV) on sm_100a.
//
// What it computes: the gradient of O = softmax(scale * Q K^T [+ causal mask]) V for an
// upstream gradient dO, from Q, K, V, O, dO and the forward's per-row log-sum-exp.  The
// pages say that training runs a backward pass that is IO-aware like the forward ("Flash
// Attention -- Module 12.3", section "Prefill vs Decode", "Training"), and that the
// forward keeps per-row softmax statistics rather than the score matrix ("FlashAttention
// 1-2-3", section "FlashAttention-1: Tiling, Recomputation, and Online Softmax").  So P is
// recomputed tile by tile from S = Q K^T and the saved LSE, and nothing N x N reaches HBM:
//     P  = exp(scale * S - LSE)      dV = P^T dO       dP = dO V^T
//     D  = rowsum(dO * O)            dS = P * (dP - D)
//     dQ = scale * dS K              dK = scale * dS^T Q
//
// Three kernels, in stream order:
//  * fa_bwd_prep: D and -LSE * log2(e) per query row (into a workspace padded to whole
//    128-row query tiles), and zeroes the fp32 dQ accumulator;
//  * fa_bwd_sm100: one CTA per (key tile of 128, b*h).  It walks the query tiles of 128
//    that see its keys, keeps dK and dV for its keys in TMEM, and adds each step's dQ
//    contribution into the fp32 accumulator (coalesced reductions at L2);
//  * fa_bwd_dq: dQ = scale * accumulator, converted to the inputs' 16-bit type.
//
// fa_bwd_sm100 roles (512 threads; our design for tcgen05, with keys as the MMA's M so the
// per-key sums dK and dV stay in TMEM for the whole walk, and every product 128 x 128 --
// the tensor core's full rate):
//  * warp 0 (one lane): TMA loads of K and V once; per query tile i, Q_i with -LSE*log2e
//    and D into a 2-stage ring, and dO_i into one buffer that is reloaded as soon as dV(i)
//    has read it;
//  * warp 1 (one lane): tcgen05.mma issue, per query tile i:
//        dV  += P^T dO_i   (A = P^T, 16-bit, from TMEM over S; B = dO_i MN-major)
//        S^T  = K Q_{i+1}^T  (M 128 keys, N 128 queries, K = d) into S, once dV(i) is issued
//        dQ^T = K^T dS^T   (M 128 = d, N 128 queries, K 128 keys; A = K read MN-major, B = dS
//                           from shared memory) into dP, whose dP(i) the softmax has read
//        dK  += dS^T Q_i   (A = dS^T, the same shared-memory tile read K-major; B = Q_i
//                           MN-major), issued after dQ^T(i) so that the drain of dQ^T(i)
//                           overlaps it
//        dP^T = V dO_{i+1}^T into dP, once the drain has read dQ^T(i) out of it
//    tcgen05.mma operations run in issue order, so an MMA that overwrites columns an
//    earlier MMA reads as its A operand needs no wait in between;
//  * warpgroups 1 and 2 (warps 4-7 and 8-11) both work on every query tile, one thread per
//    key, warpgroup w on queries 64w .. 64w+63: P^T from S^T as soon as S is ready,
//    stored back as 16-bit over the warpgroup's own S columns (64w .. 64w+31) for dV; then
//    dS^T = P^T (dP^T - D) once dP is, stored to shared memory (128-byte swizzle, one
//    128-byte row per key and 64-query block) for both dQ and dK.  At the end warpgroup 1
//    writes dV and warpgroup 2 writes scale * dK;
//  * warpgroup 3 (warps 12-15), one thread per d-row of dQ^T: TMEM -> registers (the
//    columns are then free for dP(i+1)) -> fp32 reductions into row-major dQ accumulator
//    rows, each warp instruction adding 32 consecutive floats of one query row.
// Registers: the launch gives 128 per thread; warpgroup 0 drops to kRegsSide, the softmax
// warpgroups rise to kRegsSoftmax and the drain warpgroup to kRegsDrain (setmaxnreg).
// TMEM (512 columns): dV [0,128) dK [128,256) S [256,384) dP [384,512).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_device.cuh"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kBK = 128;       // keys per CTA (MMA M)
constexpr int kBQ = 128;       // queries per step (MMA N of S^T, dP^T, dQ^T; K of dV, dK)
constexpr int kHalfQ = 64;     // queries per softmax warpgroup
constexpr int kStages = 2;     // Q ring
constexpr int kThreads = 512;
constexpr int kRegsLaunch = 128;   // 65536 / 512
constexpr int kRegsSide = 64;      // warps 0-3
constexpr int kRegsSoftmax = 152;  // warps 4-11
constexpr int kRegsDrain = 144;    // warps 12-15
static_assert(128 * kRegsSide + 256 * kRegsSoftmax + 128 * kRegsDrain <= kThreads * kRegsLaunch,
              "register split");

// D: head dimension, 64 or 128.  A tile of 128 rows is D / 64 blocks of 128 rows x 128 B.
template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;           // 128 rows of D 16-bit values
  static constexpr int kKOff = 0;                           // K tile
  // The dQ product reads K as an MN-major A operand of M = 128 rows of d: for d = 64 the
  // second 64-row block (one LBO, 16 KB, after K) is a block of zeros, so rows 64-127 of
  // dQ^T come out 0 and are not drained.
  static constexpr int kZeroOff = kKOff + kTileBytes;
  static constexpr int kVOff = (D == 64) ? kZeroOff + 16384 : kKOff + kTileBytes;  // V tile
  static constexpr int kQOff = kVOff + kTileBytes;          // Q stages
  static constexpr int kdOOff = kQOff + kStages * kTileBytes;  // dO (one buffer)
  static constexpr int kdSOff = kdOOff + kTileBytes;        // dS, 128 keys x 128 queries,
  static constexpr int kdSBytes = kBK * kBQ * 2;            // two 64-query blocks (any d)
  static constexpr int kLseOff = kdSOff + kdSBytes;         // -LSE*log2e per stage
  static constexpr int kDelOff = kLseOff + kStages * kBQ * 4;  // D per stage
  static constexpr int kBarOff = kDelOff + kStages * kBQ * 4;
  // mbarriers
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;                // + stage: Q, -LSE*log2e and D landed
  static constexpr int kBarDOFull = kBarQFull + kStages;
  static constexpr int kBarDOFree = kBarDOFull + 1;  // dV(i) done: the dO buffer may be reloaded
  static constexpr int kBarSFull = kBarDOFree + 1;   // S(i) complete
  static constexpr int kBarDPFull = kBarSFull + 1;   // dP(i) complete
  static constexpr int kBarPReady = kBarDPFull + 1;  // P^T(i) stored (8 softmax warps)
  static constexpr int kBarDSReady = kBarPReady + 1; // dS(i) stored to shared memory (8 warps)
  static constexpr int kBarDQFull = kBarDSReady + 1; // dQ^T(i) complete (and all before it)
  static constexpr int kBarDQEmpty = kBarDQFull + 1; // dQ^T(i) read out of TMEM (4 warps)
  static constexpr int kBarQFree = kBarDQEmpty + 1;  // dK(i) complete: Q stage i and dS free
  static constexpr int kBarDone = kBarQFree + 1;     // every MMA of the CTA complete
  static constexpr int kBarFinished = kBarDone + 1;  // warps 4-15 done with TMEM
  static constexpr int kNumBars = kBarFinished + 1;
  static constexpr int kTmemHolderOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemHolderOff + 4;
  static constexpr int kBytes = kAbortOff + 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(kdSOff % 1024 == 0 && kQOff % 1024 == 0 && kdOOff % 1024 == 0 &&
                kVOff % 1024 == 0, "swizzle atoms");
  static_assert(D == 64 || D == 128, "head dimension");
};

// TMEM columns.
constexpr uint32_t kTdV = 0, kTdK = 128, kTS = 256, kTdP = 384;

// Column of the 16-bit A operand P^T (8 columns per 16 queries) for K-step kk:
// warpgroup w stores its queries 64w .. 64w+63 over its own columns 64w .. 64w+31.
__device__ __forceinline__ uint32_t a16_col(int kk) { return (kk < 4) ? 8u * kk : 64u + 8u * (kk - 4); }

__device__ __forceinline__ uint32_t bar_addr(uint32_t bars, int i) { return bars + 8u * i; }

// Bounded wait without a sleep hint, for the end-of-kernel drains.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
}

// The query tiles a key tile meets: [first, p.n_qtiles).  Causal (bottom-right): query q
// sees key k iff k <= q + off, so the first query that sees key k0 is k0 - off.
__device__ __forceinline__ int first_qtile(const BwdParams& p, int k0) {
  if (!p.causal) return 0;
  const int q = k0 - p.off;
  if (q >= p.Nq) return p.n_qtiles;
  return q <= 0 ? 0 : q / kBQ;
}

// One K-major step of 16 elements (32 B) of a tile with `rows` rows: 64-element column
// blocks of rows x 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t kmajor_step(int kk, int rows) {
  return static_cast<uint64_t>(((kk >> 2) * rows * 128 + (kk & 3) * 32) >> 4);
}

// Where one CTA's data lives.  [B,H,N,d] layout: tiles at (d column, row, b*h) of the 3-D
// tensor maps, head bh's workspace rows from bh * nq_pad, dK/dV row (bh * Nkv + key).
// Packed layout (VARLEN): tiles at (d column, h, token) of the (d, H, tokens) maps, the
// sequence's first query / key token q_tok0 / k_tok0, workspace rows from wrow0 (head h's
// rows, then the sequence's padded offset), dK/dV row (k_tok0 + key) * H + h.
struct BwdCta {
  int bh;            // b * H + h ([B,H,N,d]); h (packed)
  int q_tok0, k_tok0;
  long long wrow0;   // first workspace row of this CTA's query rows
};

template <bool VARLEN>
__device__ __forceinline__ void tile_load(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int col, int row, int tok0, int bh) {
  if constexpr (VARLEN)
    tma_load_3d(dst, map, bar, col, bh, tok0 + row);
  else
    tma_load_3d(dst, map, bar, col, row, bh);
}

// ---------------------------------------------------------------- producer (TMA)
template <int D, bool VARLEN>
__device__ void producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                         const CUtensorMap* tdo, const BwdParams& p, const BwdCta& cta, int k0,
                         int i0, int n, uint32_t sbase, uint32_t bars, int* status,
                         volatile int* abort_flag) {
  using C = BwdCfg<D>;
  const uint32_t kv = bar_addr(bars, C::kBarKV);
  mbar_arrive_expect_tx(kv, 2 * C::kTileBytes);
#pragma unroll
  for (int sub = 0; sub < D / 64; ++sub) {
    tile_load<VARLEN>(sbase + C::kKOff + sub * kBK * 128, tk, kv, sub * 64, k0, cta.k_tok0, cta.bh);
    tile_load<VARLEN>(sbase + C::kVOff + sub * kBK * 128, tv, kv, sub * 64, k0, cta.k_tok0, cta.bh);
  }
  int q_issued = 0, do_issued = 0;
  bool ok = true;
  auto wait = [&](int b, uint32_t parity) {
    return mbar_wait(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutBwd);
  };
  for (int i = 0; i < n; ++i) {
    const int st = i % kStages;
    const int q0 = (i0 + i) * kBQ;
    // Q stage st held tile i - 2, whose products are all complete once its dK is (dK(i-1)
    // is issued after S(i), so it cannot complete before Q(i) is loaded: the barrier is at
    // most one phase ahead).
    if (i >= kStages && !(ok = wait(C::kBarQFree, (i - kStages) & 1))) break;
    const uint32_t qf = bar_addr(bars, C::kBarQFull + st);
    mbar_arrive_expect_tx(qf, C::kTileBytes + 2 * kBQ * 4);
#pragma unroll
    for (int sub = 0; sub < D / 64; ++sub)
      tile_load<VARLEN>(sbase + C::kQOff + st * C::kTileBytes + sub * kBQ * 128, tq, qf, sub * 64,
                        q0, cta.q_tok0, cta.bh);
    const size_t row = static_cast<size_t>(cta.wrow0) + q0;
    bulk_load(sbase + C::kLseOff + st * kBQ * 4, p.nlse2 + row, kBQ * 4, qf);
    bulk_load(sbase + C::kDelOff + st * kBQ * 4, p.delta + row, kBQ * 4, qf);
    ++q_issued;
    // dO: one buffer, free once dV(i-1) has read it.
    if (i >= 1 && !(ok = wait(C::kBarDOFree, (i - 1) & 1))) break;
    const uint32_t df = bar_addr(bars, C::kBarDOFull);
    mbar_arrive_expect_tx(df, C::kTileBytes);
#pragma unroll
    for (int sub = 0; sub < D / 64; ++sub)
      tile_load<VARLEN>(sbase + C::kdOOff + sub * kBQ * 128, tdo, df, sub * 64, q0, cta.q_tok0,
                        cta.bh);
    ++do_issued;
  }
  if (!ok) {
    // Let every copy still in flight land before the CTA's shared memory goes away.
    for (int i = (q_issued > kStages ? q_issued - kStages : 0); i < q_issued; ++i)
      drain_wait(bar_addr(bars, C::kBarQFull + i % kStages), (i / kStages) & 1);
    if (do_issued) drain_wait(bar_addr(bars, C::kBarDOFull), (do_issued - 1) & 1);
    drain_wait(kv, 0);
  }
}

// ---------------------------------------------------------------- MMA issuer
template <int D, bool BF16>
__device__ void mma_issuer(int n, uint32_t sbase, uint32_t bars, uint32_t tmem, int* status,
                           volatile int* abort_flag) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc_s = make_idesc_f16(kBK, kBQ, BF16, false);          // S^T, dP^T
  constexpr uint32_t idesc_kv = make_idesc_f16(kBK, D, BF16, true);            // dV, dK
  constexpr uint32_t idesc_q = make_idesc_f16_ab(128, kBQ, BF16, true, true);  // dQ^T (M = 128
                                                                               // rows of d)
  // Descriptors are rebuilt from these two bases where they are used (the bases pass
  // through an opaque move each step), so the compiler does not keep all forty per-MMA
  // descriptors of a step live at once.
  uint64_t kmaj0 = make_sdesc_sw128(sbase, 16, 1024);           // K-major operands
  uint64_t mn0 = make_sdesc_sw128(sbase, kBK * 128, 1024);      // MN-major operands
  auto at = [](uint64_t base, uint32_t off) { return base + (off >> 4); };
  auto k_desc = [&]() { return at(kmaj0, C::kKOff); };
  auto v_desc = [&]() { return at(kmaj0, C::kVOff); };
  // K as the MN-major A of dQ^T: 64-row d blocks 128 x 128 B = 16 KB apart (LBO), 8-key
  // groups 1024 B apart (SBO); 16 keys (2048 B) per step.
  auto kt_desc = [&]() { return at(mn0, C::kKOff); };
  // dS as the MN-major B of dQ^T: two 64-query blocks 128 keys x 128 B = 16 KB apart.
  auto ds_desc = [&]() { return at(mn0, C::kdSOff); };
  // dS as the K-major A of dK (M = 128 keys, K = 128 queries): the same tile.
  auto ds_kmaj = [&]() { return at(kmaj0, C::kdSOff); };
  auto q_kmaj = [&](int st) { return at(kmaj0, C::kQOff + st * C::kTileBytes); };
  auto do_kmaj = [&]() { return at(kmaj0, C::kdOOff); };
  // Q and dO as MN-major B (d contiguous): d blocks 128 x 128 B = 16 KB apart, 16 queries
  // (2048 B) per step.
  auto q_mn = [&](int st) { return at(mn0, C::kQOff + st * C::kTileBytes); };
  auto do_mn = [&]() { return at(mn0, C::kdOOff); };
  auto refresh = [&]() {
    asm volatile("" : "+l"(kmaj0), "+l"(mn0));
  };
  auto wait = [&](int b, uint32_t parity) {
    return mbar_wait_spin(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutBwd);
  };
  auto issue_st = [&](uint32_t d_col, uint64_t a, uint64_t b) {  // S^T or dP^T
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_ss(tmem + d_col, a + kmajor_step(kk, kBK), b + kmajor_step(kk, kBQ), idesc_s, kk > 0 ? 1u : 0u);
  };
  bool ok = n > 0 && wait(C::kBarKV, 0);  // with no query tile nothing is loaded
  if (ok && (ok = wait(C::kBarQFull + 0, 0))) {
    tc_fence_after();
    issue_st(kTS, k_desc(), q_kmaj(0));
    tc_commit(bar_addr(bars, C::kBarSFull));
    if ((ok = wait(C::kBarDOFull, 0))) {
      tc_fence_after();
      issue_st(kTdP, v_desc(), do_kmaj());
      tc_commit(bar_addr(bars, C::kBarDPFull));
    }
  }
  for (int i = 0; i < n && ok; ++i) {
    const int st = i % kStages, st1 = (i + 1) % kStages;
    refresh();
    // P^T(i) is stored over S: dV(i), then release the dO buffer.
    if (!(ok = wait(C::kBarPReady, i & 1))) break;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < kBQ / 16; ++kk)
      mma_ts(tmem + kTdV, tmem + kTS + a16_col(kk), do_mn() + ((kk * 2048) >> 4), idesc_kv,
             (i > 0 || kk > 0) ? 1u : 0u);
    tc_commit(bar_addr(bars, C::kBarDOFree));
    // S(i+1) over S right away (P^T(i) there has been read by dV(i), issued above), so the
    // softmax can compute P^T(i+1) while dK(i), dQ(i) and dP(i+1) run.
    if (i + 1 < n) {
      if (!(ok = wait(C::kBarQFull + st1, ((i + 1) / kStages) & 1))) break;
      tc_fence_after();
      issue_st(kTS, k_desc(), q_kmaj(st1));
      tc_commit(bar_addr(bars, C::kBarSFull));
    }
    // dS(i) is in shared memory (the softmax has read dP(i) out of TMEM): dQ^T(i) over dP
    // first, so that the drain starts while dK(i) runs, then dK(i) with dS^T read from the
    // same shared-memory tile as a K-major A operand.
    if (!(ok = wait(C::kBarDSReady, i & 1))) break;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < kBK / 16; ++kk)
      mma_ss(tmem + kTdP, kt_desc() + ((kk * 2048) >> 4), ds_desc() + ((kk * 2048) >> 4), idesc_q,
             kk > 0 ? 1u : 0u);
    tc_commit(bar_addr(bars, C::kBarDQFull));
#pragma unroll
    for (int kk = 0; kk < kBQ / 16; ++kk)
      mma_ss(tmem + kTdK, ds_kmaj() + kmajor_step(kk, kBK), q_mn(st) + ((kk * 2048) >> 4),
             idesc_kv, (i > 0 || kk > 0) ? 1u : 0u);
    // Tile i's products are complete: its Q stage and dS may be reused.
    tc_commit(bar_addr(bars, C::kBarQFree));
    if (i + 1 < n) {
      // dP(i+1) over dP, once the drain has read dQ^T(i) and dO(i+1) has landed.
      if (!(ok = wait(C::kBarDQEmpty, i & 1))) break;
      if (!(ok = wait(C::kBarDOFull, (i + 1) & 1))) break;
      tc_fence_after();
      issue_st(kTdP, v_desc(), do_kmaj());
      tc_commit(bar_addr(bars, C::kBarDPFull));
    }
  }
  tc_commit(bar_addr(bars, C::kBarDone));
}

// ---------------------------------------------------------------- P and dS (one thread per key)
// Warpgroup `wg` (0 or 1) takes queries 64 wg .. 64 wg + 63 of every query tile.
template <int D, bool BF16, bool VARLEN>
__device__ void softmax_grad(const BwdParams& p, const BwdCta& cta, int k0, int i0, int n, int wg,
                             uint8_t* sgen, uint32_t bars, uint32_t tmem, int* status,
                             volatile int* abort_flag) {
  using C = BwdCfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;
  const int r = wq * 32 + lane;  // key row of the tile = TMEM lane
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int kidx = k0 + r;
  // First query that sees this key (a key past the end is seen by none).
  const long long qvis = kidx >= p.Nkv ? (1ll << 40) : (p.causal ? static_cast<long long>(kidx) - p.off : -(1ll << 40));
  const bool key_tail = k0 + kBK > p.Nkv;
  const float sl2 = p.scale_log2;
  const int c0 = wg * kHalfQ;  // this warpgroup's first query (and S / dP column) of the tile
  auto wait = [&](int b, uint32_t parity) {
    const bool ok = mbar_wait(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutBwd);
    return __all_sync(0xffffffffu, ok);
  };
  auto arrive = [&](int b) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, b));
  };
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    const int st = i % kStages;
    const int q0 = (i0 + i) * kBQ;
    if (!(ok = wait(C::kBarQFull + st, (i / kStages) & 1))) break;  // LSE_i and D_i visible
    if (!(ok = wait(C::kBarSFull, i & 1))) break;                   // S(i)
    tc_fence_after();
    const uint32_t tS = lane_base + kTS + c0;
    float pr[kHalfQ];
    {
      uint32_t a[32], b[32];
      tmem_ld_32x32b_x32(tS, a);
      tmem_ld_32x32b_x32(tS + 32, b);
      tmem_ld_wait(a);
      reg_fence(b);
      const float4* nl = reinterpret_cast<const float4*>(sgen + C::kLseOff + st * kBQ * 4 + c0 * 4);
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 l = nl[c4];
        const uint32_t* s = c4 < 8 ? &a[4 * c4] : &b[4 * (c4 - 8)];
        pr[4 * c4 + 0] = ex2(fmaf(__uint_as_float(s[0]), sl2, l.x));
        pr[4 * c4 + 1] = ex2(fmaf(__uint_as_float(s[1]), sl2, l.y));
        pr[4 * c4 + 2] = ex2(fmaf(__uint_as_float(s[2]), sl2, l.z));
        pr[4 * c4 + 3] = ex2(fmaf(__uint_as_float(s[3]), sl2, l.w));
      }
    }
    // Causal diagonal or key tail: column c is visible iff q0 + c >= qvis.
    if (key_tail || (p.causal && k0 + kBK - 1 - p.off > q0)) {
      const long long cm = qvis - q0 - c0;
      const int cmin = cm < 0 ? 0 : (cm > kHalfQ ? kHalfQ : static_cast<int>(cm));
#pragma unroll
      for (int c = 0; c < kHalfQ; ++c) pr[c] = (c >= cmin) ? pr[c] : 0.f;
    }
    {
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) pk[j] = pack2<BF16>(pr[2 * j], pr[2 * j + 1]);
      tmem_st_32x32b_x32(tS, pk);  // P^T over this warpgroup's first 32 S columns (read above)
    }
    tmem_st_wait();
    arrive(C::kBarPReady);
    // dS = P (dP - D) once dP(i) is complete (dQ(i-1) and dK(i-1), issued before dP(i),
    // are complete too, so the shared-memory dS buffer is free).
    if (!(ok = wait(C::kBarDPFull, i & 1))) break;
    tc_fence_after();
    const float4* dl = reinterpret_cast<const float4*>(sgen + C::kDelOff + st * kBQ * 4 + c0 * 4);
    // dS row r (this key) of the 64-query block wg: 16-byte chunk cc at position cc ^ (r & 7).
    uint8_t* ds_row = sgen + C::kdSOff + wg * (kBK * 128) + r * 128;
    const uint32_t tdP = lane_base + kTdP + c0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t dp[32];
      tmem_ld_32x32b_x32(tdP + 32 * h, dp);
      tmem_ld_wait(dp);
      uint32_t pk[16];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 dd = dl[8 * h + c4];
        const int c = 32 * h + 4 * c4;
        const float d0 = pr[c + 0] * (__uint_as_float(dp[4 * c4 + 0]) - dd.x);
        const float d1 = pr[c + 1] * (__uint_as_float(dp[4 * c4 + 1]) - dd.y);
        const float d2 = pr[c + 2] * (__uint_as_float(dp[4 * c4 + 2]) - dd.z);
        const float d3 = pr[c + 3] * (__uint_as_float(dp[4 * c4 + 3]) - dd.w);
        pk[2 * c4] = pack2<BF16>(d0, d1);
        pk[2 * c4 + 1] = pack2<BF16>(d2, d3);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = 4 * h + j;
        *reinterpret_cast<uint4*>(ds_row + ((cc ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
    }
    fence_proxy_async_smem();
    arrive(C::kBarDSReady);
  }

  // Epilogue: dV and scale * dK rows of this thread's key.
  bool have = n > 0;
  if (have) have = ok && wait(C::kBarDone, 0);
  if (n > 0 && !have) return;
  if (have) tc_fence_after();
  const size_t orow = VARLEN ? ((static_cast<size_t>(cta.k_tok0) + kidx) * p.H + cta.bh) * D
                            : (static_cast<size_t>(cta.bh) * p.Nkv + kidx) * D;
  {
    const int which = wg;  // warpgroup 1 writes dV, warpgroup 2 writes dK
    uint16_t* dst = static_cast<uint16_t*>(which ? p.dk : p.dv) + orow;
    const float mul = which ? p.scale : 1.f;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t v[32];
      if (have) {
        tmem_ld_32x32b_x32(lane_base + (which ? kTdK : kTdV) + 32 * cc, v);
        tmem_ld_wait(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (kidx < p.Nkv) {
        uint4* out = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack2<BF16>(__uint_as_float(v[8 * j + 2 * e]) * mul,
                               __uint_as_float(v[8 * j + 2 * e + 1]) * mul);
          out[j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- dQ drain (one thread per d)
// *addr += v in global memory, done at L2 (no value returned).
__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

template <int D>
__device__ void dq_drain(const BwdParams& p, const BwdCta& cta, int i0, int n, uint32_t bars, uint32_t tmem,
                         int* status, volatile int* abort_flag) {
  using C = BwdCfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;
  const int t = wq * 32 + lane;  // d row of dQ^T = TMEM lane
  const bool live = t < D;       // warp-uniform: rows past d (zero padding for d = 64) are skipped
  const uint32_t tq = tmem + (static_cast<uint32_t>(wq * 32) << 16) + kTdP;
  for (int i = 0; i < n; ++i) {
    const bool got = mbar_wait(bar_addr(bars, C::kBarDQFull), i & 1, status, abort_flag,
                               kStatusTimeoutBwd);
    if (!__all_sync(0xffffffffu, got)) break;
    tc_fence_after();
    if (!live) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarDQEmpty));
      continue;
    }
    // The whole row of dQ^T into registers first, so the columns are free for dP(i+1) before
    // any reduction is issued.
    uint32_t a[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tq + 32 * c, a[c]);
    tmem_ld_wait_only();
#pragma unroll
    for (int c = 0; c < 4; ++c) reg_fence(a[c]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarDQEmpty));  // dP(i+1) may overwrite it
    // Accumulator row q (query q0 + q) is D contiguous floats: a warp adds 32 consecutive
    // ones per instruction.
    float* row = p.dq_acc + (static_cast<size_t>(cta.wrow0) + static_cast<size_t>(i0 + i) * kBQ) * D + t;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        red_add_f32(row, __uint_as_float(a[c][q]));
        row += D;
      }
  }
}

template <int D, bool BF16, bool VARLEN>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_sm100(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                 const BwdParams p_in, int* __restrict__ status) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::kBarOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::kAbortOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sgen + C::kTmemHolderOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // [B,H,N,d]: head by head, so the CTAs resident together share one head's Q, dO and dQ
  // accumulator in L2; within a head the heaviest first (key tile 0 meets the most causal
  // query tiles).  Packed: item it = blockIdx.x / H of the plan's list (sequence by
  // sequence, each sequence's key tiles heaviest first), head blockIdx.x % H; the launch
  // covers the most items there can be, so CTAs past the plan's count return at once.
  BwdParams p = p_in;
  BwdCta cta;
  int kt;
  if constexpr (!VARLEN) {
    cta.bh = blockIdx.x / p.n_ktiles;
    kt = blockIdx.x % p.n_ktiles;
    cta.q_tok0 = cta.k_tok0 = 0;
    cta.wrow0 = static_cast<long long>(cta.bh) * p.nq_pad;
  } else {
    const int it = blockIdx.x / p.H;
    if (it >= *p.vl_count) return;  // the whole CTA, before any barrier or TMEM use
    cta.bh = blockIdx.x - it * p.H;
    const int item = p.vl_items[it];
    const int b = item / p.n_ktiles;
    kt = item - b * p.n_ktiles;
    const int4 sq = p.vl_seqs[b];  // bounds-checked by the plan kernel
    cta.q_tok0 = sq.x;
    cta.k_tok0 = sq.z;
    p.Nq = sq.y;
    p.Nkv = sq.w;
    p.off = sq.w - sq.y;  // causal alignment bottom-right per sequence
    p.n_qtiles = (sq.y + kBQ - 1) / kBQ;
    cta.wrow0 = static_cast<long long>(cta.bh) * p.rows_max + p.vl_qpad[b];
  }
  const int k0 = kt * kBK;
  const int i0 = first_qtile(p, k0);
  const int n = p.n_qtiles - i0;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, C::kBarKV), 1);
    for (int s = 0; s < kStages; ++s) mbar_init(bar_addr(bars, C::kBarQFull + s), 1);
    mbar_init(bar_addr(bars, C::kBarDOFull), 1);
    mbar_init(bar_addr(bars, C::kBarDOFree), 1);
    mbar_init(bar_addr(bars, C::kBarSFull), 1);
    mbar_init(bar_addr(bars, C::kBarDPFull), 1);
    mbar_init(bar_addr(bars, C::kBarPReady), 8);     // one arrival per softmax warp
    mbar_init(bar_addr(bars, C::kBarDSReady), 8);
    mbar_init(bar_addr(bars, C::kBarDQFull), 1);
    mbar_init(bar_addr(bars, C::kBarDQEmpty), 4);    // one arrival per drain warp
    mbar_init(bar_addr(bars, C::kBarQFree), 1);
    mbar_init(bar_addr(bars, C::kBarDone), 1);
    mbar_init(bar_addr(bars, C::kBarFinished), 12);  // one per warp of warps 4-15
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (D == 64) {
    // The zero block of the padded K^T (16 KB, 32 bytes per thread), made visible to the
    // tensor core before any MMA can read it.
    uint4* z = reinterpret_cast<uint4*>(sgen + C::kZeroOff) + 2 * threadIdx.x;
    z[0] = make_uint4(0u, 0u, 0u, 0u);
    z[1] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tdo);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Each role runs to the end of the kernel on its own path: warps with different
  // register budgets never re-join.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSide));
    if (warp == 0) {
      if (lane == 0 && n > 0)
        producer<D, VARLEN>(&tq, &tk, &tv, &tdo, p, cta, k0, i0, n, sbase, bars, status, abort_flag);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<D, BF16>(n, sbase, bars, tmem, status, abort_flag);
      __syncwarp();
      // Release TMEM once every MMA is complete and warps 4-15 are done with it.
      drain_wait(bar_addr(bars, C::kBarFinished), 0);
      drain_wait(bar_addr(bars, C::kBarDone), 0);
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else if (warp >= 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsDrain));
    dq_drain<D>(p, cta, i0, n, bars, tmem, status, abort_flag);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarFinished));
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    softmax_grad<D, BF16, VARLEN>(p, cta, k0, i0, n, (warp - 4) >> 2, sgen, bars, tmem, status,
                                  abort_flag);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarFinished));
  }
}

// ---------------------------------------------------------------- packed-batch plan
// Builds what the packed backward's kernels read (one CTA, before them on the stream):
// every sequence's token ranges bounds-checked once (a range outside [0, total] or longer
// than the declared maximum is clamped and reported in the status word, as in the forward
// plan), its first workspace row (query rows padded to whole 128-row tiles, sequence after
// sequence; a sequence that would run past the workspace gets no query rows and is
// reported too), and the (sequence, key tile) items, sequence by sequence, key tiles in
// order (for a causal sequence, heaviest first).
constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) fa_bwd_varlen_plan(const BwdParams p,
                                                                    int* __restrict__ status) {
  __shared__ long long warp_q[kPlanThreads / 32];
  __shared__ int warp_k[kPlanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (p.B + kPlanThreads - 1) / kPlanThreads;  // sequences per thread
  const int b0 = min(p.B, tid * per), b1 = min(p.B, b0 + per);
  bool bad = false;
  long long q_sum = 0;
  int k_sum = 0;
  for (int b = b0; b < b1; ++b) {
    int q0 = p.cu_q[b], q1 = p.cu_q[b + 1], k0 = p.cu_k[b], k1 = p.cu_k[b + 1];
    if (q0 < 0 || q1 < q0 || q1 > p.total_q || q1 - q0 > p.Nq || k0 < 0 || k1 < k0 ||
        k1 > p.total_k || k1 - k0 > p.Nkv) {
      bad = true;
      q0 = min(max(q0, 0), p.total_q);
      q1 = min(max(q1, q0), min(p.total_q, q0 + p.Nq));
      k0 = min(max(k0, 0), p.total_k);
      k1 = min(max(k1, k0), min(p.total_k, k0 + p.Nkv));
    }
    p.vl_seqs[b] = make_int4(q0, q1 - q0, k0, k1 - k0);
    q_sum += static_cast<long long>((q1 - q0 + kBQ - 1) / kBQ) * kBQ;
    k_sum += (k1 - k0 + kBK - 1) / kBK;
  }
  // Exclusive prefix sums over the threads (sequence order) of the padded query rows and
  // the key tiles.
  long long q_inc = q_sum;
  int k_inc = k_sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long qn = __shfl_up_sync(0xffffffffu, q_inc, o);
    const int kn = __shfl_up_sync(0xffffffffu, k_inc, o);
    if (lane >= o) {
      q_inc += qn;
      k_inc += kn;
    }
  }
  if (lane == 31) {
    warp_q[warp] = q_inc;
    warp_k[warp] = k_inc;
  }
  __syncthreads();
  if (warp == 0) {
    long long qt = warp_q[lane];
    int kt = warp_k[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long qn = __shfl_up_sync(0xffffffffu, qt, o);
      const int kn = __shfl_up_sync(0xffffffffu, kt, o);
      if (lane >= o) {
        qt += qn;
        kt += kn;
      }
    }
    warp_q[lane] = qt;
    warp_k[lane] = kt;
  }
  __syncthreads();
  long long q_off = q_inc - q_sum + (warp > 0 ? warp_q[warp - 1] : 0);
  int k_off = k_inc - k_sum + (warp > 0 ? warp_k[warp - 1] : 0);
  for (int b = b0; b < b1; ++b) {
    int4 sq = p.vl_seqs[b];
    const long long padded = static_cast<long long>((sq.y + kBQ - 1) / kBQ) * kBQ;
    if (q_off + padded > p.rows_max) {  // overlapping ranges from bad offsets: no rows
      bad = true;
      sq.y = 0;
      p.vl_seqs[b] = sq;
    }
    p.vl_qpad[b] = static_cast<int>(min(q_off, p.rows_max));
    q_off += padded;
    const int nkt = (sq.w + kBK - 1) / kBK;
    for (int t = 0; t < nkt; ++t) p.vl_items[k_off + t] = b * p.n_ktiles + t;
    k_off += nkt;
  }
  if (tid == kPlanThreads - 1) {
    p.vl_qpad[p.B] = static_cast<int>(min(warp_q[31], p.rows_max));
    *p.vl_count = warp_k[31];
  }
  if (bad) atomicOr(status, kStatusBadInput);
}

// The sequence whose padded workspace rows hold row pr (qpad[0] = 0 <= pr < qpad[B]).
__device__ __forceinline__ int seq_of_row(const int* __restrict__ qpad, int B, long long pr) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (qpad[mid] <= pr) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// The O / dO / LSE row ([B,H,Nq]: b*h*Nq + q; packed: token * H + h) behind workspace row
// `row`, or -1 for a padding row (then *in is false past the rows in use).
template <bool VARLEN>
__device__ __forceinline__ long long source_row(const BwdParams& p, long long row, bool& in) {
  if constexpr (!VARLEN) {
    const long long bh = row / p.nq_pad, q = row - bh * p.nq_pad;
    return q < p.Nq ? bh * p.Nq + q : -1;
  } else {
    const long long h = row / p.rows_max, pr = row - h * p.rows_max;
    if (pr >= p.vl_qpad[p.B]) {
      in = false;
      return -1;
    }
    const int b = seq_of_row(p.vl_qpad, p.B, pr);
    const int4 sq = p.vl_seqs[b];
    const long long q = pr - p.vl_qpad[b];
    return q < sq.y ? (sq.x + q) * p.H + h : -1;
  }
}

// ---------------------------------------------------------------- prep and dQ conversion
// Per query row (D/8 threads, 16 bytes of O and dO each): D = dO . O, -LSE * log2(e), and
// the row's D floats of the dQ accumulator zeroed.  Rows past a sequence's queries
// (padding of its last query tile) get D = 0 and -inf, so their P is 0.
template <int D, bool BF16, bool VARLEN>
__global__ void __launch_bounds__(256)
    fa_bwd_prep(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                const float* __restrict__ lse, const BwdParams p) {
  constexpr int kTpr = D / 8;          // threads per row
  constexpr int kRpw = 32 / kTpr;      // rows per warp
  const long long rows = VARLEN ? static_cast<long long>(p.H) * p.rows_max
                                : static_cast<long long>(p.BH) * p.nq_pad;
  const int sub = threadIdx.x & (kTpr - 1);
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long base = kRpw * gw; base < rows; base += kRpw * nw) {
    const long long row = base + ((threadIdx.x & 31) / kTpr);
    bool in = row < rows;
    const long long src = in ? source_row<VARLEN>(p, row, in) : -1;
    float acc = 0.f;
    if (src >= 0) {
      const size_t e = static_cast<size_t>(src) * D + sub * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(o + e);
      const uint4 b = *reinterpret_cast<const uint4*>(dout + e);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float a0, a1, b0, b1;
        unpack2<BF16>(av[j], a0, a1);
        unpack2<BF16>(bv[j], b0, b1);
        acc = fmaf(a0, b0, acc);
        acc = fmaf(a1, b1, acc);
      }
    }
#pragma unroll
    for (int m = kTpr / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (!in) continue;
    if (sub == 0) {
      p.delta[row] = acc;
      p.nlse2[row] = src >= 0 ? -lse[src] * 1.4426950408889634f : -INFINITY;
    }
    float4* z = reinterpret_cast<float4*>(p.dq_acc + row * D) + sub * 2;
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ = scale * accumulator in the 16-bit type: 8 values (one 16-byte store) per thread per
// step, grid-stride over the accumulator's rows (padding rows are skipped).
template <int D, bool BF16, bool VARLEN>
__global__ void __launch_bounds__(256)
    fa_bwd_dq(uint16_t* __restrict__ dq, const BwdParams p) {
  const long long rows = VARLEN ? static_cast<long long>(p.H) * p.rows_max
                                : static_cast<long long>(p.BH) * p.nq_pad;
  const long long total = rows * (D / 8);
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = g / (D / 8);
    const int c8 = static_cast<int>(g - row * (D / 8));
    bool in = true;
    const long long dst = source_row<VARLEN>(p, row, in);
    if (dst < 0) continue;
    const float4* src = reinterpret_cast<const float4*>(p.dq_acc + row * D + 8 * c8);
    const float4 a = src[0], b = src[1];
    uint4 w;
    w.x = pack2<BF16>(a.x * p.scale, a.y * p.scale);
    w.y = pack2<BF16>(a.z * p.scale, a.w * p.scale);
    w.z = pack2<BF16>(b.x * p.scale, b.y * p.scale);
    w.w = pack2<BF16>(b.z * p.scale, b.w * p.scale);
    reinterpret_cast<uint4*>(dq + dst * D)[c8] = w;
  }
}

template <int D, bool BF16, bool VARLEN>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const void* o, const void* dout, const float* lse,
                     void* dq, const BwdParams& p, int sm_count, int* status, cudaStream_t stream) {
  auto kern = fa_bwd_sm100<D, BF16, VARLEN>;
  const cudaError_t config_err =
      configure_kernel(reinterpret_cast<const void*>(kern), BwdCfg<D>::kAlloc, kRegsLaunch);
  if (config_err != cudaSuccess) return config_err;
  cudaError_t e;
  if constexpr (VARLEN) {
    fa_bwd_varlen_plan<<<1, kPlanThreads, 0, stream>>>(p, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const long long rows = VARLEN ? static_cast<long long>(p.H) * p.rows_max
                                : static_cast<long long>(p.BH) * p.nq_pad;
  long long prep_blocks = (rows + 15) / 16;  // at least 16 rows per 256-thread block
  const long long cap = static_cast<long long>(sm_count) * 16;
  if (prep_blocks > cap) prep_blocks = cap;
  if (prep_blocks < 1) prep_blocks = 1;
  fa_bwd_prep<D, BF16, VARLEN><<<static_cast<int>(prep_blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // Packed: one CTA per (item, head) for the most items there can be (B * n_ktiles).
  const long long grid = VARLEN ? static_cast<long long>(p.B) * p.n_ktiles * p.H
                                : static_cast<long long>(p.BH) * p.n_ktiles;
  kern<<<static_cast<int>(grid), kThreads, BwdCfg<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  long long dq_blocks = (rows * (D / 8) + 255) / 256;
  if (dq_blocks > cap) dq_blocks = cap;
  if (dq_blocks < 1) dq_blocks = 1;
  fa_bwd_dq<D, BF16, VARLEN><<<static_cast<int>(dq_blocks), 256, 0, stream>>>(
      static_cast<uint16_t*>(dq), p);
  return cudaGetLastError();
}

}  // namespace

size_t backward_smem_bytes(int d) { return d == 64 ? BwdCfg<64>::kAlloc : BwdCfg<128>::kAlloc; }

cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const void* o, const void* dout,
                            const float* lse, void* dq, const BwdParams& p, int d, bool bf16,
                            int sm_count, int* status, cudaStream_t stream) {
#define FA_BWD_CASE(D_, B_, V_)                                                              \
  if (d == D_ && bf16 == B_ && (p.cu_q != nullptr) == V_)                                     \
    return launch_t<D_, B_, V_>(tq, tk, tv, tdo, o, dout, lse, dq, p, sm_count, status, stream);
  FA_BWD_CASE(128, true, false)
  FA_BWD_CASE(128, false, false)
  FA_BWD_CASE(64, true, false)
  FA_BWD_CASE(64, false, false)
  FA_BWD_CASE(128, true, true)
  FA_BWD_CASE(128, false, true)
  FA_BWD_CASE(64, true, true)
  FA_BWD_CASE(64, false, true)
#undef FA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa

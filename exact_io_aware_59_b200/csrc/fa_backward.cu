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
//    query tiles), and zeroes the fp32 dQ accumulator;
//  * fa_bwd_sm100: one CTA per (key tile of 128, b*h).  It walks the query tiles of 64 that
//    see its keys, keeps dK and dV for its keys in TMEM, and adds each step's dQ
//    contribution into the fp32 accumulator with one bulk reduce-add (done at L2);
//  * fa_bwd_dq: dQ = scale * accumulator, converted to the inputs' 16-bit type.
//
// fa_bwd_sm100 roles (512 threads; our design for tcgen05, with keys as the MMA's M so the
// per-key sums dK and dV stay in TMEM for the whole walk):
//  * warp 0 (one lane): TMA loads of K and V once, then Q, dO, -LSE*log2e and D of each
//    query tile into a 3-stage ring;
//  * warp 1 (one lane): tcgen05.mma issue, per query tile i (b = i % 2):
//        S^T  = K Q_i^T   (M 128 keys, N 64 queries, K = d)      into S[b]
//        dP^T = V dO_i^T  (same shape)                            into dP[b]
//        dV  += P^T dO_i  (A = P^T, 16-bit, from TMEM over S[b]; B = dO_i MN-major)
//        dK  += dS^T Q_i  (A = dS^T, 16-bit, from TMEM over dP[b]; B = Q_i MN-major)
//        dQ^T = K^T dS^T  (M 128 = d, N 64 queries, K 128 keys; A = K read MN-major,
//                          B = dS[b] from shared memory)          into dP[b], over dS^T
//    software-pipelined one tile deep: step i issues S(i+1), dP(i+1), then dV(i), dK(i),
//    dQ(i) once warpgroup b has delivered P(i) and dS(i); only dP(i+1) waits for dQ(i-1)
//    to be read out of dP[(i+1) % 2], and S(i+1) runs meanwhile.  The MMA lane is the
//    critical path (the tensor pipe's issue queue is shallow), so a tile costs it just
//    three waits and two commits: one commit covers S and dP, one covers the tile's last
//    product (its dQ is then ready and its Q/dO stage free);
//  * warpgroups 1 and 2 (warps 4-7 and 8-11) take the even and the odd query tiles, one
//    thread per key: P^T from S^T and dS^T from dP^T, each written back to TMEM as 16-bit,
//    dS also to shared memory.  With two, each has two tiles' time for one tile's work,
//    so P(i) and dS(i) are ready before the MMA lane asks for them (one warpgroup alone
//    measured about as fast, the MMA lane being the critical path).  At the end
//    warpgroup 1 writes dV and warpgroup 2 writes scale * dK;
//  * warpgroup 3 (warps 12-15), one thread per d-row of dQ^T: TMEM -> registers -> shared
//    memory -> bulk reduce-add into the accumulator tile of query tile i.
// Registers: the launch gives 128 per thread; warps 0-3 and 12-15 drop to kRegsSide and
// warpgroups 1 and 2 rise to kRegsSoftmax (setmaxnreg).
// TMEM (512 columns): dV [0,128) dK [128,256) S0 [256,320) S1 [320,384) dP0 [384,448)
// dP1 [448,512); dQ(i) overwrites dP[b] once dK(i) has read dS^T(i) from it.  tcgen05.mma
// operations run in issue order, so an MMA that overwrites columns an earlier MMA reads
// as its A operand needs no wait in between.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_device.cuh"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kD = 128;        // head dimension
constexpr int kBK = 128;       // keys per CTA (MMA M)
constexpr int kBQ = 64;        // queries per step (MMA N of S^T, dP^T, dQ^T)
constexpr int kStages = 3;     // Q / dO ring
constexpr int kThreads = 512;
constexpr int kRegsLaunch = 128;   // 65536 / 512
constexpr int kRegsSide = 96;      // warps 0-3 and 12-15
constexpr int kRegsSoftmax = 160;  // warps 4-11
static_assert(256 * kRegsSide + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");

struct BwdCfg {
  static constexpr int kKOff = 0;                           // K tile, 2 x (128 rows x 128 B)
  static constexpr int kVOff = kKOff + kBK * kD * 2;        // V tile
  static constexpr int kQOff = kVOff + kBK * kD * 2;        // Q stages, 2 x (64 x 128 B)
  static constexpr int kQBytes = kBQ * kD * 2;
  static constexpr int kdOOff = kQOff + kStages * kQBytes;  // dO stages
  static constexpr int kdSOff = kdOOff + kStages * kQBytes; // dS x2, 128 keys x 64 queries
  static constexpr int kdSBytes = kBK * kBQ * 2;
  static constexpr int kStgOff = kdSOff + 2 * kdSBytes;     // dQ^T staging, fp32 128 x 64
  static constexpr int kStgBytes = kD * kBQ * 4;
  static constexpr int kLseOff = kStgOff + kStgBytes;       // -LSE*log2e per stage
  static constexpr int kDelOff = kLseOff + kStages * kBQ * 4;  // D per stage
  static constexpr int kBarOff = kDelOff + kStages * kBQ * 4;
  // mbarriers
  static constexpr int kBarKV = 0;
  static constexpr int kBarFull = 1;                 // + stage
  static constexpr int kBarDPFull = 1 + kStages;     // + buffer: S(i) and dP(i) complete
  static constexpr int kBarDSFull = kBarDPFull + 2;  // + buffer
  static constexpr int kBarDQFull = kBarDSFull + 2;  // + buffer
  static constexpr int kBarDQEmpty = kBarDQFull + 2;
  static constexpr int kBarDone = kBarDQEmpty + 1;   // every MMA of the CTA complete
  static constexpr int kBarFinished = kBarDone + 1;  // warps 4-15 done with TMEM
  static constexpr int kNumBars = kBarFinished + 1;
  static constexpr int kTmemHolderOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemHolderOff + 4;
  static constexpr int kBytes = kAbortOff + 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(kdSOff % 1024 == 0 && kQOff % 1024 == 0 && kdOOff % 1024 == 0, "swizzle atoms");
};

// TMEM columns.
constexpr uint32_t kTdV = 0, kTdK = 128, kTS = 256, kTdP = 384;

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

// ---------------------------------------------------------------- producer (TMA)
__device__ void producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                         const CUtensorMap* tdo, const BwdParams& p, int bh, int k0, int i0,
                         int n, uint32_t sbase, uint32_t bars, int* status,
                         volatile int* abort_flag) {
  using C = BwdCfg;
  const uint32_t kv = bar_addr(bars, C::kBarKV);
  mbar_arrive_expect_tx(kv, 4 * kBK * 64 * 2);
#pragma unroll
  for (int sub = 0; sub < 2; ++sub) {
    tma_load_3d(sbase + C::kKOff + sub * kBK * 128, tk, kv, sub * 64, k0, bh);
    tma_load_3d(sbase + C::kVOff + sub * kBK * 128, tv, kv, sub * 64, k0, bh);
  }
  int issued = 0;
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    const int st = i % kStages;
    // The stage held tile i - 3, whose products are all complete once its dQ is.
    const int prev = i - kStages;
    if (prev >= 0 && !mbar_wait(bar_addr(bars, C::kBarDQFull + (prev & 1)), (prev >> 1) & 1, status,
                                abort_flag, kStatusTimeoutBwd)) {
      ok = false;
      break;
    }
    const uint32_t fb = bar_addr(bars, C::kBarFull + st);
    mbar_arrive_expect_tx(fb, 2 * C::kQBytes + 2 * kBQ * 4);
    const int q0 = (i0 + i) * kBQ;
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      tma_load_3d(sbase + C::kQOff + st * C::kQBytes + sub * kBQ * 128, tq, fb, sub * 64, q0, bh);
      tma_load_3d(sbase + C::kdOOff + st * C::kQBytes + sub * kBQ * 128, tdo, fb, sub * 64, q0, bh);
    }
    const size_t row = static_cast<size_t>(bh) * p.nq_pad + q0;
    bulk_load(sbase + C::kLseOff + st * kBQ * 4, p.nlse2 + row, kBQ * 4, fb);
    bulk_load(sbase + C::kDelOff + st * kBQ * 4, p.delta + row, kBQ * 4, fb);
    ++issued;
  }
  if (!ok) {
    // Let every copy still in flight land before the CTA's shared memory goes away.
    for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
      drain_wait(bar_addr(bars, C::kBarFull + i % kStages), (i / kStages) & 1);
    drain_wait(kv, 0);
  }
}

// ---------------------------------------------------------------- MMA issuer
template <bool BF16>
__device__ void mma_issuer(int n, uint32_t sbase, uint32_t bars, uint32_t tmem, int* status,
                           volatile int* abort_flag) {
  using C = BwdCfg;
  constexpr uint32_t idesc_s = make_idesc_f16(kBK, kBQ, BF16, false);       // S^T, dP^T
  constexpr uint32_t idesc_kv = make_idesc_f16(kBK, kD, BF16, true);        // dV, dK
  constexpr uint32_t idesc_q = make_idesc_f16_ab(kD, kBQ, BF16, true, true);  // dQ^T
  const uint64_t k_desc = make_sdesc_sw128(sbase + C::kKOff, 16, 1024);
  const uint64_t v_desc = make_sdesc_sw128(sbase + C::kVOff, 16, 1024);
  // K as the MN-major A of dQ^T: 64-row d blocks 128 x 128 B = 16 KB apart (LBO), 8-key
  // groups 1024 B apart (SBO); 16 keys per step.
  const uint64_t kt_desc = make_sdesc_sw128(sbase + C::kKOff, kBK * 128, 1024);
  // dS as the MN-major B of dQ^T: one 128-byte row of 64 queries per key.
  auto ds_desc = [&](int b) { return make_sdesc_sw128(sbase + C::kdSOff + b * C::kdSBytes, kBQ * 128, 1024); };
  auto q_kmaj = [&](int st) { return make_sdesc_sw128(sbase + C::kQOff + st * C::kQBytes, 16, 1024); };
  auto do_kmaj = [&](int st) { return make_sdesc_sw128(sbase + C::kdOOff + st * C::kQBytes, 16, 1024); };
  // Q and dO as MN-major B (d contiguous): d blocks 64 x 128 B = 8 KB apart, 16 queries
  // (2048 B) per step.
  auto q_mn = [&](int st) { return make_sdesc_sw128(sbase + C::kQOff + st * C::kQBytes, kBQ * 128, 1024); };
  auto do_mn = [&](int st) { return make_sdesc_sw128(sbase + C::kdOOff + st * C::kQBytes, kBQ * 128, 1024); };
  auto wait = [&](int b, uint32_t parity) {
    return mbar_wait_spin(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutBwd);
  };
  auto issue_st = [&](uint32_t d_col, uint64_t a, uint64_t b) {  // S^T or dP^T
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk)
      mma_ss(tmem + d_col, a + kmajor_step(kk, kBK), b + kmajor_step(kk, kBQ), idesc_s, kk > 0 ? 1u : 0u);
  };
  bool ok = n > 0 && wait(C::kBarKV, 0);  // with no query tile nothing is loaded
  if (ok && (ok = wait(C::kBarFull + 0, 0))) {
    issue_st(kTS, k_desc, q_kmaj(0));
    issue_st(kTdP, v_desc, do_kmaj(0));
    tc_commit(bar_addr(bars, C::kBarDPFull + 0));
  }
  for (int i = 0; i < n && ok; ++i) {
    const int b = i & 1, nb = b ^ 1, st = i % kStages;
    const int st1 = (i + 1) % kStages;
    if (i + 1 < n) {
      if (!(ok = wait(C::kBarFull + st1, ((i + 1) / kStages) & 1))) break;
      // S(i+1): S[nb] was last read by dV(i-1), issued earlier, and by warpgroup nb before
      // it signalled dS(i-1).
      issue_st(kTS + nb * kBQ, k_desc, q_kmaj(st1));
      // dP(i+1) into dP[nb], once dQ(i-1) has been read out of it.
      if (i > 0 && !(ok = wait(C::kBarDQEmpty, (i - 1) & 1))) break;
      tc_fence_after();
      issue_st(kTdP + nb * kBQ, v_desc, do_kmaj(st1));
      tc_commit(bar_addr(bars, C::kBarDPFull + nb));  // S(i+1) and dP(i+1)
    }
    // Warpgroup b has stored P(i) over S[b] and dS^T(i) over dP[b], and dS(i) in shared memory.
    if (!(ok = wait(C::kBarDSFull + b, (i >> 1) & 1))) break;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < kBQ / 16; ++kk)
      mma_ts(tmem + kTdV, tmem + kTS + b * kBQ + kk * 8, do_mn(st) + ((kk * 2048) >> 4), idesc_kv,
             (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < kBQ / 16; ++kk)
      mma_ts(tmem + kTdK, tmem + kTdP + b * kBQ + kk * 8, q_mn(st) + ((kk * 2048) >> 4), idesc_kv,
             (i > 0 || kk > 0) ? 1u : 0u);
    // dQ(i) over dP[b]: dS^T(i) there has been read by dK(i), issued above.
#pragma unroll
    for (int kk = 0; kk < kBK / 16; ++kk)
      mma_ss(tmem + kTdP + b * kBQ, kt_desc + ((kk * 2048) >> 4), ds_desc(b) + ((kk * 2048) >> 4),
             idesc_q, kk > 0 ? 1u : 0u);
    // Tile i's products are complete: its dQ can be drained and its stage reloaded.
    tc_commit(bar_addr(bars, C::kBarDQFull + b));
  }
  tc_commit(bar_addr(bars, C::kBarDone));
}

// ---------------------------------------------------------------- P and dS (one thread per key)
// Warpgroup `wg` (0 or 1) takes query tiles i = wg, wg + 2, ... and buffers [wg].
template <bool BF16>
__device__ void softmax_grad(const BwdParams& p, int bh, int k0, int i0, int n, int wg,
                             uint8_t* sgen, uint32_t bars, uint32_t tmem, int* status,
                             volatile int* abort_flag) {
  using C = BwdCfg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;
  const int r = wq * 32 + lane;  // key row of the tile = TMEM lane
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int kidx = k0 + r;
  // First query that sees this key (a key past the end is seen by none).
  const long long qvis = kidx >= p.Nkv ? (1ll << 40) : (p.causal ? static_cast<long long>(kidx) - p.off : -(1ll << 40));
  const bool key_tail = k0 + kBK > p.Nkv;
  const float sl2 = p.scale_log2;
  auto wait = [&](int b, uint32_t parity) {
    const bool ok = mbar_wait(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutBwd);
    return __all_sync(0xffffffffu, ok);
  };
  bool ok = true;
  for (int i = wg; i < n; i += 2) {
    const int buf = wg, st = i % kStages;
    const int q0 = (i0 + i) * kBQ;
    if (!(ok = wait(C::kBarFull + st, (i / kStages) & 1))) break;  // LSE_i and D_i visible
    if (!(ok = wait(C::kBarDPFull + buf, (i >> 1) & 1))) break;  // S(i) and dP(i)
    tc_fence_after();
    const uint32_t tS = lane_base + kTS + buf * kBQ;
    float pr[64];
    {
      uint32_t a[32], b[32];
      tmem_ld_32x32b_x32(tS, a);
      tmem_ld_32x32b_x32(tS + 32, b);
      tmem_ld_wait(a);
      reg_fence(b);
      const float4* nl = reinterpret_cast<const float4*>(sgen + C::kLseOff + st * kBQ * 4);
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
      const long long cm = qvis - q0;
      const int cmin = cm < 0 ? 0 : (cm > kBQ ? kBQ : static_cast<int>(cm));
#pragma unroll
      for (int c = 0; c < 64; ++c) pr[c] = (c >= cmin) ? pr[c] : 0.f;
    }
    {
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) pk[j] = pack2<BF16>(pr[2 * j], pr[2 * j + 1]);
      tmem_st_32x32b_x32(tS, pk);
    }
    tmem_st_wait();
    // A block boundary between the P pass and the dS pass (ok is true here): interleaving
    // the two needs more registers than this warpgroup's 160 and spills.
    if (!__all_sync(0xffffffffu, ok)) break;
    const float4* dl = reinterpret_cast<const float4*>(sgen + C::kDelOff + st * kBQ * 4);
    uint8_t* ds_row = sgen + C::kdSOff + buf * C::kdSBytes + r * 128;
    const uint32_t tdP = lane_base + kTdP + buf * kBQ;
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
      // dS^T over the first 32 dP columns (16-bit pairs), already read.
      tmem_st_32x32b_x16(tdP + 16 * h, pk);
      // dS for the dQ product: key row r, 16-byte chunk cc (queries 8cc..8cc+7) at chunk
      // position cc ^ (r & 7) (128-byte swizzle).
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = 4 * h + j;
        *reinterpret_cast<uint4*>(ds_row + ((cc ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      }
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarDSFull + buf));
  }

  // Epilogue: dV and scale * dK rows of this thread's key.
  bool have = n > 0;
  if (have) have = ok && wait(C::kBarDone, 0);
  if (n > 0 && !have) return;
  if (have) tc_fence_after();
  const size_t orow = (static_cast<size_t>(bh) * p.Nkv + kidx) * kD;
  {
    const int which = wg;  // warpgroup 1 writes dV, warpgroup 2 writes dK
    uint16_t* dst = static_cast<uint16_t*>(which ? p.dk : p.dv) + orow;
    const float mul = which ? p.scale : 1.f;
#pragma unroll 1
    for (int cc = 0; cc < kD / 32; ++cc) {
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
__device__ void dq_drain(const BwdParams& p, int bh, int i0, int n, uint8_t* sgen, uint32_t sbase,
                         uint32_t bars, uint32_t tmem, int* status, volatile int* abort_flag) {
  using C = BwdCfg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;
  const int t = wq * 32 + lane;  // d row of dQ^T = TMEM lane
  const bool leader = (t == 0);
  const uint32_t tq0 = tmem + (static_cast<uint32_t>(wq * 32) << 16) + kTdP;
  uint8_t* stg_row = sgen + C::kStgOff + t * (kBQ * 4);
  for (int i = 0; i < n; ++i) {
    if (leader) bulk_wait_read_all();  // the previous tile's reduce has read the staging
    const bool got = mbar_wait(bar_addr(bars, C::kBarDQFull + (i & 1)), (i >> 1) & 1, status, abort_flag,
                               kStatusTimeoutBwd);
    // One decision for the whole warpgroup, so no thread is left alone at a named barrier.
    if (!named_sync_and(1, 128, got)) break;
    tc_fence_after();
    const uint32_t tq = tq0 + (i & 1) * kBQ;
    uint32_t a[32], b[32];
    tmem_ld_32x32b_x32(tq, a);
    tmem_ld_32x32b_x32(tq + 32, b);
    tmem_ld_wait(a);
    reg_fence(b);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarDQEmpty));
    // Row t of the fp32 tile, 16-byte chunk c (queries 4c..4c+3) at position c ^ (t & 15).
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint32_t* s = c < 8 ? &a[4 * c] : &b[4 * (c - 8)];
      *reinterpret_cast<uint4*>(stg_row + ((c ^ (t & 15)) << 4)) = make_uint4(s[0], s[1], s[2], s[3]);
    }
    fence_proxy_async_smem();
    named_sync(1, 128);
    if (leader) {
      float* dst = p.dq_acc + (static_cast<size_t>(bh) * p.n_qtiles + i0 + i) * (kD * kBQ);
      bulk_reduce_add_f32(dst, sbase + C::kStgOff, C::kStgBytes);
      bulk_commit_group();
    }
  }
  if (leader) bulk_wait_all();
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_sm100(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                 const BwdParams p, int* __restrict__ status) {
  using C = BwdCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::kBarOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::kAbortOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sgen + C::kTmemHolderOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Head by head, so the CTAs resident together share one head's Q, dO and dQ
  // accumulator in L2; within a head the heaviest first (key tile 0 meets the most causal
  // query tiles).
  const int bh = blockIdx.x / p.n_ktiles, kt = blockIdx.x % p.n_ktiles;
  const int k0 = kt * kBK;
  const int i0 = first_qtile(p, k0);
  const int n = p.n_qtiles - i0;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, C::kBarKV), 1);
    for (int s = 0; s < kStages; ++s) mbar_init(bar_addr(bars, C::kBarFull + s), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_addr(bars, C::kBarDPFull + b), 1);
      mbar_init(bar_addr(bars, C::kBarDSFull + b), 4);  // one arrival per warp of warpgroup b+1
      mbar_init(bar_addr(bars, C::kBarDQFull + b), 1);
    }
    mbar_init(bar_addr(bars, C::kBarDQEmpty), 4);    // one arrival per warp of warpgroup 3
    mbar_init(bar_addr(bars, C::kBarDone), 1);
    mbar_init(bar_addr(bars, C::kBarFinished), 12);  // one per warp of warps 4-15
    *abort_flag = 0;
    fence_mbar_init();
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
  if (warp < 4 || warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSide));
    if (warp == 0) {
      if (lane == 0 && n > 0) producer(&tq, &tk, &tv, &tdo, p, bh, k0, i0, n, sbase, bars, status, abort_flag);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<BF16>(n, sbase, bars, tmem, status, abort_flag);
      __syncwarp();
      // Release TMEM once every MMA is complete and warps 4-15 are done with it.
      drain_wait(bar_addr(bars, C::kBarFinished), 0);
      drain_wait(bar_addr(bars, C::kBarDone), 0);
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    } else if (warp >= 12) {
      dq_drain(p, bh, i0, n, sgen, sbase, bars, tmem, status, abort_flag);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarFinished));
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    softmax_grad<BF16>(p, bh, k0, i0, n, (warp - 4) >> 2, sgen, bars, tmem, status, abort_flag);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarFinished));
  }
}

// ---------------------------------------------------------------- prep and dQ conversion
// Per query row (16 threads, 16 bytes of O and dO each): D = dO . O, -LSE * log2(e), and
// the row's 128 floats of the dQ accumulator zeroed.  Rows past Nq (padding of the last
// query tile) get D = 0 and -inf, so their P is 0.
template <bool BF16>
__global__ void __launch_bounds__(256)
    fa_bwd_prep(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                const float* __restrict__ lse, const BwdParams p) {
  const long long rows = static_cast<long long>(p.BH) * p.nq_pad;
  const int sub = threadIdx.x & 15;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long base = 2 * gw; base < rows; base += 2 * nw) {  // two rows per warp
    const long long row = base + ((threadIdx.x >> 4) & 1);
    const bool in = row < rows;
    const int bh = in ? static_cast<int>(row / p.nq_pad) : 0;
    const int q = in ? static_cast<int>(row % p.nq_pad) : 0;
    float acc = 0.f;
    if (in && q < p.Nq) {
      const size_t e = (static_cast<size_t>(bh) * p.Nq + q) * kD + sub * 8;
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
    for (int m = 8; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (!in) continue;
    if (sub == 0) {
      p.delta[row] = acc;
      p.nlse2[row] = q < p.Nq ? -lse[static_cast<size_t>(bh) * p.Nq + q] * 1.4426950408889634f : -INFINITY;
    }
    float4* z = reinterpret_cast<float4*>(p.dq_acc + row * kD) + sub * 2;
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// One block per (b*h, query tile): un-swizzles the tile's fp32 dQ^T accumulator through
// shared memory and writes scale * dQ rows in the 16-bit type.
template <bool BF16>
__global__ void __launch_bounds__(256)
    fa_bwd_dq(uint16_t* __restrict__ dq, const BwdParams p) {
  __shared__ float t[kBQ][kD + 1];
  const long long tile = blockIdx.x;
  const int bh = static_cast<int>(tile / p.n_qtiles), qt = static_cast<int>(tile % p.n_qtiles);
  const float4* src = reinterpret_cast<const float4*>(p.dq_acc + tile * (kD * kBQ));
  for (int f = threadIdx.x; f < kD * kBQ / 4; f += blockDim.x) {
    const float4 v = src[f];
    const int dd = f >> 4, qq = ((f & 15) ^ (dd & 15)) << 2;
    t[qq][dd] = v.x;
    t[qq + 1][dd] = v.y;
    t[qq + 2][dd] = v.z;
    t[qq + 3][dd] = v.w;
  }
  __syncthreads();
  for (int it = threadIdx.x; it < kBQ * kD / 8; it += blockDim.x) {
    const int qq = it >> 4, g = it & 15;
    const int q = qt * kBQ + qq;
    if (q >= p.Nq) continue;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = pack2<BF16>(t[qq][8 * g + 2 * e] * p.scale, t[qq][8 * g + 2 * e + 1] * p.scale);
    *reinterpret_cast<uint4*>(dq + (static_cast<size_t>(bh) * p.Nq + q) * kD + 8 * g) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <bool BF16>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const void* o, const void* dout, const float* lse,
                     void* dq, const BwdParams& p, int sm_count, int* status, cudaStream_t stream) {
  auto kern = fa_bwd_sm100<BF16>;
  const cudaError_t config_err =
      configure_kernel(reinterpret_cast<const void*>(kern), BwdCfg::kAlloc, kRegsLaunch);
  if (config_err != cudaSuccess) return config_err;
  const long long rows = static_cast<long long>(p.BH) * p.nq_pad;
  long long prep_blocks = (rows + 15) / 16;  // 16 rows per 256-thread block
  const long long cap = static_cast<long long>(sm_count) * 16;
  if (prep_blocks > cap) prep_blocks = cap;
  if (prep_blocks < 1) prep_blocks = 1;
  fa_bwd_prep<BF16><<<static_cast<int>(prep_blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(p.BH) * p.n_ktiles;
  kern<<<static_cast<int>(grid), kThreads, BwdCfg::kAlloc, stream>>>(tq, tk, tv, tdo, p, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long tiles = static_cast<long long>(p.BH) * p.n_qtiles;
  fa_bwd_dq<BF16><<<static_cast<int>(tiles), 256, 0, stream>>>(static_cast<uint16_t*>(dq), p);
  return cudaGetLastError();
}

}  // namespace

size_t backward_smem_bytes() { return BwdCfg::kAlloc; }

cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const void* o, const void* dout,
                            const float* lse, void* dq, const BwdParams& p, bool bf16,
                            int sm_count, int* status, cudaStream_t stream) {
  return bf16 ? launch_t<true>(tq, tk, tv, tdo, o, dout, lse, dq, p, sm_count, status, stream)
              : launch_t<false>(tq, tk, tv, tdo, o, dout, lse, dq, p, sm_count, status, stream);
}

}  // namespace fa

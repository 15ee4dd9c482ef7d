// fa_prefill.cu -- exact fused attention forward for Nq > 1 on sm_100a.
//
// The method ("FlashAttention" (fp-ai-systems), sections "The fix: tile through SRAM,
// fuse the passes" and "Online softmax: the enabling trick"; "FlashAttention 1-2-3"
// (myaihardware), sections "FlashAttention-1", "FlashAttention-2" and "The Math Behind
// the Online Softmax Trick"): each Q tile owns its output and walks the K/V tiles; the
// score tile S = Q K^T lives only on chip; a running row max m and running sum l let the
// partial output be rescaled as new tiles arrive; O is divided by l once at the end and
// written to HBM with the row's log-sum-exp.  Causal tiles beyond the diagonal are never
// loaded or computed; only tiles that straddle the diagonal or the key tail are masked.
//
// The B200 mapping (our design, not the pages' A100/H100 sketches):
//  * one persistent CTA per SM; a work unit is two 128-row Q tiles of one (b, h);
//  * warp 0 (one lane) streams Q and the K/V tiles with TMA (128-byte swizzle) into a
//    ring of shared-memory slots guarded by full/empty mbarriers;
//  * warp 1 (one lane) issues tcgen05.mma: S_t = Q_t K^T into TMEM (fp32, 128 columns),
//    then O_t += P_t V with P_t read from TMEM; the two Q tiles ping-pong so that one
//    tile's softmax overlaps the other tile's matrix products;
//  * warpgroups 1 and 2 run the softmax of tile 0 and tile 1, one thread per row: they
//    read S from TMEM, apply scale and mask, update (m, l), write P as 16-bit into the
//    S columns, rescale O in TMEM only when the max grows by more than kLazyLog2 (lazy), and
//    run the epilogue (O / l and LSE to global memory).
//  TMEM map (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256,256+d), O1 after it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_device.cuh"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr int BM = 128;  // query rows per tile (tcgen05 M)
constexpr int BN = 128;  // keys per tile (tcgen05 N of S, K of P V)
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsSide = 88;      // warpgroup 0 (load + MMA issue)
constexpr int kRegsSoftmax = 208;  // warpgroups 1 and 2; 128*88 + 256*208 == 384*168
static_assert(128 * kRegsSide + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
// Lazy rescale threshold in log2 units: the reference max m_used of a row moves only when
// a tile's max exceeds it by more than this, so p = 2^(x - m_used) <= 2^15, below the fp16
// maximum 65504 (bf16 and the fp32 O and l have far more range).  O and l share m_used,
// so the result is the same softmax whatever the lag.
constexpr float kLazyLog2 = 15.0f;

// Slots of the ring through which a packed batch's claimed units reach the CTA's roles.
constexpr int kUnitSlots = 4;
// Arrivals that free a slot: the MMA lane and the eight softmax warps.
constexpr int kUnitReaders = 9;

template <int D>
struct PrefillCfg {
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kStages = (D == 128) ? 5 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kQBytes;
  static constexpr int kBarOff = kRingOff + kStages * kKVBytes;
  // mbarriers
  static constexpr int kBarQFull = 0;
  static constexpr int kBarQEmpty = 1;
  static constexpr int kBarFull = 2;                 // + slot
  static constexpr int kBarEmpty = 2 + kStages;      // + slot
  static constexpr int kBarSFull = 2 + 2 * kStages;  // + tile
  static constexpr int kBarPFull = kBarSFull + 2;    // + 2 * tile + half (keys 0-63, 64-127)
  static constexpr int kBarOHalf = kBarPFull + 4;    // + tile: P V over the first 64 keys done
  static constexpr int kBarODone = kBarOHalf + 2;    // + tile
  static constexpr int kBarDrain = kBarODone + 2;
  static constexpr int kBarDone = kBarDrain + 1;     // softmax warps finished with TMEM
  static constexpr int kBarUnitFull = kBarDone + 1;  // + slot: a claimed unit published
  static constexpr int kBarUnitEmpty = kBarUnitFull + kUnitSlots;  // + slot: read by all
  // Interleaved-K/V units: both warpgroups' row statistics published, then both done
  // reading the two partial outputs (one arrival per softmax warp each).
  static constexpr int kBarStats = kBarUnitEmpty + kUnitSlots;
  static constexpr int kBarMerged = kBarStats + 1;
  static constexpr int kNumBars = kBarMerged + 1;
  static constexpr int kTmemHolderOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemHolderOff + 4;
  static constexpr int kUnitOff = kAbortOff + 4;     // the claimed-unit ring (packed batches)
  static constexpr int kBytes = kUnitOff + 4 * kUnitSlots;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static_assert(kAlloc <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t bars, int i) { return bars + 8u * i; }

template <bool SPLIT>
__device__ __forceinline__ void unit_coords(const PrefillParams& p, int u, int& bh, int& pair,
                                            int& split) {
  // Heaviest first: the last Q-tile pairs (most causal work) of every head go first.
  if constexpr (!SPLIT) {
    pair = p.n_pairs - 1 - u / p.BH;
    bh = u % p.BH;
    split = 0;
  } else {
    const int per_pair = p.BH * p.n_splits;  // every head's parts of one pair
    pair = p.n_pairs - 1 - u / per_pair;
    const int rem = u % per_pair;
    split = rem / p.BH;
    bh = rem % p.BH;
  }
}

// The unit a CTA takes in round r of the persistent loop.  Units are numbered heaviest
// first; rounds deal them out in alternating directions ("snake"), so a CTA that got a heavy
// unit in one round gets a light one in the next.  For causal prefill this keeps the
// busiest SM within about 2% of the mean (plain round robin: about 14%).  Every role of the
// CTA walks the same sequence.
__device__ __forceinline__ int unit_of_round(int r) {
  const int G = gridDim.x, c = blockIdx.x;
  return r * G + ((r & 1) ? (G - 1 - c) : c);
}

// Packed batches are listed sequence by sequence (so that the CTAs running together share
// one sequence's K and V in L2), an order the static snake balances poorly on ragged
// lengths (busiest CTA about 7% above the mean on a batch of lengths 512-8192, against
// 0.3% for claiming in list order).  So their units are claimed from a work counter: the
// producer lane takes the next unit with one atomicAdd (which also bounds how far it runs
// ahead) and publishes it in a shared-memory ring slot; the MMA lane and the softmax warps
// read the slots in the same order and free them.  A unit index >= the unit count ends
// every role's loop.  Which CTA runs a unit changes no result: a unit's rows depend on
// its inputs alone.
__device__ __forceinline__ int ld_shared_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void st_shared_s32(uint32_t addr, int v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_shared_f4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ int claim_unit(const PrefillParams& p, uint32_t full_bar,
                                          uint32_t empty_bar, uint32_t ring, int rnd,
                                          int* status, volatile int* abort_flag, bool& ok) {
  const int slot = rnd % kUnitSlots;
  if (!mbar_wait(empty_bar + 8u * slot, ((rnd / kUnitSlots) & 1) ^ 1, status, abort_flag,
                 kStatusTimeoutLoad)) {
    ok = false;
    return 0;
  }
  const int u = atomicAdd(p.vl_next, 1);
  st_shared_s32(ring + 4u * slot, u);
  mbar_arrive(full_bar + 8u * slot);  // release: waiters that see the phase see the slot
  return u;
}

// One work unit: its (b*H + h, Q-tile pair) and the sequence it belongs to.
struct Unit {
  int bh, pair;
  int split;   // part of the K/V range (K/V-split launches; 0 otherwise)
  int Lq, Lk;  // queries and keys of the sequence
  int q0, k0;  // first query / key token of the sequence (packed layout)
  int h;       // head within the sequence (packed layout)
};

// Work units of the launch.  A packed batch's count was written on the device by the plan
// kernel (fa_varlen_plan) that ran before this kernel on the same stream.
template <bool VARLEN>
__device__ __forceinline__ int unit_count(const PrefillParams& p) {
  if constexpr (VARLEN) return *p.vl_count * p.H;
  return p.n_units;
}

template <bool VARLEN, bool SPLIT = false>
__device__ __forceinline__ Unit unit_of(const PrefillParams& p, int u) {
  Unit x;
  x.split = 0;
  if constexpr (!VARLEN) {
    unit_coords<SPLIT>(p, u, x.bh, x.pair, x.split);
    x.Lq = p.Nq;
    x.Lk = p.Nkv;
    x.q0 = x.k0 = x.h = 0;
  } else {
    // Sequence b's units are H * np_b consecutive indices from H * first[b], head-major:
    // every pair of head 0 (last pair first), then of head 1, ...  So the CTAs running
    // together work on all pairs of a few heads and share those heads' K and V in L2.
    // u / H falls inside b's own item range, which names b.  The sequence's ranges were
    // bounds-checked by the plan kernel.
    const int b = p.vl_items[u / p.H] / p.n_pairs;
    const int4 sq = p.vl_seqs[b];
    const int np = ((sq.y + BM - 1) / BM + 1) / 2;  // Q-tile pairs of the sequence (>= 1)
    const int local = u - p.H * p.vl_first[b];
    x.h = local / np;
    x.pair = np - 1 - (local - x.h * np);
    x.bh = b * p.H + x.h;
    x.q0 = sq.x;
    x.Lq = sq.y;
    x.k0 = sq.z;
    x.Lk = sq.w;
  }
  return x;
}

// Q tile t (0 or 1) of Q-tile pair `pair`: tiles 2*pair and 2*pair+1.  In a small launch
// (p.n_splits == 0, instantiation kPairKVI) a unit is one Q tile instead (`pair` names
// it), shared by both "tiles" t, which take its even (t = 0) and odd (t = 1) K/V tiles:
// with a CTA per Q-tile pair the heaviest pair's serial chain of K/V steps set the
// launch's time (in a causal launch most of its steps had only one tile left).  Packed
// batches, K/V-split and FP8 launches always pair adjacent tiles.
constexpr int kPairAdjacent = 0, kPairKVI = 1;
template <int PAIR>
__device__ __forceinline__ int qtile_of(const PrefillParams& p, int pair, int t) {
  return PAIR == kPairKVI ? pair : 2 * pair + t;
}

// Number of K/V tiles Q tile `qtile` of unit x must visit (0 when every row is fully
// masked or the tile lies past the sequence's queries).
__device__ __forceinline__ int kv_tiles_for(const PrefillParams& p, const Unit& x, int qtile) {
  if (qtile * BM >= x.Lq) return 0;
  const int ntk = (x.Lk + BN - 1) / BN;
  if (!p.causal) return ntk;
  const int last_row = min(qtile * BM + BM - 1, x.Lq - 1);
  const int last_key = last_row + x.Lk - x.Lq;  // bottom-right alignment per sequence
  if (last_key < 0) return 0;
  return min(ntk, last_key / BN + 1);
}

// The K/V tiles [j0, j1) unit x visits, of the [0, nmax) its Q-tile pair needs: all of them,
// or (K/V-split launches) its split's consecutive part.  Tile t of the pair then visits
// [j0, min(j1, n_t)).
template <bool SPLIT>
__device__ __forceinline__ void kv_range(const PrefillParams& p, const Unit& x, int nmax, int& j0,
                                         int& j1) {
  if constexpr (!SPLIT) {
    j0 = 0;
    j1 = nmax;
  } else {
    // nmax < 2^24 (a key count over 128) and n_splits <= 64: the products fit an int.
    j0 = x.split * nmax / p.n_splits;
    j1 = (x.split + 1) * nmax / p.n_splits;
  }
}

// TMA coordinates (beyond the 64-column block) of the tile whose first row is `first`
// (a query row or a key row of the unit's sequence): (row, b*H + h) in the [B,H,N,d]
// view, (h, token) in the packed [tokens, H, d] view.
template <bool VARLEN>
__device__ __forceinline__ void tile_coords(const PrefillParams& p, const Unit& x, int first,
                                            bool query, int& c1, int& c2) {
  if constexpr (!VARLEN) {
    c1 = first;
    c2 = x.bh;
  } else {
    c1 = x.h;
    c2 = (query ? x.q0 : x.k0) + first;
  }
}

// Waits for TMA loads already issued, ignoring the abort flag (error path only).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
}

// ---------------------------------------------------------------- producer (TMA)
template <int D, bool VARLEN, bool QK8, bool SPLIT, int PAIR>
__device__ void producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                         const PrefillParams& p, uint32_t sbase, uint32_t bars, int* status,
                         volatile int* abort_flag) {
  using C = PrefillCfg<D>;
  constexpr int S = C::kStages;
  uint32_t ld = 0, q_issued = 0;
  bool ok = true;
  const int n_units = unit_count<VARLEN>(p);
  for (int rnd = 0;; ++rnd) {
    const int u = VARLEN ? claim_unit(p, bar_addr(bars, C::kBarUnitFull),
                                      bar_addr(bars, C::kBarUnitEmpty), sbase + C::kUnitOff,
                                      rnd, status, abort_flag, ok)
                         : unit_of_round(rnd);
    if (!ok || u >= n_units) break;
    const Unit x = unit_of<VARLEN, SPLIT>(p, u);
    const int pair = x.pair;
    int n0 = kv_tiles_for(p, x, qtile_of<PAIR>(p, pair, 0)), n1 = kv_tiles_for(p, x, qtile_of<PAIR>(p, pair, 1));
    if constexpr (PAIR == kPairKVI) n1 = 0;  // one Q tile; its K/V tiles stream in order
    int j0 = 0, j1 = max(n0, n1);
    if constexpr (SPLIT) {
      kv_range<SPLIT>(p, x, j1, j0, j1);
      n0 = (min(j1, n0) > j0) ? n0 : 0;  // a tile with nothing in this part loads no Q
      n1 = (min(j1, n1) > j0) ? n1 : 0;
    }
    if (j1 <= j0) continue;
    if (!mbar_wait(bar_addr(bars, C::kBarQEmpty), (q_issued & 1) ^ 1, status, abort_flag,
                   kStatusTimeoutLoad)) {
      ok = false;
      break;
    }
    const uint32_t qf = bar_addr(bars, C::kBarQFull);
    constexpr uint32_t kQLoad = QK8 ? BM * 128 : C::kQBytes;
    mbar_arrive_expect_tx(qf, ((n0 > 0) + (n1 > 0)) * kQLoad);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if ((t == 0 ? n0 : n1) == 0) continue;
      int c1, c2;
      tile_coords<VARLEN>(p, x, qtile_of<PAIR>(p, pair, t) * BM, true, c1, c2);
      if constexpr (QK8) {
        tma_load_3d(sbase + C::kQOff + t * C::kQBytes, tq, qf, 0, c1, c2);
      } else {
#pragma unroll
        for (int sub = 0; sub < D / 64; ++sub)
          tma_load_3d(sbase + C::kQOff + t * C::kQBytes + sub * BM * 128, tq, qf, sub * 64, c1, c2);
      }
    }
    ++q_issued;
    for (int j = j0; j < j1 && ok; ++j) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t slot = ld % S, ph = (ld / S) & 1;
        if (!mbar_wait(bar_addr(bars, C::kBarEmpty + slot), ph ^ 1, status, abort_flag,
                       kStatusTimeoutLoad)) {
          ok = false;
          break;
        }
        const uint32_t fb = bar_addr(bars, C::kBarFull + slot);
        const bool k8 = QK8 && which == 0;
        mbar_arrive_expect_tx(fb, k8 ? BN * 128 : C::kKVBytes);
        const uint32_t dst = sbase + C::kRingOff + slot * C::kKVBytes;
        int c1, c2;
        tile_coords<VARLEN>(p, x, j * BN, false, c1, c2);
        if (k8) {
          tma_load_3d(dst, tk, fb, 0, c1, c2);
        } else {
#pragma unroll
          for (int sub = 0; sub < D / 64; ++sub)
            tma_load_3d(dst + sub * BN * 128, which ? tv : tk, fb, sub * 64, c1, c2);
        }
        ++ld;
      }
    }
  }
  if (!ok) {
    // Let every copy still in flight land before the CTA's shared memory goes away.
    for (uint32_t i = (ld > (uint32_t)S ? ld - S : 0); i < ld; ++i)
      drain_wait(bar_addr(bars, C::kBarFull + i % S), (i / S) & 1);
    if (q_issued) drain_wait(bar_addr(bars, C::kBarQFull), (q_issued - 1) & 1);
  }
}

// ---------------------------------------------------------------- MMA issuer
// Shared-memory descriptors are built once per buffer; an MMA step's operand is the
// buffer's descriptor plus (byte offset >> 4) in the start-address field (shared-memory
// addresses are below 2^18, so the 14-bit field never carries).
template <int D, bool QK8>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc,
                                        uint32_t idesc) {
  if constexpr (QK8) {
    // One-byte codes: a row is one 128-byte swizzle row; 32 elements (32 B) per step.
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk)
      mma_ss_f8(d_tmem, q_desc + ((kk * 32) >> 4), k_desc + ((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
    return;
  }
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    // K-major operand, 128-byte swizzle: 64-element column blocks of 128 rows x 128 B,
    // 16 elements (32 B) per MMA step; 8-row groups 1024 B apart.
    const uint32_t off16 = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
    mma_ss(d_tmem, q_desc + off16, k_desc + off16, idesc, kk > 0 ? 1u : 0u);
  }
}

// O += P V over keys 64*half .. 64*half+63 of the tile (four K=16 steps).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc,
                                         uint32_t idesc, bool accumulate, int half) {
#pragma unroll
  for (int kk = half * 4; kk < half * 4 + 4; ++kk) {
    // V is MN-major (d contiguous): 16 keys per step = two 1024-byte swizzle atoms;
    // the second 64-column block of d lies BN*128 bytes further (the descriptor's LBO).
    mma_ts(d_tmem, p_tmem + kk * 8, v_desc + ((kk * 16 * 128) >> 4), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool BF16, bool VARLEN, bool QK8, bool SPLIT, int PAIR>
__device__ void mma_issuer(const PrefillParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                           int* status, volatile int* abort_flag) {
  using C = PrefillCfg<D>;
  constexpr int S = C::kStages;
  constexpr uint32_t idesc_s = QK8 ? make_idesc_e4m3(BM, BN) : make_idesc_f16(BM, BN, BF16, false);
  constexpr uint32_t idesc_o = make_idesc_f16(BM, D, BF16, true);
  uint32_t ld = 0, q_used = 0, pcount[2] = {0, 0};
  bool ok = true;
  const uint64_t q_desc0 = make_sdesc_sw128(sbase + C::kQOff, 16, 1024);
  const uint64_t kv_desc0 = make_sdesc_sw128(sbase + C::kRingOff, 16, 1024);
  const uint64_t v_desc0 = make_sdesc_sw128(sbase + C::kRingOff, BN * 128, 1024);
  auto q_desc = [&](int t) { return q_desc0 + ((t * C::kQBytes) >> 4); };
  auto k_desc = [&](uint32_t slot) { return kv_desc0 + ((slot * C::kKVBytes) >> 4); };
  auto v_desc = [&](uint32_t slot) { return v_desc0 + ((slot * C::kKVBytes) >> 4); };
  auto wait = [&](int b, uint32_t parity) {
    return mbar_wait(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutMma);
  };
  const int n_units = unit_count<VARLEN>(p);
  for (int rnd = 0;; ++rnd) {
    int u;
    if constexpr (VARLEN) {
      const int slot = rnd % kUnitSlots;
      if (!wait(C::kBarUnitFull + slot, (rnd / kUnitSlots) & 1)) { ok = false; break; }
      u = ld_shared_s32(sbase + C::kUnitOff + 4u * slot);
      mbar_arrive(bar_addr(bars, C::kBarUnitEmpty + slot));
    } else {
      u = unit_of_round(rnd);
    }
    if (u >= n_units) break;
    const Unit x = unit_of<VARLEN, SPLIT>(p, u);
    if constexpr (PAIR == kPairKVI) {
      // One Q tile; K/V tile j goes to "tile" j & 1 (its S and O columns).  The ring holds
      // K_j at index 2j and V_j at 2j + 1 from this unit's first slot on.  Per j: P V_t(j),
      // then S_t(j + 2), so each warpgroup's next scores are ready while it finishes a tile.
      const int n = kv_tiles_for(p, x, x.pair);
      if (n <= 0) continue;
      if (!wait(C::kBarQFull, q_used & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t base = ld;
      auto slot = [&](int idx) { return (base + idx) % S; };
      auto full = [&](int idx) { return wait(C::kBarFull + slot(idx), ((base + idx) / S) & 1); };
      for (int t = 0; t < 2 && t < n && ok; ++t) {
        if (!full(2 * t)) { ok = false; break; }
        tc_fence_after();
        issue_s<D, QK8>(tmem + t * 128, q_desc(0), k_desc(slot(2 * t)), idesc_s);
        tc_commit(bar_addr(bars, C::kBarSFull + t));
        tc_commit(bar_addr(bars, C::kBarEmpty + slot(2 * t)));
      }
      if (!ok) break;
      if (n <= 2) tc_commit(bar_addr(bars, C::kBarQEmpty));  // every S of the unit issued
      for (int j = 0; j < n && ok; ++j) {
        const int t = j & 1;
        const uint32_t vslot = slot(2 * j + 1);
        if (!full(2 * j + 1)) { ok = false; break; }
        tc_fence_after();
        if (!mbar_wait_spin(bar_addr(bars, C::kBarPFull + 2 * t), pcount[t] & 1, status,
                            abort_flag, kStatusTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        issue_pv<D>(tmem + 256 + t * D, tmem + t * 128, v_desc(vslot), idesc_o, j >= 2, 0);
        tc_commit(bar_addr(bars, C::kBarOHalf + t));
        if (!mbar_wait_spin(bar_addr(bars, C::kBarPFull + 2 * t + 1), pcount[t] & 1, status,
                            abort_flag, kStatusTimeoutMma)) { ok = false; break; }
        ++pcount[t];
        tc_fence_after();
        issue_pv<D>(tmem + 256 + t * D, tmem + t * 128, v_desc(vslot), idesc_o, true, 1);
        tc_commit(bar_addr(bars, C::kBarODone + t));
        if (j + 2 < n) {
          if (!full(2 * (j + 2))) { ok = false; break; }
          tc_fence_after();
          issue_s<D, QK8>(tmem + t * 128, q_desc(0), k_desc(slot(2 * (j + 2))), idesc_s);
          tc_commit(bar_addr(bars, C::kBarSFull + t));
          tc_commit(bar_addr(bars, C::kBarEmpty + slot(2 * (j + 2))));
          if (j + 2 == n - 1) tc_commit(bar_addr(bars, C::kBarQEmpty));  // the unit's last S
        }
        tc_commit(bar_addr(bars, C::kBarEmpty + vslot));
      }
      if (!ok) break;
      ld = base + 2 * n;
      ++q_used;
      continue;
    }
    // n[t]: the end of tile t's K/V range in this unit (<= j0: nothing to do).
    int n[2] = {kv_tiles_for(p, x, qtile_of<PAIR>(p, x.pair, 0)), kv_tiles_for(p, x, qtile_of<PAIR>(p, x.pair, 1))};
    int j0 = 0, j1 = max(n[0], n[1]);
    if constexpr (SPLIT) {
      kv_range<SPLIT>(p, x, j1, j0, j1);
      n[0] = min(j1, n[0]);
      n[1] = min(j1, n[1]);
    }
    if (j1 <= j0) continue;
    if (!wait(C::kBarQFull, q_used & 1)) { ok = false; break; }
    tc_fence_after();
    // S_t(j0) for both tiles from K_j0.
    const uint32_t kslot0 = ld % S;
    if (!wait(C::kBarFull + kslot0, (ld / S) & 1)) { ok = false; break; }
    tc_fence_after();
    ++ld;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (n[t] <= j0) continue;
      issue_s<D, QK8>(tmem + t * 128, q_desc(t), k_desc(kslot0), idesc_s);
      tc_commit(bar_addr(bars, C::kBarSFull + t));
    }
    tc_commit(bar_addr(bars, C::kBarEmpty + kslot0));
    // The Q tiles are free once the last S that reads them completes: release them then,
    // so the next unit's Q load overlaps this unit's last softmax and P V products.
    if (j1 - j0 == 1) tc_commit(bar_addr(bars, C::kBarQEmpty));
    for (int j = j0; j < j1 && ok; ++j) {
      const uint32_t vslot = ld % S;
      if (!wait(C::kBarFull + vslot, (ld / S) & 1)) { ok = false; break; }
      tc_fence_after();
      ++ld;
      int knext = -1;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (j >= n[t]) continue;
        // P arrives in two halves (keys 0-63, then 64-127): the first half's products run
        // while the softmax is still exponentiating the second.
        if (!mbar_wait_spin(bar_addr(bars, C::kBarPFull + 2 * t), pcount[t] & 1, status,
                            abort_flag, kStatusTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        issue_pv<D>(tmem + 256 + t * D, tmem + t * 128, v_desc(vslot), idesc_o, j > j0, 0);
        tc_commit(bar_addr(bars, C::kBarOHalf + t));
        if (!mbar_wait_spin(bar_addr(bars, C::kBarPFull + 2 * t + 1), pcount[t] & 1, status,
                            abort_flag, kStatusTimeoutMma)) { ok = false; break; }
        ++pcount[t];
        tc_fence_after();
        issue_pv<D>(tmem + 256 + t * D, tmem + t * 128, v_desc(vslot), idesc_o, true, 1);
        tc_commit(bar_addr(bars, C::kBarODone + t));
        if (j + 1 < n[t]) {
          if (knext < 0) {
            knext = ld % S;
            if (!wait(C::kBarFull + knext, (ld / S) & 1)) { ok = false; break; }
            tc_fence_after();
            ++ld;
          }
          issue_s<D, QK8>(tmem + t * 128, q_desc(t), k_desc(knext), idesc_s);
          tc_commit(bar_addr(bars, C::kBarSFull + t));
        }
      }
      if (!ok) break;
      tc_commit(bar_addr(bars, C::kBarEmpty + vslot));
      if (knext >= 0) tc_commit(bar_addr(bars, C::kBarEmpty + knext));
      if (j == j1 - 2) tc_commit(bar_addr(bars, C::kBarQEmpty));  // last S was issued above
    }
    if (!ok) break;
    ++q_used;
  }
  // No MMA may still be running when the TMEM is released.
  tc_commit(bar_addr(bars, C::kBarDrain));
  drain_wait(bar_addr(bars, C::kBarDrain), 0);
}

// ---------------------------------------------------------------- softmax + epilogue
// Max (or min) of a row's 128 raw scores: eight independent chains of 3-input max.
template <bool MAX>
__device__ __forceinline__ float row_reduce(const uint32_t (&s)[4][32]) {
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = __uint_as_float(s[k >> 1][(k & 1) * 16]);
#pragma unroll
  for (int k = 0; k < 8; ++k)
#pragma unroll
    for (int i = 1; i < 16; i += 2) {
      const float a = __uint_as_float(s[k >> 1][(k & 1) * 16 + i]);
      const float b = (i + 1 < 16) ? __uint_as_float(s[k >> 1][(k & 1) * 16 + i + 1]) : a;
      acc[k] = MAX ? max3(acc[k], a, b) : min3(acc[k], a, b);
    }
  const float x = MAX ? max3(acc[0], acc[1], acc[2]) : min3(acc[0], acc[1], acc[2]);
  const float y = MAX ? max3(acc[3], acc[4], acc[5]) : min3(acc[3], acc[4], acc[5]);
  return MAX ? max3(x, y, fmaxf(acc[6], acc[7])) : min3(x, y, fminf(acc[6], acc[7]));
}

// p = 2^(s * scale_log2 - m) for 32 scores (tile columns col0 .. col0+31), rounded in
// pairs to the 16-bit type into pk; adds the unrounded p to the running sums, and with
// XMAX folds the exponents x = s * scale_log2 - m into two running maxima.  FULL: every
// column visible.  !FULL: columns past lim_c get p = 0.  Every 2^x goes to the SFU.
template <bool BF16, bool FULL, bool XMAX = false>
__device__ __forceinline__ void exp_pack32(const uint32_t (&s)[32], uint64_t sc2, uint64_t nm2,
                                           int col0, int lim_c, uint32_t (&pk)[16],
                                           uint64_t (&acc)[4], float (&xmax)[2]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), sc2, nm2);
    float x0, x1, p0, p1;
    f2_unpack(x2, x0, x1);
    if (XMAX) xmax[i & 1] = max3(xmax[i & 1], x0, x1);
    p0 = ex2(x0);
    p1 = ex2(x1);
    if (!FULL) {
      p0 = (col0 + 2 * i <= lim_c) ? p0 : 0.f;
      p1 = (col0 + 2 * i + 1 <= lim_c) ? p1 : 0.f;
    }
    pk[i] = pack2<BF16>(p0, p1);
    acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
  }
}

// P = 2^(s * scale_log2 - m_eff) for score chunks 2H and 2H+1 (keys 64H .. 64H+63 of the
// tile), stored as 16-bit pairs over S columns 32H .. 32H+31.  Returns the sum of the
// unrounded p and sets xh to the largest exponent s * scale_log2 - m_eff of those keys
// (-inf when none is visible).  all_visible: every column visible (else columns past lim_c
// get p = 0; their scores must already hold the masking sentinel).
template <bool BF16, int H>
__device__ __forceinline__ float exp_half(const uint32_t (&s)[4][32], uint64_t sc2, float m_eff,
                                          bool all_visible, int lim_c, uint32_t tS, float& xh) {
  const uint64_t nm2 = f2_pack(-m_eff, -m_eff);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int c = 2 * H; c < 2 * H + 2; ++c) {
    uint32_t pk[16];
    if (all_visible)
      exp_pack32<BF16, true, true>(s[c], sc2, nm2, 32 * c, lim_c, pk, acc, mx);
    else
      exp_pack32<BF16, false, true>(s[c], sc2, nm2, 32 * c, lim_c, pk, acc, mx);
    tmem_st_32x32b_x16(tS + 16 * c, pk);
  }
  xh = fmaxf(mx[0], mx[1]);
  float a0, a1;
  f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
  return a0 + a1;
}

// round16(p) - p for the largest p = 2^xh of a half tile (0 when xh = -inf).
template <bool BF16>
__device__ __forceinline__ float round_error(float xh) {
  if (xh == -INFINITY) return 0.f;
  const float pmax = ex2(xh);
  float r0, r1;
  unpack2<BF16>(pack2<BF16>(pmax, 0.f), r0, r1);
  return r0 - pmax;
}

// NEG: the scale is negative, so the row maximum of scale * s comes from the minimum of s.
// QK8: E4M3 queries and keys; with per-tile scales (p.q_tscale, p.k_tscale) each score
// tile's factor is scale * (its Q tile's scale) * (its K tile's scale).
// SPLIT: the unit covers part of its pair's K/V range; it writes fp32 O / l and the natural
// LSE of that part to o / lse, here the partial arrays (the combine kernel forms the result).
template <int D, bool BF16, bool OF32, bool NEG, bool VARLEN, bool QK8, bool SPLIT, int PAIR>
__device__ void softmax_epilogue(const PrefillParams& p, uint32_t bars, uint32_t tmem, void* o,
                                 float* lse, int t, int* status, volatile int* abort_flag) {
  using C = PrefillCfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = warp & 3;          // this warp reaches TMEM lanes 32*wq .. 32*wq+31
  const int r = wq * 32 + lane;     // row of the Q tile owned by this thread
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t tS = lane_base + t * 128;
  const uint32_t tO = lane_base + 256 + t * D;
  uint32_t s_seen = 0, o_seen = 0;
  uint32_t kvi_units = 0;  // interleaved-K/V units merged so far (the merge barriers' phase)
  // Warp-uniform result: tcgen05.ld/st below are warp-collective, so a warp never splits
  // on a wait that finished on some lanes and ran out on others.
  auto wait = [&](int b, uint32_t parity) {
    const bool ok = mbar_wait(bar_addr(bars, b), parity, status, abort_flag, kStatusTimeoutSoftmax);
    return __all_sync(0xffffffffu, ok);
  };

  const int n_units = unit_count<VARLEN>(p);
  for (int rnd = 0;; ++rnd) {
    int u;
    if constexpr (VARLEN) {
      const int slot = rnd % kUnitSlots;
      if (!wait(C::kBarUnitFull + slot, (rnd / kUnitSlots) & 1)) return;
      u = ld_shared_s32(bars - C::kBarOff + C::kUnitOff + 4u * slot);
      __syncwarp();  // every lane has read the slot before it is freed
      if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarUnitEmpty + slot));
    } else {
      u = unit_of_round(rnd);
    }
    if (u >= n_units) break;
    const Unit x = unit_of<VARLEN, SPLIT>(p, u);
    const int qtile = qtile_of<PAIR>(p, x.pair, t);
    if (qtile * BM >= x.Lq) continue;
    // This tile visits n_kv K/V tiles from tile j0 on (j0 = 0 unless the K/V range is
    // split); j below counts them from j0.
    int j0 = 0, n_kv = kv_tiles_for(p, x, qtile);
    if constexpr (PAIR == kPairKVI) n_kv = (n_kv + 1 - t) / 2;  // K/V tiles t, t + 2, ...
    if constexpr (SPLIT) {
      int j1;
      kv_range<SPLIT>(p, x, max(kv_tiles_for(p, x, qtile_of<PAIR>(p, x.pair, 0)), kv_tiles_for(p, x, qtile_of<PAIR>(p, x.pair, 1))),
                      j0, j1);
      n_kv = max(0, min(j1, n_kv) - j0);
    }
    const int row = qtile * BM + r;
    // Last key this row may see (keys beyond the sequence's are padding of its last tile,
    // or the next sequence's in a packed batch), counted from key tile j0's first key.
    const int limit = (p.causal ? min(x.Lk - 1, row + x.Lk - x.Lq) : x.Lk - 1) - j0 * BN;
    float m_used = -INFINITY;  // running max in log2 units (may lag the true max by <= 8)
    float l = 0.f;             // running sum of the 16-bit-rounded 2^(x - m_used): divides O
    float l_exact = 0.f;       // the same sum before rounding: gives LSE

    // O_t *= alpha for this thread's row (TMEM round trip; the rare lazy-rescale path).
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ob[32];
        tmem_ld_32x32b_x32(tO + cc * 32, ob);
        tmem_ld_wait(ob);
#pragma unroll
        for (int i = 0; i < 32; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * alpha);
        tmem_st_32x32b_x32(tO + cc * 32, ob);
      }
    };
    // Hands keys 64*h .. 64*h+63 of this tile's P (and any O rescale) to the MMA lane.
    auto release = [&](int h) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarPFull + 2 * t + h));  // one per warp
    };

    // The score factor in log2 units (per tile with per-tile FP8 scales).
    float sl2_q = p.scale_log2;
    if constexpr (QK8) {
      if (p.q_tscale) sl2_q *= p.q_tscale[static_cast<size_t>(x.bh) * p.n_qtiles + qtile];
    }
    for (int j = 0; j < n_kv; ++j) {
      float scale_log2 = sl2_q;
      if constexpr (QK8) {  // loaded before the wait, which hides its latency
        if (p.k_tscale) scale_log2 *= p.k_tscale[static_cast<size_t>(x.bh) * p.n_kvtiles + j0 + j];
      }
      if (!wait(C::kBarSFull + t, s_seen & 1)) return;
      ++s_seen;
      tc_fence_after();
      const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
      // columns c <= lim_c are visible for this row (K/V tile 2j + t with kPairKVI)
      const int lim_c = limit - (PAIR == kPairKVI ? 2 * j + t : j) * BN;
      const bool full = __all_sync(0xffffffffu, lim_c >= BN - 1);  // warp-uniform path
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + c * 32, s[c]);
      tmem_ld_wait_only();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(s[c]);
      // O and l are divided by, and LSE taken from, sums over P: l sums the 16-bit-rounded
      // P the P V product uses, taken as the unrounded sum plus the rounding error of each
      // half tile's largest P (the term that decides a row whose weight sits on a few keys;
      // the other terms' errors, relative 2^-9 for bf16 and 2^-12 for fp16 of either sign,
      // average out); l_exact sums the unrounded P.
      bool done = false;
      if (full && __all_sync(0xffffffffu, m_used != -INFINITY)) {
        // Once a row has a finite reference max, a tile with every column visible rarely
        // moves it: exponentiate against it straight away, taking each half's largest
        // exponent in the same pass, and hand each half of P to the MMA lane as soon as it
        // is known not to move the max of any row of the warp by more than kLazyLog2.
        float xa;
        const float ra = exp_half<BF16, 0>(s, sc2, m_used, true, lim_c, tS, xa);
        if (!__any_sync(0xffffffffu, xa > kLazyLog2)) {
          release(0);
          l += ra + round_error<BF16>(xa);
          l_exact += ra;
          float xb;
          const float rb = exp_half<BF16, 1>(s, sc2, m_used, true, lim_c, tS, xb);
          if (!__any_sync(0xffffffffu, xb > kLazyLog2)) {
            l += rb + round_error<BF16>(xb);
            l_exact += rb;
          } else {
            // Keys 64-127 move the max of some row of the warp after keys 0-63 went out
            // against the old reference: bring l and O (once P V over keys 0-63 is done)
            // to the new reference, then redo keys 64-127 against it.
            const bool move = xb > kLazyLog2;
            const float alpha = move ? ex2(-xb) : 1.0f;
            if (move) {
              l *= alpha;
              l_exact *= alpha;
              m_used += xb;
            }
            if (!wait(C::kBarOHalf + t, (o_seen + j) & 1)) return;
            tc_fence_after();
            rescale_o(alpha);
#pragma unroll
            for (int c = 2; c < 4; ++c) tmem_ld_32x32b_x32(tS + c * 32, s[c]);
            tmem_ld_wait_only();
#pragma unroll
            for (int c = 2; c < 4; ++c) reg_fence(s[c]);
            float xb2;
            const float rb2 = exp_half<BF16, 1>(s, sc2, m_used, true, lim_c, tS, xb2);
            l += rb2 + round_error<BF16>(xb2);
            l_exact += rb2;
          }
          done = true;
        }
      }
      if (!done) {
        // Two passes: the row max of the raw scores (masking what this row may not see),
        // then the exponents.  Nothing of this tile has been handed out yet.
        if (!full) {
          const float sentinel = NEG ? INFINITY : -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > lim_c) s[c][i] = __float_as_uint(sentinel);
        }
        const float mr = row_reduce<!NEG>(s);
        const float m_tile = (mr == INFINITY || mr == -INFINITY) ? -INFINITY : mr * scale_log2;
        const float m_new = fmaxf(m_used, m_tile);
        // Lazy rescale: move the reference max only when it grows by more than kLazyLog2.
        // -inf -> finite always moves; -inf -> -inf gives NaN and never moves.
        const bool move = (m_new - m_used) > kLazyLog2;
        const float alpha = move ? ex2(m_used - m_new) : 1.0f;
        if (move) {
          l *= alpha;
          l_exact *= alpha;
          m_used = m_new;
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // O_t holds P V of tiles < j (complete: S(j), ready above, was issued after it):
          // bring it to the new reference before this tile's P goes out.
          if (!wait(C::kBarODone + t, (o_seen + j - 1) & 1)) return;
          tc_fence_after();
          rescale_o(alpha);
        }
        const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
        float xa, xb;
        const float ra = exp_half<BF16, 0>(s, sc2, m_eff, full, lim_c, tS, xa);
        release(0);
        const float rb = exp_half<BF16, 1>(s, sc2, m_eff, full, lim_c, tS, xb);
        l += ra + rb + round_error<BF16>(xa) + round_error<BF16>(xb);
        l_exact += ra + rb;
      }
      release(1);
    }

    // Epilogue: O = O_t / l and LSE = (m + log2 l) * ln 2.
    if (n_kv > 0) {
      if (!wait(C::kBarODone + t, (o_seen + n_kv - 1) & 1)) return;
      tc_fence_after();
      o_seen += n_kv;
    }
    const bool valid = row < x.Lq;
    // Output row: (b*H + h, row) in [B,H,Nq,d]; (token, h) in the packed [tokens, H, d].
    const size_t orow_i = !VARLEN ? static_cast<size_t>(x.bh) * p.Nq + row
                                  : (static_cast<size_t>(x.q0) + row) * p.H + x.h;
    if constexpr (PAIR == kPairKVI) {
      // Both warpgroups hold a partial result of the same rows (O_t relative to their own
      // reference max m_t).  Merge: m = max(m_0, m_1), a_t = 2^(m_t - m), l = sum a_t l_t,
      // O = sum a_t O_t / l: the rule that combines two partial softmax sums ("FlashAttention
      // 1-2-3" (myaihardware), sections "The Math Behind the Online Softmax Trick" and
      // "Beyond FlashAttention", the reduction over K/V splits).
      // Each warpgroup publishes (m_t, l_t, l_exact_t, has O_t) in the unused second Q
      // buffer, then forms half of the columns from both O tiles; warpgroup 0 writes LSE.
      // The second barrier keeps either O tile from being overwritten by the next unit
      // before the other warpgroup has read it.
      const uint32_t stats = bars - C::kBarOff + C::kQOff + C::kQBytes;
      st_shared_f4(stats + 16u * (t * BM + r), m_used, l, l_exact, n_kv > 0 ? 1.f : 0.f);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarStats));
      if (!wait(C::kBarStats, kvi_units & 1)) return;
      tc_fence_after();  // the other warpgroup saw its O tile complete before arriving
      const float4 ot = ld_shared_f4(stats + 16u * ((1 - t) * BM + r));
      const bool has_s = n_kv > 0, has_o = ot.w != 0.f;
      const float ms = has_s ? m_used : -INFINITY, mo = has_o ? ot.x : -INFINITY;
      const float m = fmaxf(ms, mo);
      const float as = ms != -INFINITY ? ex2(ms - m) : 0.f;
      const float ao = mo != -INFINITY ? ex2(mo - m) : 0.f;
      const float lt = l * as + ot.y * ao, lt_exact = l_exact * as + ot.z * ao;
      const float inv_lt = (lt > 0.f) ? 1.0f / lt : 0.f;
      const uint32_t tOs = lane_base + 256 + t * D, tOo = lane_base + 256 + (1 - t) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 64; ++cc) {
        const int col = t * (D / 2) + cc * 32;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
#pragma unroll 1
        for (int side = 0; side < 2; ++side) {
          const bool has = side == 0 ? has_s : has_o;
          if (!has) continue;
          uint32_t ob[32];
          tmem_ld_32x32b_x32((side == 0 ? tOs : tOo) + col, ob);
          tmem_ld_wait(ob);
          const float a = side == 0 ? as : ao;
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = fmaf(__uint_as_float(ob[i]), a, v[i]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= inv_lt;
        if (valid) {
          if constexpr (OF32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o) + orow_i * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(o) + orow_i * D + col);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack2<BF16>(v[8 * i], v[8 * i + 1]), pack2<BF16>(v[8 * i + 2], v[8 * i + 3]),
                                  pack2<BF16>(v[8 * i + 4], v[8 * i + 5]), pack2<BF16>(v[8 * i + 6], v[8 * i + 7]));
          }
        }
      }
      if (t == 0 && valid && lse != nullptr)
        lse[orow_i] = (lt_exact > 0.f) ? (m + log2f(lt_exact)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(bars, C::kBarMerged));
      if (!wait(C::kBarMerged, kvi_units & 1)) return;
      tc_fence_after();
      ++kvi_units;
      continue;
    }
    const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
    if constexpr (SPLIT) {
      // This part's record: O / l in fp32 and the natural LSE (-inf: no visible key).
      const size_t prow = static_cast<size_t>(x.split) * p.BH * p.Nq + orow_i;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ob[32];
        if (n_kv > 0) {
          tmem_ld_32x32b_x32(tO + cc * 32, ob);
          tmem_ld_wait(ob);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ob[i] = 0u;
        }
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o) + prow * D + cc * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(ob[4 * i]) * inv_l, __uint_as_float(ob[4 * i + 1]) * inv_l,
                                 __uint_as_float(ob[4 * i + 2]) * inv_l, __uint_as_float(ob[4 * i + 3]) * inv_l);
        }
      }
      if (valid)
        lse[prow] =
            (l_exact > 0.f) ? (m_used + log2f(l_exact)) * 0.69314718055994531f : -INFINITY;
      continue;
    }
    const size_t orow = orow_i * D;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t ob[32];
      if (n_kv > 0) {
        tmem_ld_32x32b_x32(tO + cc * 32, ob);
        tmem_ld_wait(ob);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ob[i] = 0u;
      }
      if (valid) {
        if constexpr (OF32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o) + orow + cc * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(ob[4 * i]) * inv_l, __uint_as_float(ob[4 * i + 1]) * inv_l,
                                 __uint_as_float(ob[4 * i + 2]) * inv_l, __uint_as_float(ob[4 * i + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(o) + orow + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack2<BF16>(__uint_as_float(ob[8 * i + 2 * e]) * inv_l,
                                 __uint_as_float(ob[8 * i + 2 * e + 1]) * inv_l);
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    if (valid && lse != nullptr)
      lse[orow_i] =
          (l_exact > 0.f) ? (m_used + log2f(l_exact)) * 0.69314718055994531f : -INFINITY;
  }
}

template <int D, bool BF16, bool OF32, bool VARLEN, bool QK8, bool SPLIT, int PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    fa_prefill_sm100(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, void* __restrict__ o,
                     float* __restrict__ lse, const PrefillParams p, int* __restrict__ status) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::kBarOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::kAbortOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sgen + C::kTmemHolderOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, C::kBarQFull), 1);
    mbar_init(bar_addr(bars, C::kBarQEmpty), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_addr(bars, C::kBarFull + s), 1);
      mbar_init(bar_addr(bars, C::kBarEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_addr(bars, C::kBarSFull + t), 1);
      mbar_init(bar_addr(bars, C::kBarPFull + 2 * t), 4);      // one arrival per softmax warp
      mbar_init(bar_addr(bars, C::kBarPFull + 2 * t + 1), 4);
      mbar_init(bar_addr(bars, C::kBarOHalf + t), 1);
      mbar_init(bar_addr(bars, C::kBarODone + t), 1);
    }
    mbar_init(bar_addr(bars, C::kBarDrain), 1);
    mbar_init(bar_addr(bars, C::kBarDone), 256);
    for (int s = 0; s < kUnitSlots; ++s) {
      mbar_init(bar_addr(bars, C::kBarUnitFull + s), 1);
      mbar_init(bar_addr(bars, C::kBarUnitEmpty + s), kUnitReaders);
    }
    mbar_init(bar_addr(bars, C::kBarStats), 8);   // one arrival per softmax warp
    mbar_init(bar_addr(bars, C::kBarMerged), 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
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
      if (lane == 0) producer<D, VARLEN, QK8, SPLIT, PAIR>(&tq, &tk, &tv, p, sbase, bars, status, abort_flag);
    } else if (warp == 1) {
      if (lane == 0) mma_issuer<D, BF16, VARLEN, QK8, SPLIT, PAIR>(p, sbase, bars, tmem, status, abort_flag);
      __syncwarp();
      // Release TMEM once both softmax warpgroups have finished reading it.
      drain_wait(bar_addr(bars, C::kBarDone), 0);
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // (Per-tile FP8 scales are positive: they never change the score factor's sign.)
    if (p.scale_log2 < 0.f)
      softmax_epilogue<D, BF16, OF32, true, VARLEN, QK8, SPLIT, PAIR>(p, bars, tmem, o, lse, (warp - 4) >> 2, status, abort_flag);
    else
      softmax_epilogue<D, BF16, OF32, false, VARLEN, QK8, SPLIT, PAIR>(p, bars, tmem, o, lse, (warp - 4) >> 2, status, abort_flag);
    tc_fence_before();
    mbar_arrive(bar_addr(bars, C::kBarDone));
  }
}

// ---------------------------------------------------------------- packed-batch plan
// Builds the work list of a packed batch before the prefill kernel runs (one CTA): every
// sequence's token ranges are bounds-checked once (a range outside [0, total] or longer
// than the declared maximum is clamped and reported in the status word), and every
// (sequence, Q-tile pair) that holds query rows becomes one item.  Items are listed
// sequence by sequence, sequences with more Q-tile pairs first (a counting sort on that
// count; the order among sequences of one count is whatever the atomics give, which
// changes no result: a unit's rows do not depend on where it runs), and each sequence's
// pairs last-first (for a causal batch, its heaviest first).  The prefill kernel's CTAs
// claim the units of each sequence head by head (every pair of one head, then the next
// head), so the CTAs running at one time share the K and V of a few heads of one sequence
// in L2: on the benchmark's ragged batch K and V come from HBM about once (1.18 GB read
// for 1.16 GB of Q, K, V), against 2.4 times with the pairs of all heads interleaved and
// 6 times with a list sorted by item weight alone.  Claiming in list order keeps the CTAs
// balanced, since each sequence's and the batch's last units are its lightest.
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 2 * kPlanThreads;  // counts above kPlanBuckets - 1 share a bucket

__global__ void __launch_bounds__(kPlanThreads)
    fa_varlen_plan(const PrefillParams p, int B, int* __restrict__ count, int4* __restrict__ seqs,
                   int* __restrict__ first, int* __restrict__ items, int* __restrict__ status) {
  __shared__ int bucket[kPlanBuckets];
  __shared__ int warp_total[kPlanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool bad = false;
  for (int i = tid; i < kPlanBuckets; i += kPlanThreads) bucket[i] = 0;
  __syncthreads();
  // Clamped ranges; each sequence's pair count, summed per bucket (heaviest first).
  for (int b = tid; b < B; b += kPlanThreads) {
    int q0 = p.cu_q[b], q1 = p.cu_q[b + 1], k0 = p.cu_k[b], k1 = p.cu_k[b + 1];
    if (q0 < 0 || q1 < q0 || q1 > p.total_q || q1 - q0 > p.Nq || k0 < 0 || k1 < k0 ||
        k1 > p.total_k || k1 - k0 > p.Nkv) {
      bad = true;
      q0 = min(max(q0, 0), p.total_q);
      q1 = min(max(q1, q0), min(p.total_q, q0 + p.Nq));
      k0 = min(max(k0, 0), p.total_k);
      k1 = min(max(k1, k0), min(p.total_k, k0 + p.Nkv));
    }
    seqs[b] = make_int4(q0, q1 - q0, k0, k1 - k0);
    const int np = ((q1 - q0 + BM - 1) / BM + 1) / 2;  // Q-tile pairs holding query rows
    if (np > 0) atomicAdd(&bucket[kPlanBuckets - 1 - min(np, kPlanBuckets - 1)], np);
  }
  if (bad) atomicOr(status, kStatusBadInput);
  __syncthreads();
  // Exclusive prefix sum of the per-bucket item counts: thread t owns buckets 2t and 2t+1.
  const int c0 = bucket[2 * tid], c1 = bucket[2 * tid + 1];
  int incl = c0 + c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_total[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int t = warp_total[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    warp_total[lane] = t;
  }
  __syncthreads();
  const int excl = incl - (c0 + c1) + (warp > 0 ? warp_total[warp - 1] : 0);
  bucket[2 * tid] = excl;  // each thread rewrites only its own two buckets
  bucket[2 * tid + 1] = excl + c0;
  if (tid == kPlanThreads - 1) *count = excl + c0 + c1;
  if (tid == 0) *p.vl_next = 0;  // the prefill kernel's CTAs claim units from it
  __syncthreads();
  // Each sequence takes a contiguous range of the list.
  for (int b = tid; b < B; b += kPlanThreads) {
    const int np = ((seqs[b].y + BM - 1) / BM + 1) / 2;
    first[b] = np > 0 ? atomicAdd(&bucket[kPlanBuckets - 1 - min(np, kPlanBuckets - 1)], np) : 0;
  }
  __syncthreads();
  const long long n_items = static_cast<long long>(B) * p.n_pairs;
  for (long long i = tid; i < n_items; i += kPlanThreads) {
    const int b = static_cast<int>(i / p.n_pairs);
    const int pr = static_cast<int>(i - static_cast<long long>(b) * p.n_pairs);
    const int np = ((seqs[b].y + BM - 1) / BM + 1) / 2;
    if (pr < np) items[first[b] + (np - 1 - pr)] = static_cast<int>(i);  // last pair first
  }
}

// Merges the n_splits partial records of every output row (one warp per row, D / 32
// consecutive columns per lane): with w_s = exp(lse_s - max_s lse_s),
// O = sum_s w_s O_s / sum_s w_s and LSE = max_s lse_s + log(sum_s w_s).  A row no part saw
// a key of gets O = 0 and LSE = -inf.
constexpr int kCombineThreads = 256;

template <int D, bool BF16, bool OF32>
__global__ void __launch_bounds__(kCombineThreads)
    fa_prefill_combine(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                       void* __restrict__ o, float* __restrict__ lse, long long rows, int n_splits) {
  constexpr int V = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * (kCombineThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int c0 = (threadIdx.x & 31) * V;
  float m = -INFINITY;
  for (int sp = 0; sp < n_splits; ++sp) m = fmaxf(m, part_lse[sp * rows + row]);
  float acc[V], wsum = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  if (m != -INFINITY) {
    for (int sp = 0; sp < n_splits; ++sp) {
      const float ls = part_lse[sp * rows + row];
      const float w = (ls == -INFINITY) ? 0.f : expf(ls - m);
      wsum += w;
      const float* src = part_o + (sp * rows + row) * D + c0;
      float x[V];
      if constexpr (V == 4) {
        const float4 t = *reinterpret_cast<const float4*>(src);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(src);
        x[0] = t.x; x[1] = t.y;
      }
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = fmaf(w, x[i], acc[i]);
    }
  }
  const float inv = (wsum > 0.f) ? 1.0f / wsum : 0.f;
  if constexpr (OF32) {
    float* dst = static_cast<float*>(o) + row * D + c0;
    if constexpr (V == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
  } else {
    uint16_t* dst = static_cast<uint16_t*>(o) + row * D + c0;
    if constexpr (V == 4)
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack2<BF16>(acc[0] * inv, acc[1] * inv),
                                                  pack2<BF16>(acc[2] * inv, acc[3] * inv));
    else
      *reinterpret_cast<uint32_t*>(dst) = pack2<BF16>(acc[0] * inv, acc[1] * inv);
  }
  if (lse != nullptr && (threadIdx.x & 31) == 0)
    lse[row] = (wsum > 0.f) ? m + logf(wsum) : -INFINITY;
}

template <int D, bool BF16, bool OF32, bool VARLEN, bool QK8, bool SPLIT = false, int PAIR = kPairAdjacent>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                     float* lse, const PrefillParams& p, int grid, int* status,
                     cudaStream_t stream, float* part_o = nullptr, float* part_lse = nullptr) {
  // A split launch writes fp32 partial records whatever the output type.
  auto kern = fa_prefill_sm100<D, BF16, SPLIT ? false : OF32, VARLEN, QK8, SPLIT, PAIR>;
  const cudaError_t config_err =
      configure_kernel(reinterpret_cast<const void*>(kern), PrefillCfg<D>::kAlloc, kRegsLaunch);
  if (config_err != cudaSuccess) return config_err;
  if constexpr (SPLIT) {
    kern<<<grid, kThreads, PrefillCfg<D>::kAlloc, stream>>>(tq, tk, tv, part_o, part_lse, p, status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long rows = static_cast<long long>(p.BH) * p.Nq;
    const long long blocks = (rows + kCombineThreads / 32 - 1) / (kCombineThreads / 32);
    fa_prefill_combine<D, BF16, OF32><<<static_cast<unsigned>(blocks), kCombineThreads, 0, stream>>>(
        part_o, part_lse, o, lse, rows, p.n_splits);
  } else {
    kern<<<grid, kThreads, PrefillCfg<D>::kAlloc, stream>>>(tq, tk, tv, o, lse, p, status);
  }
  return cudaGetLastError();
}

}  // namespace

size_t prefill_smem_bytes(int d) {
  return d == 128 ? PrefillCfg<128>::kAlloc : PrefillCfg<64>::kAlloc;
}

cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           void* o, float* lse, const PrefillParams& p, int d, bool bf16,
                           bool o_f32, int grid, int* status, cudaStream_t stream, bool qk8,
                           float* part_o, float* part_lse) {
  if (qk8) {  // E4M3 queries and keys: d = 128, [B,H,N,d] layout
    if (d != 128 || p.cu_q) return cudaErrorInvalidValue;
    if (bf16 && o_f32) return launch_t<128, true, true, false, true>(tq, tk, tv, o, lse, p, grid, status, stream);
    if (bf16) return launch_t<128, true, false, false, true>(tq, tk, tv, o, lse, p, grid, status, stream);
    if (o_f32) return launch_t<128, false, true, false, true>(tq, tk, tv, o, lse, p, grid, status, stream);
    return launch_t<128, false, false, false, true>(tq, tk, tv, o, lse, p, grid, status, stream);
  }
  if (p.cu_q) {
    // Packed batch: the plan kernel writes the work list the prefill kernel reads.
    fa_varlen_plan<<<1, kPlanThreads, 0, stream>>>(p, p.BH / p.H, const_cast<int*>(p.vl_count),
                                                   const_cast<int4*>(p.vl_seqs),
                                                   const_cast<int*>(p.vl_first),
                                                   const_cast<int*>(p.vl_items), status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
#define FA_PREFILL_CASE(D_, B_, F_)                                                               \
  if (d == D_ && bf16 == B_ && o_f32 == F_)                                                        \
    return p.cu_q ? launch_t<D_, B_, F_, true, false>(tq, tk, tv, o, lse, p, grid, status, stream) \
           : p.n_splits > 1                                                                        \
               ? launch_t<D_, B_, F_, false, false, true>(tq, tk, tv, o, lse, p, grid, status, stream, \
                                                          part_o, part_lse)                        \
           : p.n_splits == 0                                                                      \
               ? launch_t<D_, B_, F_, false, false, false, kPairKVI>(tq, tk, tv, o, lse, p, grid,     \
                                                                     status, stream)                \
               : launch_t<D_, B_, F_, false, false>(tq, tk, tv, o, lse, p, grid, status, stream);
  FA_PREFILL_CASE(128, true, true)
  FA_PREFILL_CASE(128, true, false)
  FA_PREFILL_CASE(128, false, true)
  FA_PREFILL_CASE(128, false, false)
  FA_PREFILL_CASE(64, true, true)
  FA_PREFILL_CASE(64, true, false)
  FA_PREFILL_CASE(64, false, true)
  FA_PREFILL_CASE(64, false, false)
#undef FA_PREFILL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa

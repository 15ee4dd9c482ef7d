// fa_decode.cu -- split-KV attention for one query per head (decode), sm_100a.
//
// The method ("FlashAttention 1-2-3" (myaihardware), section "Beyond FlashAttention":
// FlashDecoding parallelises over the KV length, computes a partial softmax per chunk
// and then reduces; "Flash Attention -- Module 12.3", section "Prefill vs Decode": one
// query against a long KV cache): each split computes, over its own keys, the
// normalised partial output O_s and its log-sum-exp lse_s with the online softmax; a
// second kernel merges the splits:  M = max_s lse_s,  L = M + ln sum_s e^(lse_s - M),
// O = sum_s e^(lse_s - L) O_s.
//
// The B200 mapping: decode reads every K/V byte once, so it is bound by HBM bandwidth.
// All (b, h) heads' keys form one flat range of 64-key chunks; CTA c of G owns chunks
// [c*T/G, (c+1)*T/G), so every SM streams the same number of bytes whatever B*H and
// Nkv are.  One producer lane streams K and V chunks with bulk copies (L2 evict-first)
// into a ring of shared-memory stages; eight consumer warps each take 8 keys of every
// chunk: lanes split the head dimension for q.k (a transposing butterfly reduces 8 dot
// products in 9 shuffles), then each lane accumulates its own d-slice of P V in fp32.
// Each time a CTA finishes the part of a head it owns, every consumer warp writes one
// partial record (O_s, lse_s) for the keys it saw; the combine kernel merges them all.
//
// Paged KV cache ("FlashAttention 1-2-3" (myaihardware), section "Integration in Major
// Inference Engines"): the same kernels, with each head given the table's capacity of
// 64-key chunk slots.  A chunk's keys are gathered page by page (one bulk copy per page
// it touches) from [num_pages, H, page_size, d] caches through the block table; slots
// past a sequence's length are skipped by producer and consumers alike.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_device.cuh"
#include "fa_internal.h"

namespace fa {
namespace {

// Consumer warps: two groups of eight.  Stage i of the ring (the i-th chunk with keys) goes
// to group i % 2, whose warps take 8 keys each.  A warp's work on a chunk is a chain of
// dependent steps (shared-memory loads, a shuffle butterfly, the softmax update, P V), so
// two groups working on consecutive chunks at once keep the ring draining at the rate the
// copies arrive; with one group of eight the ring stayed full and the copies waited.
constexpr int kGroupWarps = 8;
constexpr int kWarps = 2 * kGroupWarps;       // consumer warps
constexpr int kThreads = (kWarps + 1) * 32;   // + one producer warp
constexpr int kKeysPerWarp = kDecodeChunk / kGroupWarps;
static_assert(kKeysPerWarp == 8, "the butterfly below reduces 8 keys per warp");
static_assert(kWarps == kDecodeRecords, "one partial record per consumer warp");

template <int D>
struct DecodeCfg {
  static constexpr int kChunkBytes = kDecodeChunk * D * 2;  // K or V part of a stage
  static constexpr int kStages = (D == 128) ? 6 : 10;
  static constexpr int kStageBytes = 2 * kChunkBytes;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kAbortOff = kBarOff + 2 * kStages * 8;
  static constexpr int kBytes = kAbortOff + 16;
  static_assert(kBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ long long chunk_begin(const DecodeParams& p, int cta) {
  return static_cast<long long>(cta) * p.total / p.grid;
}

// Chunk c of the flat range: its head, first key and number of keys (<= 0: an empty slot
// past the sequence's length).  With a paged cache the length comes from seq_lens,
// clamped to [0, capacity]; `flag` (the producer) records a clamp in the status word.
template <bool PAGED>
__device__ __forceinline__ void chunk_info(const DecodeParams& p, const PagedKV& pk, long long c,
                                           int& h, int& key0, int& nk, int* status, bool flag) {
  h = static_cast<int>(c / p.n_chunks);
  key0 = static_cast<int>(c % p.n_chunks) * kDecodeChunk;
  int len = p.Nkv;
  if constexpr (PAGED) {
    const int cap = pk.max_pages << pk.page_shift;
    len = pk.seq_lens[h / pk.H];
    if (len < 0 || len > cap) {
      if (flag) atomicOr(status, kStatusBadInput);
      len = len < 0 ? 0 : cap;
    }
  }
  nk = min(kDecodeChunk, len - key0);
}

// Waits (bounded, ignoring the abort flag) for the copies of the last S stages issued, so
// that none is still in flight when the CTA's shared memory goes away (error path only).
template <int S>
__device__ __forceinline__ void drain_ring(uint32_t bars, uint32_t ld) {
  for (uint32_t i = (ld > static_cast<uint32_t>(S) ? ld - S : 0); i < ld; ++i) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bars + 8 * (i % S), (i / S) & 1))
      if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
}

template <int D, bool BF16>
__device__ __forceinline__ void load_slice(const uint8_t* row, int lane, float (&x)[D / 32]) {
  constexpr int E = D / 32;  // elements per lane
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + lane * 8);
    unpack2<BF16>(u.x, x[0], x[1]);
    unpack2<BF16>(u.y, x[2], x[3]);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(row + lane * 4);
    unpack2<BF16>(u, x[0], x[1]);
  }
}

template <int D, bool BF16, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    fa_decode_split_sm100(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                          const uint16_t* __restrict__ v, float* __restrict__ part_o,
                          float* __restrict__ part_lse, const DecodeParams p, const PagedKV pk,
                          int* __restrict__ status) {
  using C = DecodeCfg<D>;
  constexpr int S = C::kStages;
  constexpr int E = D / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::kBarOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbortOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bars + 8 * s, 1);             // full: producer's expect_tx + bytes
      mbar_init(bars + 8 * (S + s), kGroupWarps);  // empty: one arrival per warp of its group
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const long long c_begin = chunk_begin(p, blockIdx.x);
  const long long c_end = chunk_begin(p, blockIdx.x + 1);

  if (warp == kWarps) {
    // ------------------------------------------------------------ producer
    if constexpr (!PAGED) {
      if (lane == 0) {
        const uint64_t policy = l2_policy_evict_first();
        uint32_t ld = 0;
        bool ok = true;
        for (long long c = c_begin; c < c_end; ++c) {
          int h, key0, nk;
          chunk_info<PAGED>(p, pk, c, h, key0, nk, status, true);
          if (nk <= 0) continue;
          const uint32_t bytes = static_cast<uint32_t>(nk) * D * 2;
          const uint32_t slot = ld % S;
          if (!mbar_wait(bars + 8 * (S + slot), ((ld / S) & 1) ^ 1, status, abort_flag,
                         kStatusTimeoutDecode)) {
            ok = false;
            break;
          }
          const uint32_t fb = bars + 8 * slot;
          mbar_arrive_expect_tx(fb, 2 * bytes);
          const uint32_t dst = sbase + slot * C::kStageBytes;
          const size_t off = (static_cast<size_t>(h) * p.Nkv + key0) * D;
          bulk_load_stream(dst, k + off, bytes, fb, policy);
          bulk_load_stream(dst + C::kChunkBytes, v + off, bytes, fb, policy);
          ++ld;
        }
        if (!ok) drain_ring<S>(bars, ld);
      }
    } else {
      // Paged cache: the whole warp.  Lane L looks up, 32 chunks ahead, the length and the
      // block-table entries of chunk base + L, so the table reads (dependent global loads)
      // are off the copy-issue path; then a chunk's K and V segments (one per page it
      // touches: 1, 2 or 4) are issued by one lane each, in parallel.
      const uint64_t policy = l2_policy_evict_first();
      const int ps = 1 << pk.page_shift;
      const int per_chunk = ps >= kDecodeChunk ? 1 : kDecodeChunk / ps;  // pages per chunk
      auto lookup = [&](long long c, int& nk, int (&pg)[4]) {
        nk = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) pg[e] = 0;
        if (c >= c_end) return;
        int h, key0;
        chunk_info<PAGED>(p, pk, c, h, key0, nk, status, true);
        const int b = h / pk.H;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + e * ps;
          if (e < per_chunk && key < key0 + nk) {
            int page = pk.block_table[static_cast<size_t>(b) * pk.max_pages + (key >> pk.page_shift)];
            if (page < 0 || page >= pk.num_pages) {
              atomicOr(status, kStatusBadInput);
              page = 0;
            }
            pg[e] = page;
          }
        }
      };
      int cur_nk, cur_pg[4], nxt_nk, nxt_pg[4];
      lookup(c_begin + lane, cur_nk, cur_pg);
      uint32_t ld = 0;
      bool ok = true;
      for (long long base = c_begin; base < c_end && ok; base += 32) {
        lookup(base + 32 + lane, nxt_nk, nxt_pg);  // in flight while this batch is issued
        const int batch = static_cast<int>(min(32ll, c_end - base));
        for (int i = 0; i < batch; ++i) {
          const int nk = __shfl_sync(0xffffffffu, cur_nk, i);
          if (nk <= 0) continue;  // empty slot: no stage, the consumers skip it too
          const long long c = base + i;
          const int h = static_cast<int>(c / p.n_chunks);
          const int key0 = static_cast<int>(c % p.n_chunks) * kDecodeChunk;
          const int hh = h % pk.H;
          const uint32_t slot = ld % S;
          const bool got = mbar_wait(bars + 8 * (S + slot), ((ld / S) & 1) ^ 1, status,
                                     abort_flag, kStatusTimeoutDecode);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          const uint32_t fb = bars + 8 * slot;
          if (lane == 0) mbar_arrive_expect_tx(fb, 2u * static_cast<uint32_t>(nk) * D * 2);
          __syncwarp();
          // Lane 2e copies the K segment in page e of the chunk, lane 2e + 1 its V segment.
          const int e = lane >> 1;
          int page = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int pj = __shfl_sync(0xffffffffu, cur_pg[j], i);
            if (j == e) page = pj;
          }
          const int key = key0 + e * ps;
          if (lane < 2 * per_chunk && key < key0 + nk) {
            const int in_page = key & (ps - 1);
            const int seg = min(key0 + nk - key, ps - in_page);
            const size_t off = ((static_cast<size_t>(page) * pk.H + hh) * ps + in_page) * D;
            const uint32_t so = static_cast<uint32_t>(key - key0) * D * 2;
            const uint32_t dst = sbase + slot * C::kStageBytes + (lane & 1) * C::kChunkBytes + so;
            bulk_load_stream(dst, ((lane & 1) ? v : k) + off, static_cast<uint32_t>(seg) * D * 2,
                             fb, policy);
          }
          ++ld;
        }
        cur_nk = nxt_nk;
#pragma unroll
        for (int e = 0; e < 4; ++e) cur_pg[e] = nxt_pg[e];
      }
      if (!ok && lane == 0) drain_ring<S>(bars, ld);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const long long first_head = c_begin / p.n_chunks;
    const int group = warp / kGroupWarps;  // takes the stages i with i % 2 == group
    const int slice = warp % kGroupWarps;  // keys 8 * slice .. 8 * slice + 7 of a chunk
    // Key (0..7 within this warp's 8) whose full dot product this lane ends up holding.
    const int my_key = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);

    float qv[E], acc[E];
    float m = -INFINITY, l_lane = 0.f;
    int cur_h = -1;
    int len = p.Nkv;  // keys of the current head's sequence
    uint32_t ld = 0;
    bool ok = true;

    // Writes this warp's partial record for head h: its keys' normalised output and
    // log-sum-exp.  No cross-warp synchronisation: the combine kernel merges the warps.
    auto finish_segment = [&](int h) {
      float l_w = l_lane;
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) l_w += __shfl_xor_sync(0xffffffffu, l_w, s);
      const long long rec =
          (static_cast<long long>(blockIdx.x) * p.max_seg + (h - first_head)) * kWarps + warp;
      const float inv = (l_w > 0.f) ? 1.0f / l_w : 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) part_o[rec * D + lane * E + e] = acc[e] * inv;
      if (lane == 0)
        part_lse[rec] = (l_w > 0.f) ? (m + log2f(l_w)) * 0.69314718055994531f : -INFINITY;
    };

    for (long long c = c_begin; c < c_end; ++c) {
      const int h = static_cast<int>(c / p.n_chunks);
      const int key0 = static_cast<int>(c % p.n_chunks) * kDecodeChunk;
      if (h != cur_h) {
        if (cur_h >= 0) finish_segment(cur_h);
        cur_h = h;
        if constexpr (PAGED) {
          // The sequence's length, clamped as the producer clamps it (the producer reports
          // a bad length); read once per head rather than once per chunk.
          const int cap = pk.max_pages << pk.page_shift;
          len = pk.seq_lens[h / pk.H];
          len = len < 0 ? 0 : (len > cap ? cap : len);
        }
        float qf[E];
        load_slice<D, BF16>(reinterpret_cast<const uint8_t*>(q + static_cast<size_t>(h) * D), lane, qf);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          qv[e] = qf[e] * p.scale_log2;  // scores come out in log2 units
          acc[e] = 0.f;
        }
        m = -INFINITY;
        l_lane = 0.f;
      }
      const int nk = min(kDecodeChunk, len - key0);
      // An empty slot still opens its head (so every segment gets its records), but has
      // no stage to read.
      if (nk <= 0) continue;
      const uint32_t slot = ld % S;
      const uint32_t phase = (ld / S) & 1;
      const bool mine = (ld & 1) == static_cast<uint32_t>(group);
      ++ld;
      if (!mine) continue;  // the other group's stage
      const bool got = mbar_wait(bars + 8 * slot, phase, status, abort_flag,
                                 kStatusTimeoutDecode);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const uint8_t* ks = smem + slot * C::kStageBytes + slice * kKeysPerWarp * D * 2;
      const uint8_t* vs = ks + C::kChunkBytes;

      // Partial dot products of this lane's d-slice with the warp's 8 keys.
      float part[8];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        float kx[E];
        load_slice<D, BF16>(ks + kk * D * 2, lane, kx);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) a = fmaf(qv[e], kx[e], a);
        part[kk] = a;
      }
      // Transposing butterfly: after it every lane holds the full score of key my_key.
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool up = lane & 16;
        const float keep = up ? part[i + 4] : part[i];
        const float send = up ? part[i] : part[i + 4];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const bool up = lane & 8;
        const float keep = up ? part[i + 2] : part[i];
        const float send = up ? part[i] : part[i + 2];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
      {
        const bool up = lane & 4;
        const float keep = up ? part[1] : part[0];
        const float send = up ? part[0] : part[1];
        part[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      part[0] += __shfl_xor_sync(0xffffffffu, part[0], 2);
      part[0] += __shfl_xor_sync(0xffffffffu, part[0], 1);
      const int nvalid = nk - slice * kKeysPerWarp;  // keys of this warp inside the chunk
      const float x = (my_key < nvalid) ? part[0] : -INFINITY;

      // Online softmax over the warp's keys (eager: one exp2 for alpha per chunk).
      float mx = x;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m, mx);
      const float m_eff = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m - m_eff);  // 0 when m was -inf
      const float pe = ex2(x - m_eff);
      l_lane = l_lane * alpha + (((lane & 3) == 0) ? pe : 0.f);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] *= alpha;
      m = m_new;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (kk >= nvalid) break;
        const int src = (((kk >> 2) & 1) << 4) | (((kk >> 1) & 1) << 3) | ((kk & 1) << 2);
        const float pk = __shfl_sync(0xffffffffu, pe, src);
        float vx[E];
        load_slice<D, BF16>(vs + kk * D * 2, lane, vx);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(pk, vx[e], acc[e]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (S + slot));
    }
    if (ok && cur_h >= 0) finish_segment(cur_h);
  }
  __syncthreads();
}

template <int D, bool OF32>
__global__ void __launch_bounds__(128)
    fa_decode_combine(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                      void* __restrict__ o, float* __restrict__ lse, const DecodeParams p) {
  const int h = blockIdx.x;
  const int c = threadIdx.x;
  // CTAs whose chunk ranges intersect head h's chunks [x0, x1].
  const long long x0 = static_cast<long long>(h) * p.n_chunks;
  const long long x1 = x0 + p.n_chunks - 1;
  auto cta_of = [&](long long x) {
    long long g = x * p.grid / p.total;
    while (g + 1 < p.grid && chunk_begin(p, static_cast<int>(g + 1)) <= x) ++g;
    while (g > 0 && chunk_begin(p, static_cast<int>(g)) > x) --g;
    return static_cast<int>(g);
  };
  const int lo = cta_of(x0), hi = cta_of(x1);
  float M = -INFINITY;
  for (int g = lo; g <= hi; ++g) {
    const long long rec0 = (static_cast<long long>(g) * p.max_seg + (h - chunk_begin(p, g) / p.n_chunks)) * kWarps;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, part_lse[rec0 + w]);
  }
  float L = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int g = lo; g <= hi; ++g) {
      const long long rec0 = (static_cast<long long>(g) * p.max_seg + (h - chunk_begin(p, g) / p.n_chunks)) * kWarps;
      for (int w = 0; w < kWarps; ++w) {
        const float ls = part_lse[rec0 + w];
        const float wt = (ls == -INFINITY) ? 0.f : expf(ls - M);
        L += wt;
        acc = fmaf(wt, part_o[(rec0 + w) * D + c], acc);
      }
    }
  }
  const float out = (L > 0.f) ? acc / L : 0.f;
  if constexpr (OF32) {
    static_cast<float*>(o)[static_cast<size_t>(h) * D + c] = out;
  }
  if (c == 0 && lse != nullptr) lse[h] = (L > 0.f) ? M + logf(L) : -INFINITY;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(128)
    fa_decode_combine16(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                        uint16_t* __restrict__ o, float* __restrict__ lse, const DecodeParams p) {
  // Same merge as fa_decode_combine, output rounded to the input's 16-bit type.
  const int h = blockIdx.x;
  const int c = threadIdx.x;
  const long long x0 = static_cast<long long>(h) * p.n_chunks;
  const long long x1 = x0 + p.n_chunks - 1;
  auto cta_of = [&](long long x) {
    long long g = x * p.grid / p.total;
    while (g + 1 < p.grid && chunk_begin(p, static_cast<int>(g + 1)) <= x) ++g;
    while (g > 0 && chunk_begin(p, static_cast<int>(g)) > x) --g;
    return static_cast<int>(g);
  };
  const int lo = cta_of(x0), hi = cta_of(x1);
  float M = -INFINITY;
  for (int g = lo; g <= hi; ++g) {
    const long long rec0 = (static_cast<long long>(g) * p.max_seg + (h - chunk_begin(p, g) / p.n_chunks)) * kWarps;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, part_lse[rec0 + w]);
  }
  float L = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int g = lo; g <= hi; ++g) {
      const long long rec0 = (static_cast<long long>(g) * p.max_seg + (h - chunk_begin(p, g) / p.n_chunks)) * kWarps;
      for (int w = 0; w < kWarps; ++w) {
        const float ls = part_lse[rec0 + w];
        const float wt = (ls == -INFINITY) ? 0.f : expf(ls - M);
        L += wt;
        acc = fmaf(wt, part_o[(rec0 + w) * D + c], acc);
      }
    }
  }
  const float out = (L > 0.f) ? acc / L : 0.f;
  if constexpr (BF16) {
    o[static_cast<size_t>(h) * D + c] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
  } else {
    o[static_cast<size_t>(h) * D + c] = __half_as_ushort(__float2half_rn(out));
  }
  if (c == 0 && lse != nullptr) lse[h] = (L > 0.f) ? M + logf(L) : -INFINITY;
}

template <int D, bool BF16>
cudaError_t launch_t(const void* q, const void* k, const void* v, void* o, float* lse,
                     const DecodeParams& p, bool o_f32, float* part_o, float* part_lse,
                     int* status, cudaStream_t stream, const PagedKV* paged) {
  auto kern = paged ? fa_decode_split_sm100<D, BF16, true> : fa_decode_split_sm100<D, BF16, false>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), DecodeCfg<D>::kBytes, 0);
  if (e != cudaSuccess) return e;
  const PagedKV pk = paged ? *paged : PagedKV{nullptr, nullptr, 1, 0, 0, 0};
  kern<<<p.grid, kThreads, DecodeCfg<D>::kBytes, stream>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
      static_cast<const uint16_t*>(v), part_o, part_lse, p, pk, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (o_f32)
    fa_decode_combine<D, true><<<p.BH, D, 0, stream>>>(part_o, part_lse, o, lse, p);
  else
    fa_decode_combine16<D, BF16><<<p.BH, D, 0, stream>>>(part_o, part_lse,
                                                          static_cast<uint16_t*>(o), lse, p);
  return cudaGetLastError();
}

// Diagnostic: one thread waits on an mbarrier that nothing ever arrives on.  The
// bounded wait gives up after kWaitLimitNs, records kStatusTimeoutDecode in the status
// word and the kernel returns -- the same path a real stall would take.
__global__ void fa_wait_timeout_selftest(int* __restrict__ status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, status, &abort_flag, kStatusTimeoutDecode);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int* status, cudaStream_t stream) {
  fa_wait_timeout_selftest<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

size_t decode_smem_bytes(int d) {
  return d == 128 ? DecodeCfg<128>::kBytes : DecodeCfg<64>::kBytes;
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                          const DecodeParams& p, int d, bool bf16, bool o_f32, float* part_o,
                          float* part_lse, int* status, cudaStream_t stream,
                          const PagedKV* paged) {
  if (d == 128 && bf16) return launch_t<128, true>(q, k, v, o, lse, p, o_f32, part_o, part_lse, status, stream, paged);
  if (d == 128 && !bf16) return launch_t<128, false>(q, k, v, o, lse, p, o_f32, part_o, part_lse, status, stream, paged);
  if (d == 64 && bf16) return launch_t<64, true>(q, k, v, o, lse, p, o_f32, part_o, part_lse, status, stream, paged);
  if (d == 64 && !bf16) return launch_t<64, false>(q, k, v, o, lse, p, o_f32, part_o, part_lse, status, stream, paged);
  return cudaErrorInvalidValue;
}

}  // namespace fa

// fa_quant.cu -- E4M3 quantisation of queries and keys with one scale per 128-row tile.
//
// The FP8 path of "FlashAttention 1-2-3" (myaihardware), section "FlashAttention-3: FP8,
// Async Warp Overlap, and Hopper-Specific Optimizations", feeds the tensor cores FP8
// queries and keys quantised on the fly.  Here a tile of 128 consecutive rows of one head
// (the prefill kernel's Q or K tile, d = 128) shares one scale: scale = max|x| / 448 over
// the tile (1 for an all-zero tile), code = E4M3(x / scale), rounded to nearest even and
// saturated at +-448.  A scale per tile rather than per tensor needs no pass over the
// whole tensor before the first code is written, and it keeps small-magnitude tiles
// accurate.  The prefill kernel multiplies each score tile by its Q tile's and K tile's
// scales.  Memory bound: 2 bytes read and 1 written per element.
//
// The code of x is the E4M3 rounding of the correctly rounded fp32 quotient x / scale.  A
// full IEEE division per element made this kernel instruction-bound, so a tile whose scale
// lies in [2^-100, inf) takes the quotient from the tile's correctly rounded reciprocal
// r = 1 / scale and one correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990):
// q0 = x * r, e = x - q0 * scale (exact with an FMA), q = q0 + e * r.  For every 16-bit amax
// (bf16 and fp16) and every |x| <= amax of the same type, the E4M3 code of that q equals the
// code of x / scale: checked exhaustively on the host (about 1.0e9 pairs).  The floats
// themselves differ only where x / scale is below fp32's normal range, where both codes are
// 0.  Tiles with a smaller or non-finite scale divide element by element.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fa_device.cuh"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kTileRows = 128;
constexpr int kD = 128;
// One tile is 128 rows x 256 bytes = 2048 16-byte chunks: 8 per thread, chunk i of thread t
// at index t + 256 i (consecutive threads read consecutive 16 bytes).
constexpr int kChunksPerThread = kTileRows * kD * 2 / 16 / kQuantThreads;

// Two fp32 values to a packed E4M3 pair (round to nearest even, saturating to +-448),
// `lo` in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// x / scale rounded to fp32 as the E4M3 conversion needs it: by the reciprocal and one
// correction step (RECIP, scale in [2^-100, inf)), else by an IEEE division.
template <bool RECIP>
__device__ __forceinline__ float quotient(float x, float scale, float r) {
  if (!RECIP) return x / scale;
  const float q0 = x * r;
  return fmaf(fmaf(-q0, scale, x), r, q0);
}

// Codes of this thread's chunks of one tile (chunk i at index threadIdx.x + 256 i).
template <bool BF16, bool RECIP>
__device__ __forceinline__ void store_codes(const uint4 (&raw)[kChunksPerThread],
                                            uint2* __restrict__ codes, int rows, float scale) {
  const float r = 1.0f / scale;
#pragma unroll
  for (int i = 0; i < kChunksPerThread; ++i) {
    const int c = threadIdx.x + kQuantThreads * i;
    if (c / (kD / 8) < rows) {
      const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
      uint16_t q[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a, b;
        unpack2<BF16>(w[e], a, b);
        q[e] = e4m3x2(quotient<RECIP>(a, scale, r), quotient<RECIP>(b, scale, r));
      }
      codes[c] = make_uint2(q[0] | (static_cast<uint32_t>(q[1]) << 16),
                            q[2] | (static_cast<uint32_t>(q[3]) << 16));
    }
  }
}

// One tensor to quantise: [BH, N, 128] 16-bit values in, codes and one scale per tile out.
struct QuantJob {
  const uint4* x;
  uint2* codes;
  float* scales;
  int N, n_tiles;
  long long blocks;  // BH * n_tiles: one CTA per tile
};

// Blocks [0, a.blocks) quantise tensor a, the rest tensor b (b.blocks = 0: none), so that
// Q and K of one call take a single launch.
template <bool BF16>
__global__ void __launch_bounds__(kQuantThreads)
    fa_quantize_e4m3_tiles(const QuantJob a, const QuantJob b) {
  __shared__ float warp_max[kQuantThreads / 32];
  const bool second = blockIdx.x >= a.blocks;
  const long long blk = second ? blockIdx.x - a.blocks : blockIdx.x;
  const uint4* __restrict__ x = second ? b.x : a.x;
  uint2* __restrict__ codes = second ? b.codes : a.codes;
  float* __restrict__ scales = second ? b.scales : a.scales;
  const int N = second ? b.N : a.N;
  const int n_tiles = second ? b.n_tiles : a.n_tiles;
  const long long bh = blk / n_tiles;
  const int tile = static_cast<int>(blk - bh * n_tiles);
  const int rows = min(kTileRows, N - tile * kTileRows);
  const size_t base = (static_cast<size_t>(bh) * N + static_cast<size_t>(tile) * kTileRows) * (kD / 8);
  uint4 raw[kChunksPerThread];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kChunksPerThread; ++i) {
    const int c = threadIdx.x + kQuantThreads * i;
    if (c / (kD / 8) < rows) {
      raw[i] = x[base + c];
      const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a, b;
        unpack2<BF16>(w[e], a, b);
        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);
  const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
  if (threadIdx.x == 0) scales[blk] = scale;
  if (scale >= 0x1p-100f && scale < INFINITY)
    store_codes<BF16, true>(raw, codes + base, rows, scale);
  else
    store_codes<BF16, false>(raw, codes + base, rows, scale);
}

QuantJob make_job(const void* x, long long BH, int N, void* codes, float* scales) {
  QuantJob j;
  j.x = static_cast<const uint4*>(x);
  j.codes = static_cast<uint2*>(codes);
  j.scales = scales;
  j.N = N;
  j.n_tiles = (N + kTileRows - 1) / kTileRows;
  j.blocks = BH * j.n_tiles;
  return j;
}

cudaError_t launch_jobs(const QuantJob& a, const QuantJob& b, bool bf16, cudaStream_t stream) {
  const long long blocks = a.blocks + b.blocks;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (bf16)
    fa_quantize_e4m3_tiles<true><<<static_cast<int>(blocks), kQuantThreads, 0, stream>>>(a, b);
  else
    fa_quantize_e4m3_tiles<false><<<static_cast<int>(blocks), kQuantThreads, 0, stream>>>(a, b);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* x, bool bf16, long long BH, int N, void* codes,
                                 float* scales, cudaStream_t stream) {
  QuantJob none = make_job(x, 0, N, codes, scales);
  return launch_jobs(make_job(x, BH, N, codes, scales), none, bf16, stream);
}

cudaError_t launch_quantize_e4m3_qk(const void* q, int Nq, void* q8, float* qs, const void* k,
                                    int Nkv, void* k8, float* ks, bool bf16, long long BH,
                                    cudaStream_t stream) {
  return launch_jobs(make_job(q, BH, Nq, q8, qs), make_job(k, BH, Nkv, k8, ks), bf16, stream);
}

}  // namespace fa

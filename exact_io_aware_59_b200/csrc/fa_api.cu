// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, per-device state,
// TMA descriptors and kernel launches.  Host code only.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

constexpr int kMaxDevices = 64;

// The device status word the kernels OR their wait-timeout and bad-input bits into: one
// word per device (each device's copy of this array), zero when the module loads, so no
// allocation is needed for it.
__device__ __align__(256) int g_status_word[64];

struct KernelConfig {
  const void* fn;
  cudaError_t err;
};

struct DeviceState {
  bool probed = false;
  bool arch_ok = false;
  int sm_count = 0;
  int* status = nullptr;               // device address of this device's g_status_word
  cudaMemPool_t pool = nullptr;        // workspace pool (decode partials, varlen unit list)
  KernelConfig kernels[64] = {};       // kernels already configured on this device
  int n_kernels = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
thread_local int g_last_cuda_error = 0;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

// Looks up (and on first use initialises) the current device's state: architecture, SM
// count and the status word's address.  Nothing here allocates device memory or
// synchronises.
int device_state_core(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.probed) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e);
    s.arch_ok = (major == 10 && minor == 0);  // the sm_100a code runs on CC 10.0 only
    s.sm_count = sms;
    s.probed = true;
  }
  if (!s.arch_ok) return FA_ERR_ARCH;
  if (!s.status) {
    // In host code g_status_word names a host-side stand-in: kernels get the address of
    // this device's copy.
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_status_word)) != cudaSuccess)
      return e == cudaErrorMemoryAllocation ? FA_ERR_NOMEM : cuda_fail(e);
    s.status = static_cast<int*>(p);
  }
  *out = &s;
  return FA_OK;
}

// device_state_core, plus the device's workspace pool (created on the first call of any
// entry point that may need workspace; creating a pool reserves no memory).  The pool
// keeps freed memory mapped (release threshold: all of it), so after the first calls an
// allocation from it is a bookkeeping step in stream order.
int device_state(DeviceState** out) {
  DeviceState* s = nullptr;
  int rc = device_state_core(&s);
  if (rc != FA_OK) return rc;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!s->pool) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return cuda_fail(e);
    uint64_t keep = ~0ull;
    if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return cuda_fail(e);
    }
    s->pool = pool;
  }
  *out = s;
  return FA_OK;
}

// Stream-ordered workspace from the device's pool.  Under stream capture the allocation
// and the matching cudaFreeAsync become graph memory nodes.
int workspace_alloc(DeviceState* ds, size_t bytes, cudaStream_t stream, void** ptr) {
  const cudaError_t e = cudaMallocFromPoolAsync(ptr, bytes, ds->pool, stream);
  if (e == cudaErrorMemoryAllocation) return FA_ERR_NOMEM;
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int get_encoder() {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode) return FA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess) return cuda_fail(e);
  if (q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(cudaErrorNotSupported);
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return FA_OK;
}

// 3-D view (d, N, B*H) of a [B,H,N,d] tensor; box (64, box_rows, 1) with 128-byte swizzle.
int make_map(CUtensorMap* map, const void* ptr, int N, long long BH, int d, bool bf16,
             unsigned box_rows = 128) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FA_OK;
}

// 3-D view (d, N, B*H) of a [B,H,N,d] tensor of one-byte codes (d = 128); box
// (128, 128, 1): one 128-byte row per query or key, 128-byte swizzle.
int make_map_u8(CUtensorMap* map, const void* ptr, int N, long long BH, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N) * d};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FA_OK;
}

// 3-D view (d, H, tokens) of a packed [tokens, H, d] tensor; box (64, 1, 128): the same
// 128 rows x 128 B shared-memory tile as above, rows being tokens of one head.
int make_map_packed(CUtensorMap* map, const void* ptr, long long tokens, int H, int d, bool bf16) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Checks shared by every entry point.  Nothing here touches the device.
int check_args(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int Nq, int Nkv, int d, float scale, int causal, int in_dtype, int o_dtype) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 1 || Nkv < 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_F16 && in_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F16 && o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F32 && o_dtype != in_dtype) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return FA_ERR_INVALID_ARG;
  if (lse && !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t qb = BH * Nq * d * 2, kvb = BH * Nkv * d * 2;
  const size_t ob = BH * Nq * d * (o_dtype == FA_F32 ? 4 : 2), lb = BH * Nq * 4;
  if (overlaps(o, ob, q, qb) || overlaps(o, ob, k, kvb) || overlaps(o, ob, v, kvb)) return FA_ERR_INVALID_ARG;
  if (lse && (overlaps(lse, lb, o, ob) || overlaps(lse, lb, q, qb) || overlaps(lse, lb, k, kvb) ||
              overlaps(lse, lb, v, kvb)))
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

float scale_log2(float scale) { return static_cast<float>(static_cast<double>(scale) * 1.4426950408889634); }

fa::DecodeParams decode_params(int B, int H, int Nkv, float scale, int num_splits, int sm_count) {
  fa::DecodeParams p{};
  p.BH = B * H;
  p.Nkv = Nkv;
  p.n_chunks = (Nkv + fa::kDecodeChunk - 1) / fa::kDecodeChunk;
  p.total = static_cast<long long>(p.BH) * p.n_chunks;
  long long g = num_splits > 0 ? num_splits : sm_count;
  if (g > p.total) g = p.total;
  if (g < 1) g = 1;
  p.grid = static_cast<int>(g);
  const long long per_cta = (p.total + p.grid - 1) / p.grid;
  p.max_seg = static_cast<int>((per_cta + p.n_chunks - 1) / p.n_chunks + 1);
  p.scale_log2 = scale_log2(scale);
  return p;
}

size_t decode_ws_bytes(const fa::DecodeParams& p, int d) {
  const size_t recs = static_cast<size_t>(p.grid) * p.max_seg * fa::kDecodeRecords;
  return recs * (d + 1) * sizeof(float);
}

// K/V parts per (head, Q-tile pair) for a prefill with fewer work units than SMs, chosen
// with a run-time model fitted to B200 timings of 14 shapes (d 64 and 128, causal and not,
// 1 to 32 heads, 2k to 16k tokens; predicted within about 5%):
//   time(S) = steps of the busiest CTA, each unit adding kUnitSteps (its Q load and its
//             pipeline's fill and drain), units dealt heaviest first in the snake order
//             the kernel uses, times the step time (K/V tile of 128 keys for both Q tiles:
//             about 1.8 us at d = 128, 1.62 us at d = 64)
//           + for S > 1, the partial records and the combine launch: 8 us + 0.4 ns per
//             partial element (S * B*H*Nq * d).
// A split is taken only when the model predicts at least 10% less time than no split.
constexpr int kMaxSplits = 8;
constexpr double kUnitSteps = 3.75;

// Host copy of the kernel's K/V tile count for Q tile `qtile` ([B,H,N,d] layout).
int host_kv_tiles(const fa::PrefillParams& p, int qtile) {
  if (qtile * 128 >= p.Nq) return 0;
  const int ntk = p.n_kvtiles;
  if (!p.causal) return ntk;
  const int last_key = std::min(qtile * 128 + 127, p.Nq - 1) + p.Nkv - p.Nq;
  return last_key < 0 ? 0 : std::min(ntk, last_key / 128 + 1);
}

// nmax[pair]: the K/V tiles of each Q-tile pair (its heavier tile's).
double predicted_us(const fa::PrefillParams& p, const int* nmax, int S, int sm_count, int d) {
  const long long units = static_cast<long long>(p.BH) * p.n_pairs * S;
  const int G = static_cast<int>(std::min<long long>(sm_count, units));
  double load[1024] = {0.0};
  long long u = 0;
  for (int pair = p.n_pairs - 1; pair >= 0; --pair) {
    for (int split = 0; split < S; ++split) {
      const int steps = (split + 1) * nmax[pair] / S - split * nmax[pair] / S;
      const double cost = steps > 0 ? steps + kUnitSteps : 0.3;
      for (int bh = 0; bh < p.BH; ++bh, ++u) {
        const long long r = u / G, c = u - r * G;
        load[(r & 1) ? G - 1 - c : c] += cost;
      }
    }
  }
  double worst = 0.0;
  for (int c = 0; c < G; ++c) worst = std::max(worst, load[c]);
  double t = worst * (d == 128 ? 1.8 : 1.62);
  if (S > 1) t += 8.0 + 4e-7 * S * static_cast<double>(p.BH) * p.Nq * d;
  return t;
}

// Whether an unsplit launch of `pairs` Q-tile pairs on `grid` CTAs runs interleaved-K/V
// units: a causal one whenever every pair would get its own CTA; a non-causal one (whose
// pairs all take the same number of steps) only when every Q tile would, since with two
// units on some CTAs it would gain nothing and pay a merge per unit.
bool kvi_fits(int causal, int S, long long grid, long long pairs) {
  return S == 1 && (causal ? grid >= pairs : grid >= 2 * pairs);
}

// Small launches left unsplit run interleaved-K/V units (run_prefill): one Q tile
// per unit, its K/V tiles shared by two warpgroups, so a unit takes ceil(n / 2) steps of
// two tiles, with no combine launch.  Fitted to B200 timings of 10 shapes (within 11%):
// 3 steps of fill, drain and merge per unit, 1.34 times the paired kernel's step time.
double predicted_kvi_us(const fa::PrefillParams& p, int sm_count, int d) {
  const long long units = static_cast<long long>(p.BH) * p.n_qtiles;
  const int G = static_cast<int>(std::min<long long>(sm_count, units));
  double load[1024] = {0.0};
  long long u = 0;
  for (int qt = p.n_qtiles - 1; qt >= 0; --qt) {
    const int steps = (host_kv_tiles(p, qt) + 1) / 2;
    const double cost = steps > 0 ? steps + 3.0 : 0.3;
    for (int bh = 0; bh < p.BH; ++bh, ++u) {
      const long long r = u / G, c = u - r * G;
      load[(r & 1) ? G - 1 - c : c] += cost;
    }
  }
  double worst = 0.0;
  for (int c = 0; c < G; ++c) worst = std::max(worst, load[c]);
  return worst * (d == 128 ? 1.8 : 1.62) * 1.34;
}

int auto_splits_uncached(const fa::PrefillParams& p, int sm_count, int d) {
  int nmax[1024];
  for (int pair = 0; pair < p.n_pairs; ++pair)
    nmax[pair] = std::max(host_kv_tiles(p, 2 * pair), host_kv_tiles(p, 2 * pair + 1));
  const double t1 = predicted_us(p, nmax, 1, sm_count, d);
  int best = 1;
  double t_best = t1;
  for (int S = 2; S <= std::min(kMaxSplits, p.n_kvtiles); ++S) {
    const double t = predicted_us(p, nmax, S, sm_count, d);
    if (t < t_best) {
      t_best = t;
      best = S;
    }
  }
  const int split = t_best < 0.9 * t1 ? best : 1;
  // The launch may do better unsplit, as interleaved-K/V units (measured on causal
  // launches: when the model picks two parts, the units win by 14-21%; from three parts on,
  // the split wins).  The split's predictions run about 8% under its measured times.
  const long long pairs = static_cast<long long>(p.BH) * p.n_pairs;
  if (split > 1 && kvi_fits(p.causal, 1, sm_count, pairs) &&
      predicted_kvi_us(p, sm_count, d) <= 1.08 * t_best)
    return 1;
  return split;
}

// The choice for the last few shapes this thread asked about (the model's loop costs a few
// microseconds; a program repeats its shapes).
int auto_splits(const fa::PrefillParams& p, int sm_count, int d) {
  const long long units = static_cast<long long>(p.BH) * p.n_pairs;
  if (units >= sm_count || sm_count > 1024) return 1;  // then also n_pairs < 1024
  struct Entry {
    int BH, Nq, Nkv, causal, d, sm_count, S;
  };
  thread_local Entry cache[8] = {};
  thread_local int next = 0;
  for (const Entry& e : cache)
    if (e.S > 0 && e.BH == p.BH && e.Nq == p.Nq && e.Nkv == p.Nkv && e.causal == p.causal &&
        e.d == d && e.sm_count == sm_count)
      return e.S;
  const int S = auto_splits_uncached(p, sm_count, d);
  cache[next] = Entry{p.BH, p.Nq, p.Nkv, p.causal, d, sm_count, S};
  next = (next + 1) % 8;
  return S;
}

int run_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int Nq, int Nkv, int d, float scale, int causal, void* stream, int in_dtype,
                int o_dtype, int num_ctas, int num_splits) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if ((rc = get_encoder()) != FA_OK) return rc;
  const bool bf16 = in_dtype == FA_BF16;
  const long long BH = static_cast<long long>(B) * H;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, Nq, BH, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map(&tk, k, Nkv, BH, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, Nkv, BH, d, bf16)) != FA_OK) return rc;
  fa::PrefillParams p{};
  p.BH = static_cast<int>(BH);
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.off = Nkv - Nq;
  p.causal = causal;
  p.n_qtiles = (Nq + 127) / 128;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.n_kvtiles = (Nkv + 127) / 128;
  const long long units = BH * p.n_pairs;
  if (units > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  p.n_units = static_cast<int>(units);
  p.cu_q = p.cu_k = nullptr;
  p.H = H;
  p.scale_log2 = scale_log2(scale);
  const int S = num_splits > 0 ? std::min(num_splits, p.n_kvtiles) : auto_splits(p, ds->sm_count, d);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  float *part_o = nullptr, *part_lse = nullptr;
  if (S > 1) {
    // Split partials: fp32 O / l [S, BH*Nq, d] then the natural LSE [S, BH*Nq].
    const long long split_units = units * S;
    if (split_units > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
    const size_t rows = static_cast<size_t>(BH) * Nq;
    const size_t ob = static_cast<size_t>(S) * rows * d * sizeof(float);
    if ((rc = workspace_alloc(ds, ob + static_cast<size_t>(S) * rows * sizeof(float), st, &ws)) != FA_OK)
      return rc;
    p.n_splits = S;
    part_o = static_cast<float*>(ws);
    part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + ob);
    p.n_units = static_cast<int>(split_units);
  } else {
    p.n_splits = 1;
  }
  long long grid = num_ctas > 0 ? num_ctas : ds->sm_count;
  if (kvi_fits(causal, S, grid, p.n_units) && BH * p.n_qtiles <= 0x7fffffffLL) {
    // Every Q-tile pair would get its own CTA, so a unit's serial chain of K/V steps sets
    // the launch's time.  Make each Q tile a unit instead, its even K/V tiles on one
    // softmax warpgroup and its odd ones on the other (merged at the end): the chain halves
    // and both warpgroups stay busy; the CTAs take the units heaviest first.
    p.n_splits = 0;  // the launch's interleaved-K/V flag
    p.n_pairs = p.n_qtiles;
    p.n_units = static_cast<int>(BH * p.n_qtiles);
  }
  if (grid > p.n_units) grid = p.n_units;
  if (grid < 1) grid = 1;
  cudaError_t e = fa::launch_prefill(tq, tk, tv, o, lse, p, d, bf16, o_dtype == FA_F32,
                                     static_cast<int>(grid), ds->status, st, false, part_o,
                                     part_lse);
  if (ws != nullptr) {
    const cudaError_t ef = cudaFreeAsync(ws, st);
    if (e == cudaSuccess) e = ef;
  }
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int run_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_q,
               const int* cu_k, int B, int H, int total_q, int total_k, int max_q, int max_k,
               int d, float scale, int causal, void* stream, int in_dtype, int o_dtype) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if ((rc = get_encoder()) != FA_OK) return rc;
  const bool bf16 = in_dtype == FA_BF16;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map_packed(&tq, q, total_q, H, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map_packed(&tk, k, total_k, H, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map_packed(&tv, v, total_k, H, d, bf16)) != FA_OK) return rc;
  fa::PrefillParams p{};
  p.BH = B * H;
  p.Nq = max_q;
  p.Nkv = max_k;
  p.off = 0;  // per sequence in the kernel
  p.causal = causal;
  p.n_qtiles = (max_q + 127) / 128;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.n_kvtiles = (max_k + 127) / 128;
  // At most one item per (sequence, Q-tile pair) and H units per item.
  const long long items = static_cast<long long>(B) * p.n_pairs;
  const long long units = items * H;
  if (units > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  p.n_units = static_cast<int>(units);  // an upper bound: the plan kernel counts the real ones
  p.scale_log2 = scale_log2(scale);
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.H = H;
  p.total_q = total_q;
  p.total_k = total_k;
  // Call-local workspace for the plan: item count and work counter (16 bytes), B sequence
  // records, B first positions, items.
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  const size_t seq_b = static_cast<size_t>(B) * sizeof(int4), first_b = static_cast<size_t>(B) * 4;
  const size_t ws_bytes = 16 + seq_b + first_b + static_cast<size_t>(items) * 4;
  if ((rc = workspace_alloc(ds, ws_bytes, st, &ws)) != FA_OK) return rc;
  char* w = static_cast<char*>(ws);
  p.vl_count = reinterpret_cast<int*>(w);
  p.vl_next = reinterpret_cast<int*>(w) + 1;
  p.vl_seqs = reinterpret_cast<int4*>(w + 16);
  p.vl_first = reinterpret_cast<int*>(w + 16 + seq_b);
  p.vl_items = reinterpret_cast<int*>(w + 16 + seq_b + first_b);
  long long grid = ds->sm_count;
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  cudaError_t e = fa::launch_prefill(tq, tk, tv, o, lse, p, d, bf16, o_dtype == FA_F32,
                                     static_cast<int>(grid), ds->status, st);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e == cudaSuccess) e = ef;
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int check_varlen_args(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int* cu_q, const int* cu_k, int B, int H, int total_q, int total_k,
                      int max_q, int max_k, int d, float scale, int causal, int in_dtype,
                      int o_dtype) {
  if (!q || !k || !v || !o || !cu_q || !cu_k) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || total_q < 1 || total_k < 1 || max_q < 1 || max_k < 1) return FA_ERR_INVALID_ARG;
  if (max_q > total_q || max_k > total_k) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_F16 && in_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F16 && o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F32 && o_dtype != in_dtype) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(cu_q, 4) || !aligned(cu_k, 4) || (lse && !aligned(lse, 4))) return FA_ERR_INVALID_ARG;
  const size_t qb = static_cast<size_t>(total_q) * H * d * 2;
  const size_t kb = static_cast<size_t>(total_k) * H * d * 2;
  const size_t ob = static_cast<size_t>(total_q) * H * d * (o_dtype == FA_F32 ? 4 : 2);
  const size_t lb = static_cast<size_t>(total_q) * H * 4, cb = static_cast<size_t>(B + 1) * 4;
  const void* ins[5] = {q, k, v, cu_q, cu_k};
  const size_t in_bytes[5] = {qb, kb, kb, cb, cb};
  for (int i = 0; i < 5; ++i) {
    if (overlaps(o, ob, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
    if (lse && overlaps(lse, lb, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
  }
  if (lse && overlaps(lse, lb, o, ob)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

int run_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int Nkv, int d, float scale, void* stream, int in_dtype, int o_dtype,
               int num_splits, const fa::PagedKV* paged = nullptr) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  const fa::DecodeParams p = decode_params(B, H, Nkv, scale, num_splits, ds->sm_count);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The split partials live for this call only: allocated and freed in stream order, so
  // calls on different streams never share them and no call waits for the device.
  void* ws = nullptr;
  if ((rc = workspace_alloc(ds, decode_ws_bytes(p, d), st, &ws)) != FA_OK) return rc;
  float* part_o = static_cast<float*>(ws);
  float* part_lse = part_o + static_cast<size_t>(p.grid) * p.max_seg * fa::kDecodeRecords * d;
  cudaError_t e = fa::launch_decode(q, k, v, o, lse, p, d, in_dtype == FA_BF16, o_dtype == FA_F32,
                                    part_o, part_lse, ds->status, st, paged);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e == cudaSuccess) e = ef;
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

// Host checks of fa_fwd_decode_paged (everything but the device-resident table and lengths).
int check_paged_args(const void* q, const void* kc, const void* vc, const int* table,
                     const int* lens, void* o, float* lse, int B, int H, int d, int page_size,
                     int max_pages, int num_pages, float scale, int in_dtype, int o_dtype,
                     int num_splits) {
  if (!q || !kc || !vc || !table || !lens || !o) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || max_pages < 1 || num_pages < 1 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (page_size < 16 || page_size > 1024 || (page_size & (page_size - 1)) != 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_pages) * page_size > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_F16 && in_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F16 && o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F32 && o_dtype != in_dtype) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(o, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(table, 4) || !aligned(lens, 4) || (lse && !aligned(lse, 4))) return FA_ERR_INVALID_ARG;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t qb = BH * d * 2, ob = BH * d * (o_dtype == FA_F32 ? 4 : 2), lb = BH * 4;
  const size_t cb = static_cast<size_t>(num_pages) * H * page_size * d * 2;
  const size_t tb = static_cast<size_t>(B) * max_pages * 4, sb = static_cast<size_t>(B) * 4;
  const void* ins[5] = {q, kc, vc, table, lens};
  const size_t in_bytes[5] = {qb, cb, cb, tb, sb};
  for (int i = 0; i < 5; ++i) {
    if (overlaps(o, ob, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
    if (lse && overlaps(lse, lb, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
  }
  if (lse && overlaps(lse, lb, o, ob)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // namespace

namespace fa {
int check_decode_call(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int Nkv, int d, float scale, int in_dtype, int o_dtype) {
  return check_args(q, k, v, o, lse, B, H, 1, Nkv, d, scale, 0, in_dtype, o_dtype);
}
DecodeParams plan_decode(int B, int H, int Nkv, float scale, int num_splits, int sm_count) {
  return decode_params(B, H, Nkv, scale, num_splits, sm_count);
}
size_t decode_workspace_bytes(const DecodeParams& p, int d) { return decode_ws_bytes(p, d); }

int cuda_failure(cudaError_t e) { return cuda_fail(e); }

int current_device(int* sm_count, int** status) {
  DeviceState* ds = nullptr;
  const int rc = device_state_core(&ds);
  if (rc != FA_OK) return rc;
  *sm_count = ds->sm_count;
  *status = ds->status;
  return FA_OK;
}

cudaError_t configure_kernel(const void* kernel, int smem_bytes, int min_regs) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  for (int i = 0; i < s.n_kernels; ++i)
    if (s.kernels[i].fn == kernel) return s.kernels[i].err;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess && min_regs > 0) {
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, kernel);
    // setmaxnreg redistributes the registers the block was launched with; a launch with
    // fewer would make the increase wait forever.
    if (e == cudaSuccess && attr.numRegs < min_regs) e = cudaErrorInvalidConfiguration;
  }
  if (s.n_kernels < static_cast<int>(sizeof(s.kernels) / sizeof(s.kernels[0])))
    s.kernels[s.n_kernels++] = KernelConfig{kernel, e};
  return e;
}
}  // namespace fa

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
           int Nq, int Nkv, int d, float scale, int causal, void* stream, int in_dtype,
           int o_dtype) {
  int rc = check_args(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (Nq == 1) return run_decode(q, k, v, o, lse, B, H, Nkv, d, scale, stream, in_dtype, o_dtype, 0);
  return run_prefill(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype, o_dtype, 0,
                     0);
}

int fa_fwd_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
                   int in_dtype, int o_dtype, int num_ctas) {
  int rc = check_args(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (num_ctas < 0) return FA_ERR_INVALID_ARG;
  // An explicit grid runs the unsplit units; the automatic one may split them.
  return run_prefill(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype, o_dtype,
                     num_ctas, num_ctas > 0 ? 1 : 0);
}

int fa_prefill_num_splits(int B, int H, int Nq, int Nkv, int d, int causal, int sm_count,
                          int* num_splits) {
  if (!num_splits || B < 1 || H < 1 || Nq < 1 || Nkv < 1 || (d != 64 && d != 128) ||
      (causal != 0 && causal != 1) || sm_count < 0)
    return FA_ERR_INVALID_ARG;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (sm_count == 0) {
    DeviceState* ds = nullptr;
    const int rc = device_state(&ds);
    if (rc != FA_OK) return rc;
    sm_count = ds->sm_count;
  }
  fa::PrefillParams p{};
  p.BH = static_cast<int>(BH);
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.causal = causal;
  p.n_qtiles = (Nq + 127) / 128;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.n_kvtiles = (Nkv + 127) / 128;
  *num_splits = auto_splits(p, sm_count, d);
  return FA_OK;
}

int fa_fwd_prefill_split(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
                         int in_dtype, int o_dtype, int num_ctas, int num_splits) {
  int rc = check_args(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (num_ctas < 0 || num_splits < 0 || num_splits > 64) return FA_ERR_INVALID_ARG;
  return run_prefill(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype, o_dtype,
                     num_ctas, num_splits);
}

int fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int H, int Nkv, int d, float scale, void* stream, int in_dtype, int o_dtype,
                  int num_splits) {
  int rc = check_args(q, k, v, o, lse, B, H, 1, Nkv, d, scale, 0, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (num_splits < 0) return FA_ERR_INVALID_ARG;
  return run_decode(q, k, v, o, lse, B, H, Nkv, d, scale, stream, in_dtype, o_dtype, num_splits);
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* v, void* o, float* lse, int B,
               int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
               float q_scale, float k_scale, int v_dtype, int o_dtype) {
  if (!q8 || !k8 || !v || !o) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 1 || Nkv < 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !std::isfinite(q_scale) || !std::isfinite(k_scale)) return FA_ERR_INVALID_ARG;
  const float s_all = scale * q_scale * k_scale;
  if (!std::isfinite(s_all)) return FA_ERR_INVALID_ARG;
  if (v_dtype != FA_F16 && v_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F16 && o_dtype != FA_BF16 && o_dtype != FA_F32) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_F32 && o_dtype != v_dtype) return FA_ERR_UNSUPPORTED;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v, 16) || !aligned(o, 16)) return FA_ERR_INVALID_ARG;
  if (lse && !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t qb = BH * Nq * d, kb = BH * Nkv * d, vb = BH * Nkv * d * 2;
  const size_t ob = BH * Nq * d * (o_dtype == FA_F32 ? 4 : 2), lb = BH * Nq * 4;
  const void* ins[3] = {q8, k8, v};
  const size_t in_bytes[3] = {qb, kb, vb};
  for (int i = 0; i < 3; ++i) {
    if (overlaps(o, ob, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
    if (lse && overlaps(lse, lb, ins[i], in_bytes[i])) return FA_ERR_INVALID_ARG;
  }
  if (lse && overlaps(lse, lb, o, ob)) return FA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if ((rc = get_encoder()) != FA_OK) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map_u8(&tq, q8, Nq, static_cast<long long>(BH), d)) != FA_OK) return rc;
  if ((rc = make_map_u8(&tk, k8, Nkv, static_cast<long long>(BH), d)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, Nkv, static_cast<long long>(BH), d, v_dtype == FA_BF16)) != FA_OK) return rc;
  fa::PrefillParams p{};
  p.BH = static_cast<int>(BH);
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.off = Nkv - Nq;
  p.causal = causal;
  p.n_qtiles = (Nq + 127) / 128;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.n_kvtiles = (Nkv + 127) / 128;
  const long long units = static_cast<long long>(BH) * p.n_pairs;
  if (units > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  p.n_units = static_cast<int>(units);
  p.scale_log2 = scale_log2(s_all);  // the per-tensor scales fold into the score scale
  p.cu_q = p.cu_k = nullptr;
  p.H = H;
  long long grid = ds->sm_count;
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  cudaError_t e = fa::launch_prefill(tq, tk, tv, o, lse, p, d, v_dtype == FA_BF16,
                                     o_dtype == FA_F32, static_cast<int>(grid), ds->status,
                                     static_cast<cudaStream_t>(stream), true);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

namespace {

// Workspace layout of fa_bwd: -LSE*log2(e) [BH, nq_pad], D [BH, nq_pad], then the fp32
// dQ accumulator [BH, nq_pad, d]; nq_pad = Nq rounded up to 128 (each part a multiple of
// 512 bytes).
size_t bwd_ws_bytes(size_t BH, int Nq, int d) {
  const size_t nq_pad = (static_cast<size_t>(Nq) + 127) / 128 * 128;
  return BH * nq_pad * (4 + 4 + static_cast<size_t>(d) * 4);
}

// Packed backward workspace: per head, rows_max rows (total_q + 128 * B rounded up to a
// multiple of 128: every sequence's query rows padded to whole 128-row tiles fit, and every
// head's rows, hence every tile's 512 bytes of -LSE*log2(e) and D that the main kernel
// bulk-copies, start on a 16-byte boundary) of -LSE*log2(e), D and the fp32 dQ accumulator;
// then the plan: item count (16 bytes), B sequence records, B + 1 padded row offsets
// (rounded up to 16 bytes), B * n_ktiles items.
struct VarlenBwdLayout {
  long long rows_max;
  size_t rows_bytes, plan_off, seqs_off, qpad_off, items_off, total;
};

VarlenBwdLayout varlen_bwd_layout(int B, int H, int total_q, int max_k, int d) {
  VarlenBwdLayout l;
  l.rows_max = (static_cast<long long>(total_q) + 128LL * B + 127) / 128 * 128;
  l.rows_bytes = static_cast<size_t>(H) * l.rows_max * (4 + 4 + static_cast<size_t>(d) * 4);
  const size_t n_ktiles = (static_cast<size_t>(max_k) + 127) / 128;
  l.plan_off = l.rows_bytes;
  l.seqs_off = l.plan_off + 16;
  l.qpad_off = l.seqs_off + static_cast<size_t>(B) * 16;
  l.items_off = l.qpad_off + (static_cast<size_t>(B + 1) * 4 + 15) / 16 * 16;
  l.total = l.items_off + static_cast<size_t>(B) * n_ktiles * 4;
  return l;
}

}  // namespace

int fa_bwd_workspace_bytes(int B, int H, int Nq, int d, size_t* bytes) {
  if (!bytes || B < 1 || H < 1 || Nq < 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  *bytes = bwd_ws_bytes(static_cast<size_t>(B) * H, Nq, d);
  return FA_OK;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, void* workspace,
           size_t workspace_bytes, int B, int H, int Nq, int Nkv, int d, float scale,
           int causal, void* stream, int in_dtype) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 1 || Nkv < 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_F16 && in_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const void* a16[9] = {q, k, v, o, dout, dq, dk, dv, workspace};
  for (const void* ptr : a16)
    if (!aligned(ptr, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t ws = bwd_ws_bytes(BH, Nq, d);
  if (workspace_bytes < ws) return FA_ERR_INVALID_ARG;
  const long long n_ktiles = (Nkv + 127) / 128, n_qtiles = (Nq + 127) / 128;
  if (static_cast<long long>(BH) * n_ktiles > 0x7fffffffLL ||
      static_cast<long long>(BH) * n_qtiles > 0x7fffffffLL)
    return FA_ERR_INVALID_ARG;
  const size_t qb = BH * Nq * d * 2, kb = BH * Nkv * d * 2, lb = BH * Nq * 4;
  const void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {qb, kb, kb, ws};
  const void* ins[6] = {q, k, v, o, dout, lse};
  const size_t in_bytes[6] = {qb, kb, kb, qb, qb, lb};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 6; ++j)
      if (overlaps(outs[i], out_bytes[i], ins[j], in_bytes[j])) return FA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], out_bytes[i], outs[j], out_bytes[j])) return FA_ERR_INVALID_ARG;
  }
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if ((rc = get_encoder()) != FA_OK) return rc;
  const bool bf16 = in_dtype == FA_BF16;
  CUtensorMap tq, tk, tv, tdo;
  if ((rc = make_map(&tq, q, Nq, static_cast<long long>(BH), d, bf16)) != FA_OK) return rc;
  if ((rc = make_map(&tdo, dout, Nq, static_cast<long long>(BH), d, bf16)) != FA_OK) return rc;
  if ((rc = make_map(&tk, k, Nkv, static_cast<long long>(BH), d, bf16)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, Nkv, static_cast<long long>(BH), d, bf16)) != FA_OK) return rc;
  fa::BwdParams p{};
  p.BH = static_cast<int>(BH);
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.off = Nkv - Nq;
  p.causal = causal;
  p.n_qtiles = static_cast<int>(n_qtiles);
  p.nq_pad = p.n_qtiles * 128;
  p.n_ktiles = static_cast<int>(n_ktiles);
  p.scale = scale;
  p.scale_log2 = scale_log2(scale);
  float* w = static_cast<float*>(workspace);
  p.nlse2 = w;
  p.delta = w + BH * p.nq_pad;
  p.dq_acc = w + 2 * BH * p.nq_pad;
  p.dk = dk;
  p.dv = dv;
  cudaError_t e = fa::launch_backward(tq, tk, tv, tdo, o, dout, lse, dq, p, d, bf16,
                                      ds->sm_count, ds->status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_bwd_varlen_workspace_bytes(int B, int H, int total_q, int max_seqlen_k, int d,
                                  size_t* bytes) {
  if (!bytes || B < 1 || H < 1 || total_q < 1 || max_seqlen_k < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  *bytes = varlen_bwd_layout(B, H, total_q, max_seqlen_k, d).total;
  return FA_OK;
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dout, void* dq, void* dk, void* dv, void* workspace,
                  size_t workspace_bytes, const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                  int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                  float scale, int causal, void* stream, int in_dtype) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace ||
      !cu_seqlens_q || !cu_seqlens_k)
    return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || total_q < 1 || total_k < 1 || max_seqlen_q < 1 || max_seqlen_k < 1)
    return FA_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q || max_seqlen_k > total_k) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_F16 && in_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const void* a16[9] = {q, k, v, o, dout, dq, dk, dv, workspace};
  for (const void* ptr : a16)
    if (!aligned(ptr, 16)) return FA_ERR_INVALID_ARG;
  if (!aligned(lse, 4) || !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return FA_ERR_INVALID_ARG;
  const VarlenBwdLayout lay = varlen_bwd_layout(B, H, total_q, max_seqlen_k, d);
  if (lay.rows_max > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < lay.total) return FA_ERR_INVALID_ARG;
  const long long n_ktiles = (max_seqlen_k + 127) / 128;
  if (static_cast<long long>(B) * n_ktiles * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  const size_t qb = static_cast<size_t>(total_q) * H * d * 2;
  const size_t kb = static_cast<size_t>(total_k) * H * d * 2;
  const size_t lb = static_cast<size_t>(total_q) * H * 4, cb = static_cast<size_t>(B + 1) * 4;
  const void* outs[4] = {dq, dk, dv, workspace};
  const size_t out_bytes[4] = {qb, kb, kb, lay.total};
  const void* ins[8] = {q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k};
  const size_t in_bytes[8] = {qb, kb, kb, qb, qb, lb, cb, cb};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 8; ++j)
      if (overlaps(outs[i], out_bytes[i], ins[j], in_bytes[j])) return FA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], out_bytes[i], outs[j], out_bytes[j])) return FA_ERR_INVALID_ARG;
  }
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  if ((rc = get_encoder()) != FA_OK) return rc;
  const bool bf16 = in_dtype == FA_BF16;
  CUtensorMap tq, tk, tv, tdo;
  if ((rc = make_map_packed(&tq, q, total_q, H, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map_packed(&tdo, dout, total_q, H, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map_packed(&tk, k, total_k, H, d, bf16)) != FA_OK) return rc;
  if ((rc = make_map_packed(&tv, v, total_k, H, d, bf16)) != FA_OK) return rc;
  fa::BwdParams p{};
  p.BH = B * H;
  p.Nq = max_seqlen_q;
  p.Nkv = max_seqlen_k;
  p.off = 0;  // per sequence in the kernels
  p.causal = causal;
  p.n_qtiles = (max_seqlen_q + 127) / 128;
  p.nq_pad = p.n_qtiles * 128;
  p.n_ktiles = static_cast<int>(n_ktiles);
  p.scale = scale;
  p.scale_log2 = scale_log2(scale);
  float* w = static_cast<float*>(workspace);
  const size_t hr = static_cast<size_t>(H) * lay.rows_max;
  p.nlse2 = w;
  p.delta = w + hr;
  p.dq_acc = w + 2 * hr;
  p.dk = dk;
  p.dv = dv;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.B = B;
  p.H = H;
  p.total_q = total_q;
  p.total_k = total_k;
  p.rows_max = lay.rows_max;
  char* base = static_cast<char*>(workspace);
  p.vl_count = reinterpret_cast<int*>(base + lay.plan_off);
  p.vl_seqs = reinterpret_cast<int4*>(base + lay.seqs_off);
  p.vl_qpad = reinterpret_cast<int*>(base + lay.qpad_off);
  p.vl_items = reinterpret_cast<int*>(base + lay.items_off);
  cudaError_t e = fa::launch_backward(tq, tk, tv, tdo, o, dout, lse, dq, p, d, bf16,
                                      ds->sm_count, ds->status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_fwd_fp8_quant(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
                     int in_dtype, int o_dtype) {
  int rc = check_args(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != FA_OK) return rc;
  if ((rc = get_encoder()) != FA_OK) return rc;
  const size_t BH = static_cast<size_t>(B) * H;
  const int nqt = (Nq + 127) / 128, nkt = (Nkv + 127) / 128;
  const long long units = static_cast<long long>(BH) * ((nqt + 1) / 2);
  if (units > 0x7fffffffLL || static_cast<long long>(BH) * nkt > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  auto up256 = [](size_t x) { return (x + 255) / 256 * 256; };
  // Call-local workspace: Q codes, K codes, Q tile scales, K tile scales.
  const size_t qb = up256(BH * Nq * d), kb = up256(BH * Nkv * d);
  const size_t qsb = up256(BH * nqt * 4), ksb = up256(BH * nkt * 4);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  if ((rc = workspace_alloc(ds, qb + kb + qsb + ksb, st, &ws)) != FA_OK) return rc;
  char* w = static_cast<char*>(ws);
  void* q8 = w;
  void* k8 = w + qb;
  float* qs = reinterpret_cast<float*>(w + qb + kb);
  float* ks = reinterpret_cast<float*>(w + qb + kb + qsb);
  const bool bf16 = in_dtype == FA_BF16;
  cudaError_t e = fa::launch_quantize_e4m3_qk(q, Nq, q8, qs, k, Nkv, k8, ks, bf16,
                                              static_cast<long long>(BH), st);
  CUtensorMap tq, tk, tv;
  if (e == cudaSuccess) {
    if ((rc = make_map_u8(&tq, q8, Nq, static_cast<long long>(BH), d)) != FA_OK ||
        (rc = make_map_u8(&tk, k8, Nkv, static_cast<long long>(BH), d)) != FA_OK ||
        (rc = make_map(&tv, v, Nkv, static_cast<long long>(BH), d, bf16)) != FA_OK) {
      cudaFreeAsync(ws, st);
      return rc;
    }
    fa::PrefillParams p{};
    p.BH = static_cast<int>(BH);
    p.Nq = Nq;
    p.Nkv = Nkv;
    p.off = Nkv - Nq;
    p.causal = causal;
    p.n_qtiles = nqt;
    p.n_pairs = (nqt + 1) / 2;
    p.n_kvtiles = nkt;
    p.n_units = static_cast<int>(units);
    p.scale_log2 = scale_log2(scale);
    p.H = H;
    p.q_tscale = qs;
    p.k_tscale = ks;
    long long grid = ds->sm_count;
    if (grid > units) grid = units;
    if (grid < 1) grid = 1;
    e = fa::launch_prefill(tq, tk, tv, o, lse, p, d, bf16, o_dtype == FA_F32,
                           static_cast<int>(grid), ds->status, st, true);
  }
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (e == cudaSuccess) e = ef;
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_quantize_e4m3(const void* x, int in_dtype, int BH, int N, int d, void* codes,
                     float* scales, void* stream) {
  if (!x || !codes || !scales) return FA_ERR_INVALID_ARG;
  if (BH < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (in_dtype != FA_F16 && in_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return FA_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(BH) * N * d;
  const size_t sb = static_cast<size_t>(BH) * ((N + 127) / 128) * 4;
  if (overlaps(codes, n, x, 2 * n) || overlaps(scales, sb, x, 2 * n) || overlaps(scales, sb, codes, n))
    return FA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  const int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  const cudaError_t e = fa::launch_quantize_e4m3(x, in_dtype == FA_BF16, BH, N, codes, scales,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int total_q,
                  int total_k, int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal,
                  void* stream, int in_dtype, int o_dtype) {
  const int rc = check_varlen_args(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q,
                                   total_k, max_seqlen_q, max_seqlen_k, d, scale, causal,
                                   in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  return run_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k,
                    max_seqlen_q, max_seqlen_k, d, scale, causal, stream, in_dtype, o_dtype);
}

int fa_fwd_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                        const int* block_table, const int* seq_lens, void* o, float* lse,
                        int B, int H, int d, int page_size, int max_pages_per_seq,
                        int num_pages, float scale, void* stream, int in_dtype, int o_dtype,
                        int num_splits) {
  const int rc = check_paged_args(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, H, d,
                                  page_size, max_pages_per_seq, num_pages, scale, in_dtype,
                                  o_dtype, num_splits);
  if (rc != FA_OK) return rc;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  const fa::PagedKV pk{block_table, seq_lens, H, shift, max_pages_per_seq, num_pages};
  // Every head gets the table's capacity of key slots; the kernels skip the empty ones.
  return run_decode(q, k_cache, v_cache, o, lse, B, H, max_pages_per_seq * page_size, d, scale,
                    stream, in_dtype, o_dtype, num_splits, &pk);
}

int fa_decode_workspace_bytes(int B, int H, int Nkv, int d, int num_splits, size_t* bytes) {
  if (!bytes || B < 1 || H < 1 || Nkv < 1 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  int sms = 148;
  DeviceState* ds = nullptr;
  if (num_splits == 0) {
    int rc = device_state(&ds);
    if (rc != FA_OK) return rc;
    sms = ds->sm_count;
  }
  *bytes = decode_ws_bytes(decode_params(B, H, Nkv, 1.0f, num_splits, sms), d);
  return FA_OK;
}

int fa_device_status(int* status, int clear) {
  if (!status) return FA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  int word = 0;
  cudaError_t e = cudaMemcpy(&word, ds->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear && word != 0) {
    e = cudaMemset(ds->status, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *status = word;
  return word ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
}

int fa_selftest_wait_timeout(void* stream) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != FA_OK) return rc;
  cudaError_t e = fa::launch_wait_timeout_selftest(ds->status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_release_workspace(void) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (s.pool) {
    // Every free the kernels' calls enqueued has completed once the device is idle.
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemPoolTrimTo(s.pool, 0)) != cudaSuccess) return cuda_fail(e);
  }
  return FA_OK;
}

int fa_get_last_cuda_error(int* cuda_err) {
  if (!cuda_err) return FA_ERR_INVALID_ARG;
  *cuda_err = g_last_cuda_error;
  g_last_cuda_error = 0;
  return FA_OK;
}

int fa_last_cuda_error(void) { return g_last_cuda_error; }

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_ARCH: return "device is not sm_100 (B200)";
    case FA_ERR_CUDA: return "CUDA runtime error";
    case FA_ERR_NOMEM: return "out of device memory";
    case FA_ERR_DEVICE_TIMEOUT: return "a kernel wait timed out";
    default: return "unknown status";
  }
}

int fa_version(void) { return 100; }

}  // extern "C"

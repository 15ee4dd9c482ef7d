// fa_noalloc.cu -- split-KV decode that allocates no device memory.
//
// fa_fwd_decode keeps its split partials in a workspace it allocates with cudaMalloc on
// first use.  Some callers cannot allow that: a runtime that has already handed all
// device memory to its own pool, a plug-in inside a host program that forbids device
// allocations after start-up, or latency-critical code that cannot pay for the device
// synchronisation cudaMalloc and cudaFree imply.  fa_fwd_decode_noalloc runs the same
// two kernels with the partials (and the kernels' status word) in the fixed array below
// instead.  Every GPU that loads this library holds the array until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

// Static scratch: [0, 256) status word, then the decode partials (O_s, then lse_s).
static __device__ __align__(256) unsigned char g_decode_scratch[FA_NOALLOC_SCRATCH_BYTES];
constexpr size_t kStatusBytes = 256;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_ready[kMaxDevices] = {};
unsigned char* g_scratch_ptr[kMaxDevices] = {};  // device address of g_decode_scratch
int g_sm_count[kMaxDevices] = {};
thread_local int g_noalloc_cuda_error = 0;

// Once per device, with that device current: checks the architecture and looks up the
// device address of the static array.  In host code `g_decode_scratch` names only a host
// stand-in, never the device memory, so kernels must be given this address.
int setup_device(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) { g_noalloc_cuda_error = e; return FA_ERR_CUDA; }
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ready[dev]) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) {
      g_noalloc_cuda_error = e;
      return FA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return FA_ERR_ARCH;
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      g_noalloc_cuda_error = (e != cudaSuccess) ? e : cudaErrorInvalidSymbol;
      return FA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<unsigned char*>(ptr);
    g_sm_count[dev] = sms;
    g_ready[dev] = true;
  }
  *dev_out = dev;
  return FA_OK;
}

}  // namespace

extern "C" int fa_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* o,
                                     float* lse, int B, int H, int Nkv, int d, float scale,
                                     void* stream, int in_dtype, int o_dtype, int num_splits) {
  int rc = fa::check_decode_call(q, k, v, o, lse, B, H, Nkv, d, scale, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (num_splits < 0) return FA_ERR_INVALID_ARG;
  int dev = 0;
  if ((rc = setup_device(&dev)) != FA_OK) return rc;
  const fa::DecodeParams p = fa::plan_decode(B, H, Nkv, scale, num_splits, g_sm_count[dev]);
  // Too large for the fixed array: refuse before anything is enqueued.
  if (kStatusBytes + fa::decode_workspace_bytes(p, d) > FA_NOALLOC_SCRATCH_BYTES)
    return FA_ERR_UNSUPPORTED;
  // The partials need no clearing: every record the combine kernel reads is written by the
  // split kernel of the same call.  The status word is only ever OR-ed into.
  unsigned char* base = g_scratch_ptr[dev];
  int* status = reinterpret_cast<int*>(base);
  float* part_o = reinterpret_cast<float*>(base + kStatusBytes);
  float* part_lse = part_o + static_cast<size_t>(p.grid) * p.max_seg * 8 * d;
  cudaError_t e = fa::launch_decode(q, k, v, o, lse, p, d, in_dtype == FA_BF16,
                                    o_dtype == FA_F32, part_o, part_lse, status,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) { g_noalloc_cuda_error = e; return FA_ERR_CUDA; }
  return FA_OK;
}

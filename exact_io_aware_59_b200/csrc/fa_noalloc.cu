// fa_noalloc.cu -- split-KV decode that allocates no device memory.
//
// fa_fwd_decode takes its split partials from a stream-ordered memory pool that the
// library creates and grows on demand.  Some callers cannot allow any device allocation
// by a library: a runtime that has already handed all device memory to its own pool, a
// plug-in inside a host program that forbids device allocations after start-up, or code
// that must not depend on an allocator's state for its latency.  fa_fwd_decode_noalloc
// runs the same two kernels with the partials in the fixed array below instead.  Every
// GPU that loads this file's module holds the array until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

// Static scratch for the decode partials (O_s, then lse_s).
static __device__ __align__(256) unsigned char g_decode_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_scratch_ptr[kMaxDevices] = {};  // device address of g_decode_scratch

// Once per device, with that device current: looks up the device address of the static
// array.  In host code `g_decode_scratch` names only a host stand-in, never the device
// memory, so kernels must be given this address.  With CUDA's lazy module loading this
// lookup is what loads the module, and so what commits the array's memory on the device:
// an allocation failure there is reported as FA_ERR_NOMEM.
int setup_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fa::cuda_failure(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e == cudaErrorMemoryAllocation) return FA_ERR_NOMEM;
    if (e != cudaSuccess) return fa::cuda_failure(e);
    if (ptr == nullptr) return fa::cuda_failure(cudaErrorInvalidSymbol);
    g_scratch_ptr[dev] = static_cast<unsigned char*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" int fa_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* o,
                                     float* lse, int B, int H, int Nkv, int d, float scale,
                                     void* stream, int in_dtype, int o_dtype, int num_splits) {
  int rc = fa::check_decode_call(q, k, v, o, lse, B, H, Nkv, d, scale, in_dtype, o_dtype);
  if (rc != FA_OK) return rc;
  if (num_splits < 0) return FA_ERR_INVALID_ARG;
  // The architecture check, the SM count and the status word (a static device variable,
  // shared with the other entry points) come from the library's per-device state, which
  // allocates nothing.
  int sm_count = 0;
  int* status = nullptr;
  if ((rc = fa::current_device(&sm_count, &status)) != FA_OK) return rc;
  const fa::DecodeParams p = fa::plan_decode(B, H, Nkv, scale, num_splits, sm_count);
  // Too large for the fixed array: refuse before anything is enqueued.
  if (fa::decode_workspace_bytes(p, d) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  unsigned char* base = nullptr;
  if ((rc = setup_scratch(&base)) != FA_OK) return rc;
  // The partials need no clearing: every record the combine kernel reads is written by the
  // split kernel of the same call, unless a split kernel's wait runs out, which the status
  // word reports (fa_device_status); the outputs of such a call are undefined.
  float* part_o = reinterpret_cast<float*>(base);
  float* part_lse = part_o + static_cast<size_t>(p.grid) * p.max_seg * fa::kDecodeRecords * d;
  const cudaError_t e = fa::launch_decode(q, k, v, o, lse, p, d, in_dtype == FA_BF16,
                                          o_dtype == FA_F32, part_o, part_lse, status,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : fa::cuda_failure(e);
}

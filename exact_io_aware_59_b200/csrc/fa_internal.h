// fa_internal.h -- launch interfaces shared by the host API and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Work description of one prefill launch (all sizes in elements / rows / tiles).

struct PrefillParams {
  int BH;           // B * H
  int Nq, Nkv;
  int off;          // Nkv - Nq: causal query i sees keys j <= i + off
  int causal;       // 0: no mask; 1: causal (bottom-right aligned when Nq != Nkv)
  int n_qtiles;     // ceil(Nq / 128)
  int n_pairs;      // ceil(n_qtiles / 2): a CTA work unit is two consecutive Q tiles
                    // (n_qtiles with interleaved-K/V units: one Q tile)
  int n_kvtiles;    // ceil(Nkv / 128)
  int n_units;      // BH * n_pairs
  float scale_log2; // scale * log2(e)
  // Packed variable-length batches (null cu_q: the [B,H,N,d] layout above).  Then
  // Nq / Nkv are the longest query / key sequences, q/o are [total_q, H, d], k/v
  // [total_k, H, d], and sequence b owns tokens cu[b] .. cu[b+1]-1.
  const int* cu_q;
  const int* cu_k;
  int H;            // heads per sequence (bh = b * H + h)
  int total_q, total_k;
  // K/V split of problems with fewer units than SMs (> 1; 1: no split; 0: no split, and
  // interleaved-K/V units: a unit is one Q tile whose even K/V tiles go to one softmax
  // warpgroup and odd ones to the other, the two partial outputs merged at the end, for
  // small launches, see run_prefill): each (b*h,
  // Q-tile pair) becomes n_splits units over consecutive parts of its K/V tile range.  A
  // unit writes its rows' partial output (divided by the part's own row sum) and natural
  // log-sum-exp in fp32 to the kernel's o [n_splits, BH*Nq, d] and lse [n_splits, BH*Nq]
  // arguments, which the combine kernel then merges into the caller's O and LSE.
  int n_splits;
  // The packed batch's work list, built on the device by the plan kernel that runs before
  // the prefill kernel (call-local workspace): the number of (sequence, Q-tile pair) items
  // that hold query rows, each sequence's (q0, Lq, k0, Lk) after the bounds checks and the
  // position of its first item, and the items, each as b * n_pairs + pair.  Work unit u is
  // head u % H of item u / H.
  const int* vl_count;
  // Work counter of the packed batch: zeroed by the plan kernel; the prefill kernel's CTAs
  // claim units from it in list order.
  int* vl_next;
  const int4* vl_seqs;
  const int* vl_first;
  const int* vl_items;
  // E4M3 queries and keys with one scale per 128-row tile (null: per-tensor scales folded
  // into scale_log2): [BH, n_qtiles] and [BH, n_kvtiles].
  const float* q_tscale;
  const float* k_tscale;
};

// Work description of one backward launch ([B,H,N,d] layout, d = 64 or 128).
struct BwdParams {
  int BH;
  int Nq, Nkv;
  int off;          // Nkv - Nq: causal query i sees keys j <= i + off
  int causal;
  int n_qtiles;     // ceil(Nq / 128)
  int nq_pad;       // n_qtiles * 128: rows of the per-row workspace arrays
  int n_ktiles;     // ceil(Nkv / 128): one CTA per (key tile, b*h)
  float scale;
  float scale_log2; // scale * log2(e)
  // Workspace (written by the prep kernel): -LSE*log2(e) and D = rowsum(dO * O) per padded
  // query row, and the fp32 dQ accumulator, [BH, nq_pad, d] row-major.
  float* nlse2;
  float* delta;
  float* dq_acc;
  void* dk;         // [BH, Nkv, d], the inputs' 16-bit type
  void* dv;
  // Packed variable-length batches (null cu_q: the [B,H,N,d] layout above).  Then q, o,
  // dO, dQ are [total_q, H, d], k, v, dK, dV [total_k, H, d] and lse [total_q, H]; Nq and
  // Nkv are the longest sequences (n_qtiles, n_ktiles taken from them); head h's workspace
  // rows start at h * rows_max, each sequence's query rows padded to whole 128-row tiles.
  const int* cu_q;
  const int* cu_k;
  int B, H;
  int total_q, total_k;
  long long rows_max;
  // Written by the plan kernel that runs first (workspace): each sequence's (q0, Lq, k0,
  // Lk) after the bounds checks, its first workspace row (entry B: the rows used), the
  // (sequence, key tile) items as b * n_ktiles + kt, and their count.
  int4* vl_seqs;
  int* vl_qpad;
  int* vl_items;
  int* vl_count;
};

// Work description of one split-KV decode launch.
struct DecodeParams {
  int BH;
  int Nkv;
  int n_chunks;       // chunks of kDecodeChunk keys per head
  long long total;    // BH * n_chunks
  int grid;           // CTAs: CTA c owns chunks [c*total/grid, (c+1)*total/grid)
  int max_seg;        // most heads one CTA's chunk range can touch
  float scale_log2;
};

constexpr int kDecodeChunk = 64;
// Partial records the split decode writes per CTA and head segment: one per consumer warp.
constexpr int kDecodeRecords = 16;

// Paged KV cache of a decode launch (null block_table: contiguous [B,H,Nkv,d] K/V).
struct PagedKV {
  const int* block_table;  // [B, max_pages] physical page of each logical page
  const int* seq_lens;     // [B] keys per sequence
  int H;                   // heads per sequence (flat head = b * H + h)
  int page_shift;          // log2(page_size)
  int max_pages;           // logical pages per sequence (table row length)
  int num_pages;           // physical pages in the caches
};

// Kernel launchers (fa_prefill.cu, fa_decode.cu).  Return the launch's cudaError_t.
// qk8: tq / tk hold E4M3 codes (d = 128, box 128 x 128 bytes); bf16 then names V's type.
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           void* o, float* lse, const PrefillParams& p, int d, bool bf16,
                           bool o_f32, int grid, int* status, cudaStream_t stream,
                           bool qk8 = false, float* part_o = nullptr, float* part_lse = nullptr);

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                          const DecodeParams& p, int d, bool bf16, bool o_f32, float* part_o,
                          float* part_lse, int* status, cudaStream_t stream,
                          const PagedKV* paged = nullptr);

// Backward: prep, main and dQ-conversion kernels on `stream` (fa_backward.cu).  All four
// maps have 128-row boxes.
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const void* o, const void* dout,
                            const float* lse, void* dq, const BwdParams& p, int d, bool bf16,
                            int sm_count, int* status, cudaStream_t stream);
size_t backward_smem_bytes(int d);

// E4M3 codes of x [BH, N, 128] (16-bit) with one scale per 128-row tile of one head
// (fa_quant.cu): codes [BH, N, 128] bytes, scales [BH, ceil(N / 128)] fp32.
cudaError_t launch_quantize_e4m3(const void* x, bool bf16, long long BH, int N, void* codes,
                                 float* scales, cudaStream_t stream);
// Q and K of one call in a single launch (each [BH, N, 128], one scale per 128-row tile).
cudaError_t launch_quantize_e4m3_qk(const void* q, int Nq, void* q8, float* qs, const void* k,
                                    int Nkv, void* k8, float* ks, bool bf16, long long BH,
                                    cudaStream_t stream);

// Diagnostic kernel whose only wait can never finish (see fa_selftest_wait_timeout).
cudaError_t launch_wait_timeout_selftest(int* status, cudaStream_t stream);

// Host-side pieces of the decode entry point, shared with other entry files (fa_api.cu).
int check_decode_call(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int Nkv, int d, float scale, int in_dtype, int o_dtype);
DecodeParams plan_decode(int B, int H, int Nkv, float scale, int num_splits, int sm_count);
size_t decode_workspace_bytes(const DecodeParams& p, int d);

// Records `e` as this host thread's last CUDA error (what fa_get_last_cuda_error reports)
// and returns FA_ERR_CUDA (fa_api.cu).
int cuda_failure(cudaError_t e);

// The current device's SM count and status-word address, set up on first use (checks the
// architecture; allocates nothing).  Returns an FA_* status (fa_api.cu).
int current_device(int* sm_count, int** status);

// One-time, thread-safe set-up of a kernel on the CURRENT device: opts it into
// `smem_bytes` of dynamic shared memory and, when min_regs > 0, checks that it was built
// with at least that many registers per thread (setmaxnreg redistributes them).  Later
// calls on the same device return the first call's result (fa_api.cu).
cudaError_t configure_kernel(const void* kernel, int smem_bytes, int min_regs);

// Bytes of dynamic shared memory each kernel needs.
size_t prefill_smem_bytes(int d);
size_t decode_smem_bytes(int d);

}  // namespace fa

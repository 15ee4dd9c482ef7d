/*
 * fa.h -- C ABI of libfa_b200.so: exact fused scaled-dot-product attention on NVIDIA
 * B200 (sm_100a): the forward (prefill, decode, paged decode, packed varlen, FP8 Q/K) and
 * the backward (fa_bwd).
 *
 * What is computed ("Flash Attention -- Module 12.3" (aicurriculum), section
 * "Definition": exact softmax(Q K^T / sqrt(d)) V; "FlashAttention" (fp-ai-systems),
 * sections "The problem: the n x n score matrix" and "The fix: tile through SRAM, fuse
 * the passes"; "FlashAttention 1-2-3" (myaihardware), sections "FlashAttention-1",
 * "FlashAttention-2" (causal block skipping), "The Math Behind the Online Softmax
 * Trick" and "Beyond FlashAttention" (split-KV decoding)):
 *
 *     S   = scale * Q K^T            (never written to memory)
 *     P   = softmax(S [+ causal mask]) over each row
 *     O   = P V
 *     LSE = per-row natural log of sum_j exp(S_ij) over the visible keys
 *
 * Layouts (all contiguous, d innermost, no strides):
 *     q   [B, H, Nq,  d]   16-bit (in_dtype)
 *     k   [B, H, Nkv, d]   16-bit (in_dtype)
 *     v   [B, H, Nkv, d]   16-bit (in_dtype)
 *     o   [B, H, Nq,  d]   o_dtype (FA_F32, or the same 16-bit type as the inputs)
 *     lse [B, H, Nq]       fp32, natural log; may be NULL (then not written)
 * All pointers are DEVICE pointers on the current CUDA device; q, k, v and o must be
 * 16-byte aligned, lse 4-byte aligned.  K and V have H heads like Q.
 *
 * Causal masking: query i sees key j iff j <= i + (Nkv - Nq) (aligned bottom-right; the
 * pages only show square masks, where this is the usual lower triangle).  A query that
 * sees no key (only possible when Nq > Nkv) gets O = 0 and LSE = -inf.
 *
 * Ownership and ordering: the caller owns every buffer.  Calls only enqueue work on
 * `stream` (a cudaStream_t; NULL = the legacy default stream) and never synchronise
 * it; the buffers must stay valid until that work has finished.  The library keeps no
 * pointer to caller memory after a call returns.  Per device it owns a status word (a
 * static device variable: nothing is allocated for it) and a stream-ordered memory pool
 * for call-local workspace (the decode split partials, the varlen unit list): a call
 * that needs workspace allocates it from the pool on `stream` (cudaMallocFromPoolAsync)
 * and frees it on `stream` after its last kernel (cudaFreeAsync), so calls on different
 * streams never share workspace, no call synchronises, and under stream capture the pair
 * becomes graph memory nodes.  The pool is created on the first call that needs it and
 * keeps freed memory mapped for reuse until fa_release_workspace().
 *
 * Errors: argument checks run on the host before anything is enqueued; a failed check
 * returns its code and launches nothing.  FA_ERR_CUDA means a CUDA runtime call failed;
 * fa_get_last_cuda_error() returns the cudaError_t.  Device-side faults are never raised on
 * purpose: every wait inside the kernels is bounded (about 1 s); a wait that runs out
 * sets bits in the device status word and the kernel returns early, leaving the outputs
 * undefined.  Read (and clear) that word with fa_device_status() after synchronising.
 *
 * Determinism: tile sizes, the CTA count and the split partition depend only on the
 * shape and the device, so equal inputs give bitwise-equal outputs.  The one exception
 * is fa_bwd's dQ, summed in fp32 across key tiles in arrival order (its dK and dV are
 * bitwise reproducible).
 */
#ifndef FA_B200_H_
#define FA_B200_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, misalignment, overlap, ... */
  FA_ERR_UNSUPPORTED = 2,     /* valid request the library does not implement (d, dtype pair) */
  FA_ERR_ARCH = 3,            /* current device is not compute capability 10.0 (B200) */
  FA_ERR_CUDA = 4,            /* a CUDA runtime call failed: see fa_get_last_cuda_error() */
  FA_ERR_NOMEM = 5,           /* device memory for workspace (or a static array) ran out */
  FA_ERR_DEVICE_TIMEOUT = 6   /* fa_device_status(): a kernel's bounded wait ran out */
};

/* Element types. */
enum { FA_F16 = 0, FA_BF16 = 1, FA_F32 = 2 };

/*
 * fa_fwd -- attention forward; the general entry point.
 *   Nq == 1 runs the split-KV decode path (every key is visible to the single query
 *   whatever `causal` says, by the bottom-right alignment); Nq > 1 runs the tiled
 *   prefill path.
 *   B, H, Nq, Nkv >= 1; d in {64, 128}; B*H <= 2^31-1; scale any finite float (use
 *   1/sqrt(d) for the usual attention); causal 0 or 1; in_dtype FA_F16 or FA_BF16;
 *   o_dtype FA_F32 or equal to in_dtype.  o must not overlap q, k, v or lse.
 * Returns FA_OK once the work is enqueued.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
           int Nq, int Nkv, int d, float scale, int causal, void* stream, int in_dtype,
           int o_dtype);

/*
 * fa_fwd_prefill -- the tiled prefill path for any Nq >= 1 (the work of fa_fwd with
 * Nq > 1).  num_ctas: persistent CTAs to launch; 0 picks one per SM (and splits the K/V
 * range of small problems as fa_fwd_prefill_split does with num_splits = 0), larger values
 * are clamped to the number of work units and run them unsplit.  A work unit is a pair of
 * 128-row query tiles; in an unsplit launch with at least one CTA per pair (causal) or per
 * query tile (non-causal) it is a single query tile whose even and odd key tiles two
 * warpgroups of the CTA take at once (the two partial results merged by their
 * log-sum-exp).  Results do not depend on the grid size within either regime.  Same
 * arguments, layouts and errors as fa_fwd.
 */
int fa_fwd_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
                   int in_dtype, int o_dtype, int num_ctas);

/*
 * fa_fwd_prefill_split -- the prefill path with the K/V range of every (head, Q-tile pair)
 * cut into num_splits consecutive parts of whole 128-key tiles, each part a work unit of
 * its own.  Each unit writes, per query row, the softmax-weighted mean of V over its part's
 * keys and that part's log-sum-exp (fp32, to workspace from the library's stream-ordered
 * pool); a combine kernel then merges the parts exactly: with w_s = exp(lse_s - max lse),
 * O = sum w_s O_s / sum w_s and LSE = max lse + log sum w_s.  This is the decode path's
 * split-KV merge ("FlashAttention 1-2-3" (myaihardware), the FlashDecoding split of section
 * "Beyond FlashAttention") applied to prefills with fewer Q-tile pairs than SMs, where the
 * longest pair would otherwise set the run time alone.
 *   num_splits: 0 chooses (fa_prefill_num_splits: 1 once there are at least as many
 *   units as SMs, else the count, up to 8, that a run-time model of the kernel predicts
 *   to be fastest, if it beats no split by at least 10%); 1 runs unsplit; 2..64 forces
 *   that many parts (clamped to the K/V tile count).
 *   num_ctas as for fa_fwd_prefill (0: one per SM; clamped to the split unit count).
 *   Workspace: num_splits * B*H*Nq * (d + 1) * 4 bytes, allocated and freed on `stream`.
 *   Same arguments, layouts, results (up to the merge's rounding) and errors as fa_fwd,
 *   plus FA_ERR_INVALID_ARG for num_ctas < 0 or num_splits outside 0..64, and FA_ERR_NOMEM
 *   when the pool cannot supply the workspace.
 */
int fa_fwd_prefill_split(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int Nq, int Nkv, int d, float scale, int causal,
                         void* stream, int in_dtype, int o_dtype, int num_ctas, int num_splits);

/*
 * fa_prefill_num_splits -- the K/V part count the prefill path chooses by itself (fa_fwd
 * with Nq > 1, fa_fwd_prefill with num_ctas = 0, fa_fwd_prefill_split with num_splits = 0)
 * for this shape on a GPU with sm_count SMs (0: the current device's), written to
 * *num_splits; the split workspace of a call is then *num_splits * B*H*Nq * (d + 1) * 4
 * bytes when *num_splits > 1.  Host arithmetic only when sm_count > 0.  FA_ERR_INVALID_ARG
 * for a null pointer, B, H, Nq or Nkv < 1, d not 64 or 128, causal not 0 or 1, or
 * sm_count < 0.
 */
int fa_prefill_num_splits(int B, int H, int Nq, int Nkv, int d, int causal, int sm_count,
                          int* num_splits);

/*
 * fa_fwd_decode -- split-KV decode for one query per head: q [B,H,1,d], k/v [B,H,Nkv,d],
 * o [B,H,1,d], lse [B,H,1].  num_splits: CTAs that split the flat range of all heads'
 * 64-key chunks evenly between them (0 picks one per SM; clamped to the chunk count).
 * Enqueues the split kernel and the fp32 log-sum-exp combine kernel on `stream`.
 */
int fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int H, int Nkv, int d, float scale, void* stream, int in_dtype, int o_dtype,
                  int num_splits);

/*
 * fa_fwd_decode_noalloc -- fa_fwd_decode for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment variant, not part of the method.
 *   Who needs it: fa_fwd_decode takes its split partials from a memory pool the library
 *   creates and grows on demand, and some callers cannot allow a library to allocate --
 *   a runtime that has handed all device memory to its own pool, a plug-in whose host
 *   program forbids device allocations after start-up, or code whose latency must not
 *   depend on an allocator's state.
 *   What it does: the same split-KV decode and combine kernels, same arguments, layouts
 *   and results as fa_fwd_decode, with the split partials kept in one fixed static device
 *   array of FA_NOALLOC_SCRATCH_BYTES bytes.  The caller still passes q, k, v, o and lse.
 *   No cudaMalloc, cudaFree or other allocating routine is called.
 *   Limit: a call whose partials need more than the array (G * max_seg * 16 * (d+1) * 4
 *   bytes, the figure fa_decode_workspace_bytes returns) is refused with
 *   FA_ERR_UNSUPPORTED before anything is enqueued.  With the default split count (one
 *   CTA per SM, 148 on B200) that holds for B*H up to 740 heads at d = 128 and 1,776 at
 *   d = 64, for any Nkv (B=16, H=32, d=128 needs 6.1 MB).
 *   First call: the first call on each device (made with that device current) looks up
 *   the array's device address.  Under CUDA's default lazy module loading that lookup is
 *   what loads the array's module, so it is the moment the 8 MiB are committed on that
 *   device (FA_ERR_NOMEM if they cannot be); make that first call before the caller's own
 *   pool claims the device's memory.  Every GPU where that happened holds the array until
 *   the process exits.
 *   Sharing: every call on a device uses the same array, which keeps the last call's
 *   contents.  Nothing in it needs clearing between calls.  Calls whose kernels can
 *   overlap on the GPU (different streams without ordering between them) race on the
 *   array.  A kernel wait that runs out is recorded in the same device status word as for
 *   the other entry points (fa_device_status); the outputs of that call are undefined.
 */
#define FA_NOALLOC_SCRATCH_BYTES (8u << 20)
int fa_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int Nkv, int d, float scale, void* stream,
                          int in_dtype, int o_dtype, int num_splits);

/*
 * fa_fwd_fp8 -- prefill with FP8 queries and keys ("FlashAttention 1-2-3" (myaihardware),
 * section "FlashAttention-3: FP8, Async Warp Overlap, and Hopper-Specific Optimizations":
 * FP8 inputs to the tensor cores for Q K^T).
 *   q8 [B,H,Nq,d] and k8 [B,H,Nkv,d] hold E4M3 codes (one byte each, the "fn" variant:
 *   no infinities); they stand for q_scale * Q and k_scale * K (per-tensor scales).
 *   v [B,H,Nkv,d] in v_dtype (FA_F16 or FA_BF16), o [B,H,Nq,d] in FA_F32 or v_dtype,
 *   lse [B,H,Nq] fp32 (may be NULL).  S = Q K^T runs on tcgen05 kind::f8f6f4 (E4M3 x
 *   E4M3, fp32 accumulate); P is rounded to v_dtype for P V as in fa_fwd.  The result is
 *   softmax(scale * q_scale * k_scale * Q8 K8^T [+ causal]) V.  d must be 128.
 *   Same ownership, alignment (16 bytes for q8, k8, v, o) and error rules as fa_fwd.
 */
int fa_fwd_fp8(const void* q8, const void* k8, const void* v, void* o, float* lse, int B,
               int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
               float q_scale, float k_scale, int v_dtype, int o_dtype);

/*
 * fa_fwd_fp8_quant -- prefill with queries and keys quantised to FP8 on the fly
 * ("FlashAttention 1-2-3" (myaihardware), section "FlashAttention-3: FP8, Async Warp
 * Overlap, and Hopper-Specific Optimizations").  Same arguments, layouts and errors as
 * fa_fwd (q, k, v in in_dtype; d must be 128; Nq > 1 or 1).  Q and K are quantised with
 * fa_quantize_e4m3 (one scale per 128-row tile) into call-local workspace from the
 * library's stream-ordered pool; then S = Q8 K8^T runs on tcgen05 kind::f8f6f4 and each
 * score tile is multiplied by scale and its two tile scales; P and V stay in in_dtype.
 * The result is softmax(scale * Qd Kd^T [+ causal]) V with Qd, Kd the dequantised tensors.
 */
int fa_fwd_fp8_quant(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Nq, int Nkv, int d, float scale, int causal, void* stream,
                     int in_dtype, int o_dtype);

/*
 * fa_quantize_e4m3 -- E4M3 codes of a [BH, N, d] tensor with one scale per tile of 128
 * consecutive rows of one head ("FlashAttention 1-2-3" (myaihardware), section
 * "FlashAttention-3: FP8, Async Warp Overlap, and Hopper-Specific Optimizations": queries
 * and keys quantised to FP8 on the fly).
 *   x: [BH, N, d] in in_dtype (FA_F16 or FA_BF16), 16-byte aligned; d must be 128.
 *   codes: [BH, N, d] bytes (16-byte aligned); scales: [BH, ceil(N/128)] fp32.
 *   For the tile of rows 128t .. 128t+127 of head bh: scales[bh][t] = max|x| / 448 in fp32
 *   (1 for an all-zero tile) and code = E4M3(x / scale) in fp32, rounded to nearest even
 *   and saturated at +-448 (the "fn" variant: no infinities).  x ~ decode(code) * scale.
 *   Buffers are device memory owned by the caller and must not overlap.  Enqueues one
 *   kernel on `stream`.
 */
int fa_quantize_e4m3(const void* x, int in_dtype, int BH, int N, int d, void* codes,
                     float* scales, void* stream);

/*
 * fa_fwd_varlen -- prefill over a packed batch of sequences of different lengths
 * ("FlashAttention 1-2-3" (myaihardware), section "When FlashAttention Doesn't Help":
 * continuous batching, each sequence of the batch an independent problem).
 *   q [total_q, H, d], k/v [total_k, H, d] (token-major, fp16/bf16), o [total_q, H, d]
 *   (fp32 or q's 16-bit type), lse [total_q, H] fp32 (may be NULL).
 *   cu_seqlens_q / cu_seqlens_k: int32 [B+1] device arrays, non-decreasing, starting at
 *   0 and ending at total_q / total_k: sequence b owns query tokens cu_seqlens_q[b] ..
 *   cu_seqlens_q[b+1]-1 and key tokens likewise, and attends to its own keys only
 *   (causal mask aligned bottom-right per sequence, as for fa_fwd).  max_seqlen_q /
 *   max_seqlen_k bound every sequence's length (they size the work).  A query token
 *   whose sequence has no visible key gets O = 0 and LSE = -inf.
 *   All pointers are device memory owned by the caller, valid until the work completes;
 *   q, k, v, o 16-byte aligned, the rest 4-byte.
 *   Errors: FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED for what the host can check (nothing
 *   is enqueued).  The offsets live on the device: a range outside [0, total] or longer
 *   than its max_seqlen is clamped and FA_DEV_BAD_INPUT is set in the status word.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int total_q,
                  int total_k, int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal,
                  void* stream, int in_dtype, int o_dtype);

/*
 * fa_fwd_decode_paged -- split-KV decode for one query per head against a paged KV cache
 * ("FlashAttention 1-2-3" (myaihardware), section "Integration in Major Inference
 * Engines": each KV-cache page of vLLM's PagedAttention is a block the kernel tiles over;
 * with the FlashDecoding split of section "Beyond FlashAttention").
 *   q [B,H,d] and o [B,H,d] (o fp32 or q's 16-bit type), lse [B,H] fp32 (may be NULL).
 *   k_cache, v_cache: [num_pages, H, page_size, d] in q's 16-bit type; the page_size x d
 *   block of one head in one page is contiguous.
 *   block_table: int32 [B, max_pages_per_seq]; logical key i of sequence b is slot
 *   i % page_size of page block_table[b * max_pages_per_seq + i / page_size].
 *   seq_lens: int32 [B], keys of each sequence, 0 <= seq_lens[b] <= max_pages_per_seq *
 *   page_size; a sequence with no keys gets O = 0 and LSE = -inf.
 *   All pointers are device memory owned by the caller and must stay valid until the
 *   enqueued work completes; q, the caches and o 16-byte aligned, the rest 4-byte.
 *   page_size: a power of two from 16 to 1024.  num_splits as for fa_fwd_decode; the
 *   split covers max_pages_per_seq * page_size key slots per head, and slots past a
 *   sequence's length cost nothing but their share of the split.
 *   Errors: FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED for arguments checkable on the host
 *   (nothing is enqueued).  Table entries and lengths live on the device: an entry
 *   outside [0, num_pages) is replaced by page 0 and a length outside its range is
 *   clamped, and FA_DEV_BAD_INPUT is set in the status word (fa_device_status); no
 *   out-of-bounds read happens.  Same workspace as fa_fwd_decode.
 */
int fa_fwd_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                        const int* block_table, const int* seq_lens, void* o, float* lse,
                        int B, int H, int d, int page_size, int max_pages_per_seq,
                        int num_pages, float scale, void* stream, int in_dtype, int o_dtype,
                        int num_splits);

/*
 * fa_bwd -- gradients of fa_fwd for an upstream gradient dO ("Flash Attention -- Module
 * 12.3", section "Prefill vs Decode", "Training": the backward pass is IO-aware too).
 *   For O = softmax(scale * Q K^T [+ causal mask, bottom-right]) V and the forward's lse:
 *     P = exp(scale * Q K^T - lse) (masked entries 0), D = rowsum(dO * O),
 *     dV = P^T dO,  dS = P * (dO V^T - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
 *   P is recomputed on chip tile by tile; nothing of size Nq x Nkv is stored.
 *   q, o, dout, dq [B,H,Nq,d]; k, v, dk, dv [B,H,Nkv,d]; all in_dtype (FA_F16 or FA_BF16),
 *   contiguous, 16-byte aligned.  lse [B,H,Nq] fp32 natural log as fa_fwd writes it (a
 *   row with no visible key has -inf and gets dQ = 0).  d must be 64 or 128.
 *   workspace: caller-owned device memory of at least fa_bwd_workspace_bytes bytes,
 *   16-byte aligned; overwritten (it holds the fp32 dQ accumulator and per-row D and lse).
 *   dq, dk, dv and the workspace must not overlap each other or any input.
 *   Enqueues three kernels on `stream` and returns FA_OK; no allocation, no
 *   synchronisation.  Errors as for fa_fwd: a failed host check launches nothing; a
 *   kernel wait that runs out sets FA_DEV_TIMEOUT_BACKWARD (outputs then undefined).
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, void* workspace,
           size_t workspace_bytes, int B, int H, int Nq, int Nkv, int d, float scale,
           int causal, void* stream, int in_dtype);

/* Bytes of workspace an fa_bwd call with these sizes needs (B*H*ceil(Nq/128)*128*(8+4d)). */
int fa_bwd_workspace_bytes(int B, int H, int Nq, int d, size_t* bytes);

/*
 * fa_bwd_varlen -- fa_bwd for a packed batch of sequences of different lengths, the
 * gradients of fa_fwd_varlen: each sequence is an independent problem ("FlashAttention
 * 1-2-3" (myaihardware), section "When FlashAttention Doesn't Help"), and its backward
 * is fa_bwd's ("Flash Attention -- Module 12.3", section "Prefill vs Decode", "Training").
 *   q, o, dout, dq [total_q, H, d]; k, v, dk, dv [total_k, H, d]; lse [total_q, H] fp32 as
 *   fa_fwd_varlen writes it; cu_seqlens_q / cu_seqlens_k int32 device arrays [B+1] as for
 *   fa_fwd_varlen (sequence b: query tokens cu_q[b] .. cu_q[b+1]-1, key tokens cu_k[b] ..
 *   cu_k[b+1]-1, causal alignment bottom-right per sequence), max_seqlen_q / max_seqlen_k
 *   bounds on the lengths.  Offsets are checked on the device like fa_fwd_varlen's (a range
 *   outside [0, total] or longer than the maximum is clamped, sequences whose clamped query
 *   ranges would overrun the workspace get none, and FA_DEV_BAD_INPUT is set).  Rows of dq
 *   for tokens outside every sequence, and of dk / dv for keys outside every sequence, are
 *   not written.
 *   workspace: caller-owned device memory of at least fa_bwd_varlen_workspace_bytes bytes,
 *   16-byte aligned, overwritten: per head, total_q + 128 B rows (rounded up to a multiple
 *   of 128) of the fp32 dQ
 *   accumulator, -LSE*log2(e) and D, then the plan of the call (sequence records, padded
 *   row offsets, (sequence, key tile) work items).
 *   Four kernels on `stream` (plan, prep, main, dQ conversion); no allocation, no
 *   synchronisation.  Same dtype, alignment, overlap and error rules as fa_bwd.
 */
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dout, void* dq, void* dk, void* dv, void* workspace,
                  size_t workspace_bytes, const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                  int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                  float scale, int causal, void* stream, int in_dtype);

/* Bytes of workspace an fa_bwd_varlen call with these sizes needs. */
int fa_bwd_varlen_workspace_bytes(int B, int H, int total_q, int max_seqlen_k, int d,
                                  size_t* bytes);

/* Bytes of decode workspace a fa_fwd_decode call with these arguments needs. */
int fa_decode_workspace_bytes(int B, int H, int Nkv, int d, int num_splits, size_t* bytes);

/*
 * fa_device_status -- reads the current device's status word into *status (0 = no
 * kernel wait ran out; otherwise FA_DEV_* bits) and clears it when clear != 0.
 * Synchronous (a device-to-host copy on the legacy stream).  Returns FA_OK, or
 * FA_ERR_DEVICE_TIMEOUT when the word is non-zero.
 */
int fa_device_status(int* status, int clear);

/* Bits of the device status word. */
enum {
  FA_DEV_TIMEOUT_LOAD = 1,      /* prefill: a TMA producer wait ran out */
  FA_DEV_TIMEOUT_MMA = 2,       /* prefill: the MMA issuer's wait ran out */
  FA_DEV_TIMEOUT_SOFTMAX = 4,   /* prefill: a softmax / epilogue wait ran out */
  FA_DEV_TIMEOUT_DECODE = 8,    /* decode: a split kernel wait ran out */
  FA_DEV_BAD_INPUT = 16,        /* paged decode / varlen: a device-side table or offset out of range */
  FA_DEV_TIMEOUT_BACKWARD = 32  /* fa_bwd: a kernel wait ran out */
};

/*
 * fa_selftest_wait_timeout -- diagnostic for the error path above: enqueues a one-thread
 * kernel that waits on an mbarrier nothing ever signals.  Its bounded wait gives up after
 * about 1 s, sets FA_DEV_TIMEOUT_DECODE in the status word and returns; no fault, trap or
 * hang.  Synchronise, then fa_device_status() reports it.
 */
int fa_selftest_wait_timeout(void* stream);

/*
 * fa_release_workspace -- returns the memory the current device's workspace pool keeps
 * mapped for reuse.  Synchronises the device first (so every enqueued free has
 * completed); do not call it during stream capture.  Later calls that need workspace
 * allocate it again.
 */
int fa_release_workspace(void);

/*
 * fa_get_last_cuda_error -- writes the cudaError_t behind the last FA_ERR_CUDA returned on
 * this host thread (0 if none since the last read) to *cuda_err and clears it, like
 * cudaGetLastError.  Returns FA_OK, or FA_ERR_INVALID_ARG when cuda_err is NULL.
 */
int fa_get_last_cuda_error(int* cuda_err);

/* The same value as fa_get_last_cuda_error, without clearing it. */
int fa_last_cuda_error(void);

/* A static, human-readable name for a status code. */
const char* fa_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H_ */

"""ctypes binding of libfa_b200.so (declared in include/fa.h).

Argument marshalling only: every step of the attention runs in the library's CUDA
kernels.  The raw functions keep the C names and argument order; ``attention`` is a
convenience wrapper that takes torch CUDA tensors, allocates O and LSE and passes torch's
current stream.  There is no fallback: if the library cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional

from . import build as _build

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ARCH = 0, 1, 2, 3
FA_ERR_CUDA, FA_ERR_NOMEM, FA_ERR_DEVICE_TIMEOUT = 4, 5, 6
FA_F16, FA_BF16, FA_F32 = 0, 1, 2
FA_DEV_BAD_INPUT = 16
FA_DEV_TIMEOUT_BACKWARD = 32

HEADER = os.path.join(_build.INCLUDE, "fa.h")

_lib = None


class FaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where} failed: {status_string(code)} ({code})"
        if code == FA_ERR_CUDA and _lib is not None:
            msg += f", cudaError {int(_lib.fa_last_cuda_error())}"
        super().__init__(msg)


_VP, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_SIGNATURES = {
    "fa_fwd": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _I, _I],
    "fa_fwd_prefill": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _I, _I, _I],
    "fa_fwd_prefill_split": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _I, _I, _I,
                             _I],
    "fa_prefill_num_splits": [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_I)],
    "fa_fwd_decode": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _VP, _I, _I, _I],
    "fa_fwd_decode_noalloc": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _VP, _I, _I, _I],
    "fa_fwd_fp8": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _F, _F, _I, _I],
    "fa_fwd_varlen": [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _I, _VP,
                      _I, _I],
    "fa_fwd_decode_paged": [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP,
                            _I, _I, _I],
    "fa_quantize_e4m3": [_VP, _I, _I, _I, _I, _VP, _VP, _VP],
    "fa_fwd_fp8_quant": [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, _I, _I],
    "fa_bwd": [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _I, _I, _I, _I,
               _I, _F, _I, _VP, _I],
    "fa_bwd_workspace_bytes": [_I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)],
    "fa_bwd_varlen": [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP, _VP,
                      _I, _I, _I, _I, _I, _I, _I, _F, _I, _VP, _I],
    "fa_bwd_varlen_workspace_bytes": [_I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)],
    "fa_decode_workspace_bytes": [_I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)],
    "fa_device_status": [ctypes.POINTER(_I), _I],
    "fa_selftest_wait_timeout": [_VP],
    "fa_release_workspace": [],
    "fa_get_last_cuda_error": [ctypes.POINTER(_I)],
    "fa_last_cuda_error": [],
    "fa_status_string": [_I],
    "fa_version": [],
}


def declared_functions() -> list:
    """Names of the functions include/fa.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", text, flags=re.M)


def library(build_if_missing: bool = True) -> ctypes.CDLL:
    """Loads libfa_b200.so (building it first when it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.LIB_PATH
        if build_if_missing and not _build.up_to_date():
            _build.build()
        if not os.path.exists(path):
            raise RuntimeError(f"libfa_b200.so is missing ({path}); build it with "
                               "`python -m exact_io_aware_59_b200.build`")
        lib = ctypes.CDLL(path)
        for name, argtypes in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_char_p if name == "fa_status_string" else ctypes.c_int
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    return library().fa_status_string(int(code)).decode()


# ---------------------------------------------------------------- raw C calls
def fa_fwd(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype, o_dtype) -> int:
    return library().fa_fwd(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream,
                            in_dtype, o_dtype)


def fa_fwd_prefill(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype,
                   o_dtype, num_ctas) -> int:
    return library().fa_fwd_prefill(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream,
                                    in_dtype, o_dtype, num_ctas)


def fa_fwd_prefill_split(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype,
                         o_dtype, num_ctas, num_splits) -> int:
    return library().fa_fwd_prefill_split(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal,
                                          stream, in_dtype, o_dtype, num_ctas, num_splits)


def prefill_num_splits(B, H, Nq, Nkv, d, causal, sm_count=0) -> int:
    """The K/V part count the prefill path chooses for this shape (fa_prefill_num_splits)."""
    out = ctypes.c_int(0)
    rc = library().fa_prefill_num_splits(B, H, Nq, Nkv, d, int(bool(causal)), sm_count,
                                         ctypes.byref(out))
    if rc != FA_OK:
        raise FaError(rc, "fa_prefill_num_splits")
    return out.value


def fa_fwd_decode(q, k, v, o, lse, B, H, Nkv, d, scale, stream, in_dtype, o_dtype,
                  num_splits) -> int:
    return library().fa_fwd_decode(q, k, v, o, lse, B, H, Nkv, d, scale, stream, in_dtype,
                                   o_dtype, num_splits)


def fa_fwd_decode_noalloc(q, k, v, o, lse, B, H, Nkv, d, scale, stream, in_dtype, o_dtype,
                          num_splits) -> int:
    """fa_fwd_decode with the split partials in the library's fixed static device array
    instead of a cudaMalloc'd workspace, for callers that cannot allocate device memory."""
    return library().fa_fwd_decode_noalloc(q, k, v, o, lse, B, H, Nkv, d, scale, stream,
                                           in_dtype, o_dtype, num_splits)


def fa_fwd_fp8(q8, k8, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, q_scale, k_scale,
               v_dtype, o_dtype) -> int:
    return library().fa_fwd_fp8(q8, k8, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream,
                                q_scale, k_scale, v_dtype, o_dtype)


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k, d, scale,
                  causal, stream, in_dtype, o_dtype) -> int:
    return library().fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q,
                                   max_k, d, scale, causal, stream, in_dtype, o_dtype)


def fa_fwd_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, H, d, page_size,
                        max_pages_per_seq, num_pages, scale, stream, in_dtype, o_dtype,
                        num_splits) -> int:
    return library().fa_fwd_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, H,
                                         d, page_size, max_pages_per_seq, num_pages, scale,
                                         stream, in_dtype, o_dtype, num_splits)


def fa_quantize_e4m3(x, in_dtype, BH, N, d, codes, scales, stream) -> int:
    return library().fa_quantize_e4m3(x, in_dtype, BH, N, d, codes, scales, stream)


def fa_fwd_fp8_quant(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream, in_dtype,
                     o_dtype) -> int:
    return library().fa_fwd_fp8_quant(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, stream,
                                      in_dtype, o_dtype)


def fp8_quant_attention(q, k, v, causal: bool = False, scale: Optional[float] = None,
                        out_dtype=None, stream=None):
    """attention() with Q and K quantised to E4M3 on the fly (one scale per 128-row tile):
    q [B,H,Nq,128], k/v [B,H,Nkv,128] contiguous fp16/bf16 CUDA tensors.  Returns (o, lse)."""
    import torch

    if not all(t.is_cuda and t.is_contiguous() for t in (q, k, v)):
        raise ValueError("fp8_quant_attention() takes contiguous CUDA tensors")
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, H, Nq, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    s = torch.cuda.current_stream(q.device) if stream is None else stream
    with torch.cuda.device(q.device):
        rc = fa_fwd_fp8_quant(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), B, H, Nq, Nkv, d, scale, int(bool(causal)),
                              s.cuda_stream, _dtype_code(q.dtype), _dtype_code(o.dtype))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_fp8_quant")
    return o, lse


def quantize_e4m3(x, stream=None):
    """E4M3 codes (uint8, x's shape) and per-128-row-tile scales (fp32 [B*H, ceil(N/128)])
    of a contiguous CUDA tensor x [B, H, N, 128] (fp16/bf16)."""
    import torch

    if not (x.is_cuda and x.is_contiguous()) or x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("quantize_e4m3() takes a contiguous fp16/bf16 CUDA tensor")
    B, H, N, d = x.shape
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty((B * H, (N + 127) // 128), dtype=torch.float32, device=x.device)
    s = torch.cuda.current_stream(x.device) if stream is None else stream
    with torch.cuda.device(x.device):
        rc = fa_quantize_e4m3(x.data_ptr(), _dtype_code(x.dtype), B * H, N, d, codes.data_ptr(),
                              scales.data_ptr(), s.cuda_stream)
    if rc != FA_OK:
        raise FaError(rc, "fa_quantize_e4m3")
    return codes, scales


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Nq, Nkv, d,
           scale, causal, stream, in_dtype) -> int:
    return library().fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H,
                            Nq, Nkv, d, scale, causal, stream, in_dtype)


def fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, cu_seqlens_q,
                  cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, d, scale,
                  causal, stream, in_dtype) -> int:
    return library().fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                                   cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k,
                                   max_seqlen_q, max_seqlen_k, d, scale, causal, stream, in_dtype)


def fa_bwd_varlen_workspace_bytes(B, H, total_q, max_seqlen_k, d) -> int:
    out = ctypes.c_size_t(0)
    rc = library().fa_bwd_varlen_workspace_bytes(B, H, total_q, max_seqlen_k, d, ctypes.byref(out))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_varlen_workspace_bytes")
    return int(out.value)


def fa_bwd_workspace_bytes(B, H, Nq, d) -> int:
    out = ctypes.c_size_t(0)
    rc = library().fa_bwd_workspace_bytes(B, H, Nq, d, ctypes.byref(out))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_workspace_bytes")
    return int(out.value)


def fa_decode_workspace_bytes(B, H, Nkv, d, num_splits) -> int:
    out = ctypes.c_size_t(0)
    rc = library().fa_decode_workspace_bytes(B, H, Nkv, d, num_splits, ctypes.byref(out))
    if rc != FA_OK:
        raise FaError(rc, "fa_decode_workspace_bytes")
    return int(out.value)


def fa_device_status(clear: bool = True) -> int:
    """The current device's status word (0 = no kernel wait ran out)."""
    word = ctypes.c_int(0)
    rc = library().fa_device_status(ctypes.byref(word), int(bool(clear)))
    if rc not in (FA_OK, FA_ERR_DEVICE_TIMEOUT):
        raise FaError(rc, "fa_device_status")
    return int(word.value)


def fa_selftest_wait_timeout(stream=None) -> int:
    return library().fa_selftest_wait_timeout(stream)


def fa_get_last_cuda_error() -> int:
    """The cudaError_t behind this thread's last FA_ERR_CUDA (0 if none); clears it."""
    err = ctypes.c_int(0)
    rc = library().fa_get_last_cuda_error(ctypes.byref(err))
    if rc != FA_OK:
        raise FaError(rc, "fa_get_last_cuda_error")
    return int(err.value)


def fa_release_workspace() -> None:
    rc = library().fa_release_workspace()
    if rc != FA_OK:
        raise FaError(rc, "fa_release_workspace")


# ---------------------------------------------------------------- torch convenience
def _dtype_code(t):
    import torch

    return {torch.float16: FA_F16, torch.bfloat16: FA_BF16, torch.float32: FA_F32}[t]


def attention(q, k, v, causal: bool = False, scale: Optional[float] = None,
              out_dtype=None, out=None, lse=None, num_ctas: int = 0, num_splits: int = 0,
              path: str = "auto", stream=None):
    """O, LSE = softmax(scale * Q K^T [+ causal]) V for contiguous CUDA tensors
    q [B,H,Nq,d], k/v [B,H,Nkv,d] (fp16 or bf16).  out_dtype: torch.float32 (default) or
    the input dtype.  path: "auto" (decode when Nq == 1), "prefill" or "decode".
    num_ctas: the prefill's persistent grid (0: one CTA per SM).  num_splits: decode, the
    split CTAs (0: one per SM); prefill, the K/V parts of each Q-tile pair (0: chosen by
    the library, which splits only small problems and never under an explicit num_ctas).
    Enqueues on `stream` (default: torch's current stream) and returns (o, lse)."""
    import torch

    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("attention() takes CUDA tensors")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k and v must be contiguous [B,H,N,d]")
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q, k, v must share one dtype, float16 or bfloat16")
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if tuple(k.shape) != (B, H, Nkv, d) or tuple(v.shape) != (B, H, Nkv, d):
        raise ValueError("k and v must be [B,H,Nkv,d] with q's B, H and d")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    s = torch.cuda.current_stream(q.device) if stream is None else stream
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr())
    ic, oc = _dtype_code(q.dtype), _dtype_code(out.dtype)
    with torch.cuda.device(q.device):
        if path == "decode" or (path == "auto" and Nq == 1):
            if Nq != 1:
                raise ValueError("the decode path takes exactly one query per head")
            rc = fa_fwd_decode(*args, B, H, Nkv, d, scale, s.cuda_stream, ic, oc, num_splits)
            where = "fa_fwd_decode"
        elif path in ("prefill", "auto") and num_splits == 0:
            rc = fa_fwd_prefill(*args, B, H, Nq, Nkv, d, scale, int(bool(causal)), s.cuda_stream,
                                ic, oc, num_ctas)
            where = "fa_fwd_prefill"
        elif path in ("prefill", "auto"):
            rc = fa_fwd_prefill_split(*args, B, H, Nq, Nkv, d, scale, int(bool(causal)),
                                      s.cuda_stream, ic, oc, num_ctas, num_splits)
            where = "fa_fwd_prefill_split"
        else:
            raise ValueError(f"unknown path {path!r}")
    if rc != FA_OK:
        raise FaError(rc, where)
    return out, lse


def paged_decode(q, k_cache, v_cache, block_table, seq_lens, scale: Optional[float] = None,
                 out_dtype=None, num_splits: int = 0, stream=None):
    """Decode against a paged KV cache: q [B,H,d]; k_cache, v_cache
    [num_pages,H,page_size,d] (q's fp16/bf16 type); block_table int32 [B,P]; seq_lens int32
    [B] -- all contiguous CUDA tensors.  Returns (o [B,H,d], lse [B,H]); out_dtype
    torch.float32 (default) or q's dtype."""
    import torch

    ts = (q, k_cache, v_cache, block_table, seq_lens)
    if not all(t.is_cuda and t.is_contiguous() for t in ts):
        raise ValueError("paged_decode() takes contiguous CUDA tensors")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    B, H, d = q.shape
    num_pages, Hc, page_size, dc = k_cache.shape
    if (Hc, dc) != (H, d) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("caches must be [num_pages, H, page_size, d] with q's H and d")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [B, P] and seq_lens [B]")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    s = torch.cuda.current_stream(q.device) if stream is None else stream
    with torch.cuda.device(q.device):
        rc = fa_fwd_decode_paged(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                 block_table.data_ptr(), seq_lens.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), B, H, d, page_size, block_table.shape[1],
                                 num_pages, scale, s.cuda_stream, _dtype_code(q.dtype),
                                 _dtype_code(o.dtype), num_splits)
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_decode_paged")
    return o, lse


def varlen_attention(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                     causal: bool = False, scale: Optional[float] = None, out_dtype=None,
                     stream=None):
    """Attention over a packed batch: q [total_q,H,d], k/v [total_k,H,d] (fp16/bf16),
    cu_seqlens_q/k int32 [B+1] -- all contiguous CUDA tensors.  Returns
    (o [total_q,H,d], lse [total_q,H])."""
    import torch

    ts = (q, k, v, cu_seqlens_q, cu_seqlens_k)
    if not all(t.is_cuda and t.is_contiguous() for t in ts):
        raise ValueError("varlen_attention() takes contiguous CUDA tensors")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    total_q, H, d = q.shape
    total_k = k.shape[0]
    if tuple(k.shape) != (total_k, H, d) or tuple(v.shape) != (total_k, H, d):
        raise ValueError("k and v must be [total_k, H, d] with q's H and d")
    B = cu_seqlens_q.numel() - 1
    if B < 1 or cu_seqlens_k.numel() != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B+1 entries")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((total_q, H, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((total_q, H), dtype=torch.float32, device=q.device)
    s = torch.cuda.current_stream(q.device) if stream is None else stream
    with torch.cuda.device(q.device):
        rc = fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, total_q,
                           total_k, int(max_seqlen_q), int(max_seqlen_k), d, scale,
                           int(bool(causal)), s.cuda_stream, _dtype_code(q.dtype),
                           _dtype_code(o.dtype))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_varlen")
    return o, lse


def fp8_attention(q8, k8, v, q_scale: float, k_scale: float, causal: bool = False,
                  scale: Optional[float] = None, out_dtype=None, stream=None):
    """Attention with E4M3 queries and keys: q8 [B,H,Nq,128], k8 [B,H,Nkv,128] as uint8 (or
    torch.float8_e4m3fn) codes standing for q_scale * Q and k_scale * K; v [B,H,Nkv,128]
    fp16/bf16.  Returns (o, lse) like attention()."""
    import torch

    if q8.dtype == torch.float8_e4m3fn:
        q8 = q8.view(torch.uint8)
    if k8.dtype == torch.float8_e4m3fn:
        k8 = k8.view(torch.uint8)
    ts = (q8, k8, v)
    if not all(t.is_cuda and t.is_contiguous() for t in ts):
        raise ValueError("fp8_attention() takes contiguous CUDA tensors")
    if q8.dtype != torch.uint8 or k8.dtype != torch.uint8:
        raise ValueError("q8 and k8 must hold E4M3 codes (uint8 or float8_e4m3fn)")
    B, H, Nq, d = q8.shape
    Nkv = k8.shape[2]
    if tuple(k8.shape) != (B, H, Nkv, d) or tuple(v.shape) != (B, H, Nkv, d):
        raise ValueError("k8 and v must be [B,H,Nkv,d] with q8's B, H and d")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, H, Nq, d), dtype=out_dtype, device=v.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=v.device)
    s = torch.cuda.current_stream(v.device) if stream is None else stream
    with torch.cuda.device(v.device):
        rc = fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                        B, H, Nq, Nkv, d, scale, int(bool(causal)), s.cuda_stream,
                        float(q_scale), float(k_scale), _dtype_code(v.dtype), _dtype_code(o.dtype))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_fp8")
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal: bool = False, scale: Optional[float] = None,
                       workspace=None, stream=None):
    """dQ, dK, dV of attention() for the upstream gradient dout.  q, o, dout [B,H,Nq,d],
    k, v [B,H,Nkv,d] (d 64 or 128) contiguous CUDA tensors of one 16-bit dtype; o and lse are the
    forward's outputs (o in the inputs' dtype, lse fp32 [B,H,Nq]).  workspace: optional
    uint8 CUDA tensor of at least fa_bwd_workspace_bytes; allocated when omitted.
    Returns (dq, dk, dv) in the inputs' dtype."""
    import torch

    ts = (q, k, v, o, dout)
    if not all(t.is_cuda and t.is_contiguous() for t in ts) or not (lse.is_cuda and lse.is_contiguous()):
        raise ValueError("attention_backward() takes contiguous CUDA tensors")
    if any(t.dtype != q.dtype for t in ts) or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q, k, v, o and dout must share one dtype, float16 or bfloat16")
    if lse.dtype != torch.float32:
        raise ValueError("lse must be float32")
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if (tuple(k.shape) != (B, H, Nkv, d) or tuple(v.shape) != (B, H, Nkv, d)
            or tuple(o.shape) != (B, H, Nq, d) or tuple(dout.shape) != (B, H, Nq, d)
            or tuple(lse.shape) != (B, H, Nq)):
        raise ValueError("shapes must be q/o/dout [B,H,Nq,d], k/v [B,H,Nkv,d], lse [B,H,Nq]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nbytes = fa_bwd_workspace_bytes(B, H, Nq, d)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    s = torch.cuda.current_stream(q.device) if stream is None else stream
    with torch.cuda.device(q.device):
        rc = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                    dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                    workspace.data_ptr(), workspace.numel() * workspace.element_size(), B, H, Nq,
                    Nkv, d, scale, int(bool(causal)), s.cuda_stream, _dtype_code(q.dtype))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


def varlen_attention_backward(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k,
                              max_seqlen_q: int, max_seqlen_k: int, causal: bool = False,
                              scale: Optional[float] = None, workspace=None, stream=None):
    """dQ, dK, dV of varlen_attention() for the upstream gradient dout.  q, o, dout
    [total_q, H, d], k, v [total_k, H, d] (d 64 or 128) contiguous CUDA tensors of one 16-bit
    dtype, lse fp32 [total_q, H] (the forward's), cu_seqlens int32 CUDA [B+1].  workspace:
    optional uint8 CUDA tensor of at least fa_bwd_varlen_workspace_bytes; allocated when
    omitted.  Returns (dq, dk, dv) in the inputs' dtype; rows of tokens outside every
    sequence are left as torch.zeros_like gives them."""
    import torch

    ts = (q, k, v, o, dout)
    if not all(t.is_cuda and t.is_contiguous() for t in ts) or not (lse.is_cuda and lse.is_contiguous()):
        raise ValueError("varlen_attention_backward() takes contiguous CUDA tensors")
    if any(t.dtype != q.dtype for t in ts) or q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("q, k, v, o and dout must share one dtype, float16 or bfloat16")
    if lse.dtype != torch.float32 or cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise ValueError("lse must be float32 and cu_seqlens int32")
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.numel() - 1
    if (tuple(k.shape) != (total_k, H, d) or tuple(v.shape) != (total_k, H, d)
            or tuple(o.shape) != (total_q, H, d) or tuple(dout.shape) != (total_q, H, d)
            or tuple(lse.shape) != (total_q, H) or cu_seqlens_k.numel() != B + 1):
        raise ValueError("shapes must be q/o/dout [total_q,H,d], k/v [total_k,H,d], lse [total_q,H]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nbytes = fa_bwd_varlen_workspace_bytes(B, H, total_q, max_seqlen_k, d)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq = torch.zeros_like(q)
    dk = torch.zeros_like(k)
    dv = torch.zeros_like(v)
    s = torch.cuda.current_stream(q.device) if stream is None else stream
    with torch.cuda.device(q.device):
        rc = fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                           workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                           cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, total_q,
                           total_k, max_seqlen_q, max_seqlen_k, d, scale, int(bool(causal)),
                           s.cuda_stream, _dtype_code(q.dtype))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_varlen")
    return dq, dk, dv

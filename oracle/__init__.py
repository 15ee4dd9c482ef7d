"""fp64 CPU oracle for exact scaled-dot-product attention forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares no code
with the CUDA library and never imports it.

Contents
--------
``attention``                 the plain definition, in C (``attn_oracle.c``), fp64, one
                              query row at a time.  Sources: "FlashAttention"
                              (fp-ai-systems) section "The problem: the n x n score
                              matrix"; "Flash Attention -- Module 12.3" section
                              "Definition"; "FlashAttention 1-2-3" section "The Math
                              Behind the Online Softmax Trick" (two-pass stable softmax).
``online_softmax_attention``  the method's own algorithm restated in numpy fp64: keys in
                              blocks, running max m and running sum l per row, the
                              partial output rescaled by exp(m_old - m_new), one division
                              by l at the end ("FlashAttention 1-2-3" sections
                              "FlashAttention-1" and "The Math Behind the Online Softmax
                              Trick"; "FlashAttention" section "Online softmax: the
                              enabling trick").  An optional threshold tau keeps a stale
                              max until the new one exceeds it by more than tau (log2
                              units); the result is the same in exact arithmetic.
``attention_backward``        dQ, dK, dV of attention() for an upstream gradient dO: the
                              gradient of the definition, written out with the whole
                              score matrix of a head in numpy fp64 ("Flash Attention --
                              Module 12.3" section "Prefill vs Decode", "Training").
``paged_decode_attention``,   attention() over a paged KV cache, over a packed batch of
``varlen_attention``,         sequences, and over FP8 (E4M3) queries and keys decoded
``fp8_qk_attention``          from the format's definition (``e4m3_to_f64``), with one
``fp8_tile_scaled_attention`` scale per tensor or one per 128-row tile.
``e4m3_encode``,              quantisation to E4M3 written from the format (round to
``e4m3_quantize_tiles``       nearest even, saturating), with per-tile scales.
``lse_combine``               merges partial results over disjoint key sets by their
                              log-sum-exp, the reduction step of split-KV decoding
                              ("FlashAttention 1-2-3" section "Beyond FlashAttention":
                              partial softmax per KV chunk, then a reduction).
``score_matrix_bytes``,       byte counts the pages print ("FlashAttention" section "The
``standard_attention_traffic`` problem"; "FlashAttention 1-2-3" section "The Memory Wall").

Parity status: every function above is pinned by ``tests/test_oracle.py`` (closed forms,
invariants, brute force, a library routine, and the pages' printed byte counts).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libattn_oracle.so")
_lib = None

F64, F16, BF16 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compiles attn_oracle.c with gcc (no fast-math) into libattn_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared", "-pthread", _SRC,
             "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def default_threads() -> int:
    """Host threads the C oracle uses by default (the CPUs this process may run on)."""
    return int(_load().attn_oracle_default_threads())


def _as_bits(x):
    """Returns (contiguous numpy array, dtype code) without changing any value."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.float16:
            return x.view(torch.int16).numpy(), F16
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy(), BF16
        return x.to(torch.float64).numpy(), F64
    a = np.ascontiguousarray(x)
    if a.dtype == np.float16:
        return a.view(np.int16), F16
    return np.ascontiguousarray(a, dtype=np.float64), F64


def load_library(path: str):
    """Opens an oracle shared library built from attn_oracle.c (or a copy of it)."""
    lib = ctypes.CDLL(path)
    lib.attn_oracle_fwd.restype = ctypes.c_int
    lib.attn_oracle_fwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
    ]
    lib.attn_oracle_default_threads.restype = ctypes.c_int
    return lib


def attention(q, k, v, scale: float, causal: bool, rows: Optional[Sequence[int]] = None,
              nthreads: int = 0, lib=None):
    """O and LSE of softmax(scale * Q K^T [+ causal mask]) V in fp64.

    q: [B,H,Nq,d], k/v: [B,H,Nkv,d] (torch fp16/bf16/any float tensor, or numpy), all
    three of one dtype.  Causal masking is aligned bottom-right (query i sees keys
    j <= i + Nkv - Nq).  rows: optional global row ids (b*H*Nq + h*Nq + i); the result
    then has one row per id.  Returns (o, lse) as numpy float64: o [B,H,Nq,d] and
    lse [B,H,Nq], or o [len(rows), d] and lse [len(rows)].  ``lib`` selects another
    build of attn_oracle.c (the mutation tests use it); default: this package's.
    """
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    assert tuple(k.shape) == (B, H, Nkv, d) and tuple(v.shape) == (B, H, Nkv, d)
    qa, dt = _as_bits(q)
    ka, dk = _as_bits(k)
    va, dv = _as_bits(v)
    assert dt == dk == dv, "q, k and v must share one dtype"
    if rows is None:
        nrows = B * H * Nq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = int(rows_arr.size)
    o = np.zeros((max(nrows, 1), d), dtype=np.float64)
    lse = np.zeros((max(nrows, 1),), dtype=np.float64)
    if nrows == 0:
        return o[:0], lse[:0]
    rc = (lib or _load()).attn_oracle_fwd(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, dt,
        o.ctypes.data, lse.ctypes.data, B, H, Nq, Nkv, d, float(scale), int(bool(causal)),
        None if rows_arr is None else rows_arr.ctypes.data, nrows, int(nthreads),
    )
    if rc != 0:
        raise RuntimeError(f"attn_oracle_fwd failed with {rc}")
    if rows is None:
        return o.reshape(B, H, Nq, d), lse.reshape(B, H, Nq)
    return o, lse


def paged_decode_attention(q, k_cache, v_cache, block_table, seq_lens, scale: float,
                           nthreads: int = 0, lib=None):
    """Decode (one query per head) against a paged KV cache, in fp64.

    q: [B,H,d]; k_cache, v_cache: [num_pages, H, page_size, d]; block_table: [B, P]
    integers; seq_lens: [B].  Logical key i of sequence b is slot i mod page_size of page
    block_table[b, i // page_size] -- the KV-cache pages of PagedAttention ("FlashAttention
    1-2-3" (myaihardware), section "Integration in Major Inference Engines": each KV cache
    page is a block the attention kernel tiles over).  The keys of each sequence are gathered in logical order and the
    result is attention() over them (no mask: the query follows every cached key).  A
    sequence with no keys gives O = 0 and LSE = -inf.  Returns (o [B,H,d], lse [B,H]).
    """
    import torch
    B, H, d = q.shape
    ps = k_cache.shape[2]
    o = np.zeros((B, H, d), dtype=np.float64)
    lse = np.full((B, H), -np.inf, dtype=np.float64)
    bt = torch.as_tensor(block_table).to(torch.int64).cpu()
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        pages = bt[b, : (L + ps - 1) // ps]
        kb = k_cache[pages].permute(1, 0, 2, 3).reshape(H, -1, d)[:, :L]
        vb = v_cache[pages].permute(1, 0, 2, 3).reshape(H, -1, d)[:, :L]
        ob, lb = attention(q[b].reshape(1, H, 1, d), kb.reshape(1, H, L, d).contiguous(),
                           vb.reshape(1, H, L, d).contiguous(), scale, False,
                           nthreads=nthreads, lib=lib)
        o[b] = ob[0, :, 0]
        lse[b] = lb[0, :, 0]
    return o, lse


def varlen_attention(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool,
                     nthreads: int = 0, lib=None):
    """Attention over a batch of sequences of different lengths, packed token-major.

    q: [total_q, H, d], k/v: [total_k, H, d]; sequence b owns query tokens
    cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key tokens cu_seqlens_k[b] ..
    cu_seqlens_k[b+1]-1, and attends only to its own keys (causal alignment per sequence,
    bottom-right as in attention()).  This is attention() applied sequence by sequence --
    the "batch of independent problems" the pages tile over ("FlashAttention 1-2-3"
    (myaihardware), section "When FlashAttention Doesn't Help": each query in the batch
    processed independently).  Query tokens of a sequence with no keys, or fully masked,
    get O = 0 and LSE = -inf.  Returns (o [total_q,H,d], lse [total_q,H]) in float64.
    """
    total_q, H, d = q.shape
    o = np.zeros((total_q, H, d), dtype=np.float64)
    lse = np.full((total_q, H), -np.inf, dtype=np.float64)
    cq = [int(x) for x in cu_seqlens_q]
    ck = [int(x) for x in cu_seqlens_k]
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue
        qb = q[q0:q1].permute(1, 0, 2).reshape(1, H, q1 - q0, d).contiguous()
        kb = k[k0:k1].permute(1, 0, 2).reshape(1, H, k1 - k0, d).contiguous()
        vb = v[k0:k1].permute(1, 0, 2).reshape(1, H, k1 - k0, d).contiguous()
        ob, lb = attention(qb, kb, vb, scale, causal, nthreads=nthreads, lib=lib)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[q0:q1] = lb[0].T
    return o, lse


def e4m3_to_f64(bits):
    """Values of FP8 E4M3 codes (uint8 array or tensor): sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN and
    there is no infinity (the "fn" variant used for FP8 tensor-core inputs).  Returns
    numpy float64."""
    try:
        import torch
        if isinstance(bits, torch.Tensor):
            bits = bits.detach().cpu().view(torch.uint8).numpy()
    except ImportError:  # pragma: no cover
        pass
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    out = sign * mag
    return np.where((e == 15) & ((b & 7) == 7), np.nan, out)


def e4m3_encode(x):
    """E4M3 ("fn") codes of float32 values: round to the nearest representable value, ties
    to the even mantissa, magnitudes beyond the largest finite value 448 saturate to +-448
    (no infinities).  Written from the format: for a normal magnitude 2^e * (1 + f) the
    representable neighbours are spaced 2^(e - 3) apart; below 2^-6 (the subnormals
    m * 2^-9) the spacing is 2^-9.  Returns a numpy uint8 array of x's shape."""
    a = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.signbit(a)
    mag = np.abs(a)
    _, e = np.frexp(mag)            # mag = f * 2^e with f in [0.5, 1): floor(log2 mag) = e - 1
    e = e.astype(np.int64) - 1
    normal = mag >= 2.0 ** -6
    spacing = np.where(normal, np.exp2(np.maximum(e, -6) - 3.0), 2.0 ** -9)
    q = np.round(mag / spacing)     # numpy rounds halves to even: ties to the even mantissa
    # normal: q in [8, 16]; q == 16 carries into the next binade
    code_n = np.where(q >= 16, ((e + 1 + 7) << 3) | 0, ((e + 7) << 3) | (q.astype(np.int64) - 8))
    code_s = q.astype(np.int64)      # subnormal: 0..8 (8 is the smallest normal, code 0x08)
    code = np.where(normal, code_n, code_s)
    code = np.where(mag >= 448.0, 0x7E, code)   # saturate (this also covers rounding past 448)
    code = np.minimum(code, 0x7E)
    return (code | (sign.astype(np.int64) << 7)).astype(np.uint8)


def e4m3_quantize_tiles(x, tile_rows: int = 128):
    """Quantises x [BH, N, d] (any float type, taken exactly as float32) to E4M3 codes
    with one scale per tile of `tile_rows` consecutive rows of one head: scale =
    float32(max |x| over the tile) / 448 in float32 arithmetic (1 when the tile is all
    zero), code = e4m3_encode(float32(x) / scale) with a float32 division.  Returns (codes
    uint8 [BH, N, d], scales float32 [BH, ceil(N / tile_rows)]): x ~ codes * scale."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().to(torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x, dtype=np.float32)
    BH, N, d = x.shape
    nt = (N + tile_rows - 1) // tile_rows
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.ones((BH, nt), dtype=np.float32)
    for t in range(nt):
        blk = x[:, t * tile_rows:(t + 1) * tile_rows]
        amax = np.abs(blk).reshape(BH, -1).max(axis=1).astype(np.float32)
        sc = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        scales[:, t] = sc
        codes[:, t * tile_rows:(t + 1) * tile_rows] = e4m3_encode(blk / sc[:, None, None])
    return codes, scales


def fp8_tile_scaled_attention(q8, q_scales, k8, k_scales, v, scale: float, causal: bool,
                              tile_rows: int = 128, rows=None, nthreads: int = 0, lib=None):
    """attention() of FP8 queries and keys with one scale per tile of `tile_rows` rows:
    q8 [B,H,Nq,d], k8 [B,H,Nkv,d] E4M3 codes; q_scales [B*H, ceil(Nq/tile_rows)] and
    k_scales [B*H, ceil(Nkv/tile_rows)]; row i of head bh stands for
    decode(q8[.., i, :]) * q_scales[bh, i // tile_rows] (likewise for keys).  fp64."""
    import torch
    q8 = np.asarray(q8.cpu().numpy() if hasattr(q8, "cpu") else q8)
    k8 = np.asarray(k8.cpu().numpy() if hasattr(k8, "cpu") else k8)
    B, H, Nq, d = q8.shape
    Nkv = k8.shape[2]
    qs = np.repeat(np.asarray(q_scales, dtype=np.float64), tile_rows, axis=1)[:, :Nq]
    ks = np.repeat(np.asarray(k_scales, dtype=np.float64), tile_rows, axis=1)[:, :Nkv]
    qf = e4m3_to_f64(q8) * qs.reshape(B, H, Nq, 1)
    kf = e4m3_to_f64(k8) * ks.reshape(B, H, Nkv, 1)
    vf = torch.as_tensor(v).detach().cpu().to(torch.float64)
    return attention(torch.from_numpy(qf), torch.from_numpy(kf), vf, scale, causal, rows=rows,
                     nthreads=nthreads, lib=lib)


def fp8_qk_attention(q8, k8, v, q_scale: float, k_scale: float, scale: float, causal: bool,
                     rows=None, nthreads: int = 0, lib=None):
    """Attention with FP8 queries and keys ("FlashAttention 1-2-3" (myaihardware), section
    "FlashAttention-3: FP8, Async Warp Overlap, and Hopper-Specific Optimizations": FP8
    tensor-core inputs).  q8 [B,H,Nq,d] and k8 [B,H,Nkv,d] hold E4M3
    codes; the tensors they stand for are q_scale * decode(q8) and k_scale * decode(k8)
    (per-tensor scales).  v [B,H,Nkv,d] in its own type.  The result is attention() of
    those values in fp64, same layout and conventions."""
    import torch
    qf = torch.from_numpy(e4m3_to_f64(q8) * float(q_scale))
    kf = torch.from_numpy(e4m3_to_f64(k8) * float(k_scale))
    vf = torch.as_tensor(v).detach().cpu().to(torch.float64)
    return attention(qf, kf, vf, scale, causal, rows=rows, nthreads=nthreads, lib=lib)


def attention_backward(q, k, v, do, scale: float, causal: bool, heads=None):
    """Gradients dQ, dK, dV of attention() for an upstream gradient dO, in fp64.

    The pages say only that training runs a backward pass that is IO-aware as the forward
    is ("Flash Attention -- Module 12.3", section "Prefill vs Decode", "Training"), and
    that the forward keeps per-row softmax statistics so that nothing N x N has to be
    stored ("FlashAttention 1-2-3" (myaihardware), section "FlashAttention-1: Tiling,
    Recomputation, and Online Softmax").  What it must compute is the gradient of the
    definition O = softmax(scale * Q K^T [+ causal mask]) V, written out here with the
    whole score matrix of one head (numpy matmuls as the only library step):

        P    = softmax of the masked, scaled scores, row by row (masked entries 0)
        dV   = P^T dO
        dP   = dO V^T
        D_i  = sum_j P_ij dP_ij            (equal to dO_i . O_i)
        dS   = P * (dP - D)                (the softmax Jacobian applied row by row)
        dQ   = scale * dS K
        dK   = scale * dS^T Q

    q, do: [B,H,Nq,d]; k, v: [B,H,Nkv,d] (torch tensors of any float type, or numpy).
    Causal masking is aligned bottom-right as in attention(); a query row that sees no key
    has P = 0 and contributes nothing.  heads: optional list of flat head ids b*H + h;
    only those heads are computed (the others stay 0).  Returns numpy float64
    (dq [B,H,Nq,d], dk [B,H,Nkv,d], dv [B,H,Nkv,d]).
    """
    qf, kf, vf, gf = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, Nq, d = qf.shape
    Nkv = kf.shape[2]
    assert kf.shape == (B, H, Nkv, d) and vf.shape == (B, H, Nkv, d) and gf.shape == qf.shape
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    if Nq == 0 or Nkv == 0:
        return dq, dk, dv
    visible = np.ones((Nq, Nkv), dtype=bool)
    if causal:
        visible = np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)
    ids = range(B * H) if heads is None else heads
    for bh in ids:
        b, h = divmod(int(bh), H)
        Q, K, V, G = qf[b, h], kf[b, h], vf[b, h], gf[b, h]
        s = np.where(visible, scale * (Q @ K.T), -np.inf)
        m = s.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.where(visible, np.exp(s - m), 0.0)
        z = e.sum(axis=1, keepdims=True)
        P = e / np.where(z > 0, z, 1.0)
        dv[b, h] = P.T @ G
        dP = G @ V.T
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        dq[b, h] = scale * (dS @ K)
        dk[b, h] = scale * (dS.T @ Q)
    return dq, dk, dv


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def online_softmax_attention(q, k, v, scale: float, causal: bool, block_sizes=(128,),
                             tau: float = 0.0):
    """The tiled online-softmax forward, restated in numpy fp64.

    Keys are visited in consecutive blocks whose sizes cycle through ``block_sizes``.
    Per query row the state is (m, l, O~): running max (in log2 units), running sum of
    2^(x - m) and the unnormalised output.  For each block with scores x (already
    multiplied by log2(e) * scale, masked entries -inf):

        m_new = max(m, max(x))
        if m_new - m > tau:   O~ *= 2^(m - m_new);  l *= 2^(m - m_new);  m = m_new
        p = 2^(x - m);  l += sum(p);  O~ += p @ V_block

    and at the end O = O~ / l and LSE = (m + log2 l) * ln 2.  tau = 0 is the eager update
    the pages describe; tau > 0 keeps the stale max (lazy rescale), exact in exact
    arithmetic because O~ and l always share the same m.  Rows that see no key give O=0,
    LSE=-inf.  Returns numpy (o [B,H,Nq,d], lse [B,H,Nq]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    log2e = 1.0 / np.log(2.0)
    o = np.zeros((B, H, Nq, d))
    lse = np.full((B, H, Nq), -np.inf)
    rows = np.arange(Nq)[:, None]
    for b in range(B):
        for h in range(H):
            m = np.full(Nq, -np.inf)
            l = np.zeros(Nq)
            acc = np.zeros((Nq, d))
            start, bi = 0, 0
            while start < Nkv:
                bs = int(block_sizes[bi % len(block_sizes)])
                bi += 1
                cols = np.arange(start, min(start + bs, Nkv))[None, :]
                x = (q[b, h] @ k[b, h, cols[0]].T) * (scale * log2e)
                if causal:
                    x = np.where(cols <= rows + (Nkv - Nq), x, -np.inf)
                m_new = np.maximum(m, x.max(axis=1))
                with np.errstate(invalid="ignore"):
                    jump = m_new - m
                    move = (jump > tau) | (np.isneginf(m) & np.isfinite(m_new))
                    alpha = np.where(move, np.exp2(np.where(move, m - m_new, 0.0)), 1.0)
                acc *= alpha[:, None]
                l *= alpha
                m = np.where(move, m_new, m)
                m_safe = np.where(np.isneginf(m), 0.0, m)
                p = np.exp2(x - m_safe[:, None])
                l += p.sum(axis=1)
                acc += p @ v[b, h, cols[0]]
                start += bs
            seen = l > 0
            o[b, h] = np.where(seen[:, None], acc / np.where(seen, l, 1.0)[:, None], 0.0)
            with np.errstate(divide="ignore"):
                lse[b, h] = np.where(seen, (m + np.log2(np.where(seen, l, 1.0))) * np.log(2.0),
                                     -np.inf)
    return o, lse


def lse_combine(o_parts, lse_parts):
    """Merges S partial results over disjoint key sets into the full result.

    o_parts: [S, ..., d], each normalised over its own keys; lse_parts: [S, ...] with
    -inf for a part that saw no key.  With M = max_s lse_s and
    L = M + ln sum_s exp(lse_s - M):  O = sum_s exp(lse_s - L) * O_s,  LSE = L.
    All parts empty gives O = 0, LSE = -inf.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    M = lse_parts.max(axis=0)
    M_safe = np.where(np.isneginf(M), 0.0, M)
    w = np.exp(lse_parts - M_safe)
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        L = np.where(tot > 0, M_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    L_safe = np.where(np.isneginf(L), 0.0, L)
    wn = np.where(np.isneginf(lse_parts), 0.0, np.exp(lse_parts - L_safe))
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, L


def score_matrix_bytes(n: int, elem_bytes: int) -> int:
    """Bytes of one head's n x n score matrix ("FlashAttention", section "The problem")."""
    return n * n * elem_bytes


def standard_attention_traffic(n: int, d: int, elem_bytes: int) -> dict:
    """Per-head HBM bytes of materialising attention, term by term, as the
    "FlashAttention 1-2-3" page estimates it in section "The Memory Wall": read Q, K, V;
    write and read S; write and read P; write O."""
    qkv = 3 * n * d * elem_bytes
    s = 2 * n * n * elem_bytes
    p = 2 * n * n * elem_bytes
    o = n * d * elem_bytes
    return {"qkv_read": qkv, "s_write_read": s, "p_write_read": p, "o_write": o,
            "total": qkv + s + p + o}

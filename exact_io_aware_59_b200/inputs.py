"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws Q, K, V.  Both the CUDA path's
tests and the CPU oracle's tests take their inputs from here.

Recipe: every element is an iid standard normal draw in fp32 from torch's generator
(CPU or CUDA), seeded per tensor, optionally multiplied by a standard deviation, then
rounded once to the workload's 16-bit type.  Workload c seeds Q, K, V with
1000*c + 0, 1, 2.  The pages give their workloads only as shapes (the FlashAttention-2
benchmark at 1x32x8192x128, the SDPA example at 2x8x2048x64, the H100 figures at
N=16384, d=128, and decode with one query against a long KV cache), so no dataset is
involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int          # seed family: Q, K, V use 1000*index + 0, 1, 2
    B: int
    H: int
    Nq: int
    Nkv: int
    d: int
    dtype: torch.dtype
    causal: bool
    q_std: float = 1.0
    scale: Optional[float] = None  # None: 1/sqrt(d)
    note: str = ""

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    def shapes(self):
        return (self.B, self.H, self.Nq, self.d), (self.B, self.H, self.Nkv, self.d)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 1, 1, 128, 128, 64, torch.float16, False),
        Workload("tiny_causal", 1, 1, 1, 128, 128, 64, torch.float16, True),
        Workload("prefill_mha", 2, 2, 8, 2048, 2048, 64, torch.float16, True),
        Workload("long_prefill_causal", 3, 1, 32, 8192, 8192, 128, torch.bfloat16, True),
        Workload("long_prefill", 3, 1, 32, 8192, 8192, 128, torch.bfloat16, False),
        Workload("long_prefill_peaky", 3, 1, 32, 8192, 8192, 128, torch.bfloat16, True,
                 q_std=4.0, note="Q drawn with std 4 to stress the running-max rescale"),
        Workload("long_ctx_16k", 4, 1, 16, 16384, 16384, 128, torch.bfloat16, True),
        Workload("long_ctx_32k", 4, 1, 16, 32768, 32768, 128, torch.bfloat16, True),
        Workload("decode", 5, 16, 32, 1, 32768, 128, torch.bfloat16, False),
        # Smaller cases of the same kernels, for profiler captures (still larger than L2).
        Workload("decode_4k", 6, 16, 32, 1, 4096, 128, torch.bfloat16, False,
                 note="profiling size: 1 GiB of K+V"),
        Workload("prefill_causal_4k", 7, 1, 32, 4096, 4096, 128, torch.bfloat16, True,
                 note="profiling size"),
    ]
}


def randn(shape, seed: int, dtype: torch.dtype, std: float = 1.0, device="cpu"):
    """iid N(0, std^2) drawn in fp32 from a generator seeded with `seed`, rounded once
    to `dtype`."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def make_qkv(B, H, Nq, Nkv, d, dtype, seed_base: int, q_std: float = 1.0, device="cpu"):
    """Q [B,H,Nq,d], K and V [B,H,Nkv,d], seeded with seed_base + 0, 1, 2."""
    q = randn((B, H, Nq, d), seed_base + 0, dtype, q_std, device)
    k = randn((B, H, Nkv, d), seed_base + 1, dtype, 1.0, device)
    v = randn((B, H, Nkv, d), seed_base + 2, dtype, 1.0, device)
    return q, k, v


def workload_qkv(w: Workload, device="cpu"):
    return make_qkv(w.B, w.H, w.Nq, w.Nkv, w.d, w.dtype, 1000 * w.index, w.q_std, device)


def paged_decode_inputs(B: int, H: int, L: int, d: int, page_size: int, dtype: torch.dtype,
                        seed_base: int, device="cpu"):
    """A paged KV cache holding B sequences of L keys each: q [B,H,d]; k_cache, v_cache
    [B*ceil(L/page_size), H, page_size, d] iid N(0,1) rounded to `dtype`; block_table
    int32 [B, P] a seeded random permutation of all pages (so a sequence's pages are
    scattered over the pool); seq_lens int32 [B] all L.  Seeds seed_base + 0..3."""
    P = (L + page_size - 1) // page_size
    q = randn((B, H, d), seed_base + 0, dtype, 1.0, device)
    k_cache = randn((B * P, H, page_size, d), seed_base + 1, dtype, 1.0, device)
    v_cache = randn((B * P, H, page_size, d), seed_base + 2, dtype, 1.0, device)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed_base + 3))
    table = torch.randperm(B * P, generator=g, device=device).to(torch.int32).reshape(B, P)
    seq_lens = torch.full((B,), L, dtype=torch.int32, device=device)
    return q, k_cache, v_cache, table.contiguous(), seq_lens


def varlen_lengths(n: int, lo: int, hi: int, seed: int):
    """n sequence lengths drawn log-uniformly from [lo, hi] with a seeded generator (a
    mix of short and long requests, as in a continuously batched prefill)."""
    g = torch.Generator()
    g.manual_seed(int(seed))
    u = torch.rand(n, generator=g, dtype=torch.float64)
    import math
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo))))) for x in u]


def varlen_inputs(lengths, H: int, d: int, dtype: torch.dtype, seed_base: int, device="cpu"):
    """A packed batch: q, k, v [sum(lengths), H, d] iid N(0,1) rounded to `dtype` (seeds
    seed_base + 0, 1, 2) and cu_seqlens int32 [len(lengths)+1]."""
    total = int(sum(lengths))
    q = randn((total, H, d), seed_base + 0, dtype, 1.0, device)
    k = randn((total, H, d), seed_base + 1, dtype, 1.0, device)
    v = randn((total, H, d), seed_base + 2, dtype, 1.0, device)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return q, k, v, torch.tensor(cu, dtype=torch.int32, device=device)


def make_grad_out(B: int, H: int, Nq: int, d: int, dtype: torch.dtype, seed: int, device="cpu"):
    """Upstream gradient dO [B,H,Nq,d] for the backward pass: iid N(0,1) rounded to
    `dtype`.  Workloads seed it with 1000*index + 3 (after Q, K, V)."""
    return randn((B, H, Nq, d), seed, dtype, 1.0, device)

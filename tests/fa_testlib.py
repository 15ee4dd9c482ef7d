"""Shared helpers for the GPU parity tests: tolerances and comparisons."""
import math

import numpy as np
import torch

# Binding tolerances for fp16/bf16 inputs with fp32 outputs.
MAX_ABS_O = 1e-2
MEAN_ABS_O = 1e-3
MAX_ABS_LSE = 1e-3
# O rounded to a 16-bit type adds up to half an ulp of |O|: 2^-8 |O| for bf16 (2^-11 for
# fp16), on top of the fp32 tolerance.
REL_O16 = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


def has_b200() -> bool:
    return torch.cuda.is_available() and torch.cuda.get_device_capability(0) == (10, 0)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, rel_o: float = 0.0):
    """Element-by-element comparison; returns (max|dO|, mean|dO|, max|dLSE|) and asserts
    the tolerances.  Rows whose reference LSE is -inf must be exactly 0 / -inf."""
    o = o_gpu.detach().float().cpu().double().numpy().reshape(o_ref.shape)
    l = lse_gpu.detach().cpu().double().numpy().reshape(lse_ref.shape)
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l), dead), "fully masked rows differ"
    assert (o[dead] == 0).all(), "fully masked rows must give O = 0"
    assert np.isfinite(o).all(), "non-finite O"
    d_o = np.abs(o - o_ref)
    tol = MAX_ABS_O + rel_o * np.abs(o_ref)
    worst = float(d_o.max()) if d_o.size else 0.0
    mean = float(d_o.mean()) if d_o.size else 0.0
    live = ~dead
    d_l = float(np.abs(l[live] - lse_ref[live]).max()) if live.any() else 0.0
    assert (d_o <= tol).all(), f"max|dO| = {worst:.3e} exceeds tolerance"
    assert mean <= MEAN_ABS_O, f"mean|dO| = {mean:.3e} > {MEAN_ABS_O}"
    assert d_l <= MAX_ABS_LSE, f"max|dLSE| = {d_l:.3e} > {MAX_ABS_LSE}"
    return worst, mean, d_l


def sample_rows(B, H, Nq, per_head=48, heads=None, seed=0):
    """Global row ids (b*H*Nq + h*Nq + i) spread over tile starts, tile ends, the tail
    and random rows, for the heads in `heads` (default: first, last and one middle)."""
    rng = np.random.default_rng(seed)
    BH = B * H
    if heads is None:
        heads = sorted({0, BH // 2, BH - 1})
    rows = []
    for bh in heads:
        fixed = [0, 1, 127, 128, 129, 255, 256, Nq // 2, Nq - 129, Nq - 128, Nq - 2, Nq - 1]
        fixed = [i for i in fixed if 0 <= i < Nq]
        rand = rng.choice(Nq, size=min(Nq, max(0, per_head - len(fixed))), replace=False)
        for i in sorted(set(fixed) | set(int(x) for x in rand)):
            rows.append(bh * Nq + i)
    return np.asarray(rows, dtype=np.int64)


def scale_for(d):
    return 1.0 / math.sqrt(d)

"""GPU parity: the CUDA path against the fp64 CPU oracle on every named workload.

Every output is compared, the full-size workloads (the launch configuration the benchmark
times) included; only N = 32768 is compared on a sample (every head's tile-boundary rows
and 256 random rows per head) that the oracle computes row by row.
Tolerances: max|dO| <= 1e-2, mean|dO| <= 1e-3, max|dLSE| <= 1e-3 (fp32 O).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import WORKLOADS, randn, workload_qkv
from fa_testlib import REL_O16, compare, has_b200, scale_for

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    binding.fa_device_status(clear=True)
    yield
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0, "a kernel wait timed out"


def _run(w, out_dtype=torch.float32):
    q, k, v = workload_qkv(w, device="cuda")
    o, lse = binding.attention(q, k, v, causal=w.causal, scale=w.softmax_scale,
                               out_dtype=out_dtype)
    torch.cuda.synchronize()
    return q, k, v, o, lse


@pytest.mark.parametrize("name", ["tiny", "tiny_causal", "prefill_mha"])
def test_full_compare(name):
    w = WORKLOADS[name]
    q, k, v, o, lse = _run(w)
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, w.causal)
    compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("name", ["tiny", "prefill_mha"])
def test_full_compare_16bit_out(name):
    w = WORKLOADS[name]
    q, k, v, o, lse = _run(w, out_dtype=w.dtype)
    assert o.dtype == w.dtype
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, w.causal)
    compare(o, lse, o_ref, l_ref, rel_o=REL_O16[w.dtype])


_ORACLE_CACHE = {}


def _oracle_full(w, q, k, v):
    """The oracle's O and LSE for every row of workload w (cached: the fp32-O and the
    16-bit-O tests of one workload share the inputs)."""
    if w.name not in _ORACLE_CACHE:
        _ORACLE_CACHE.clear()
        _ORACLE_CACHE[w.name] = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale,
                                                 w.causal)
    return _ORACLE_CACHE[w.name]


def boundary_and_random_rows(B, H, Nq, n_random, seed):
    """Global row ids (b*H*Nq + h*Nq + i) of EVERY head: the first and last two rows of each
    128-row tile, the sequence's last rows, and n_random random rows per head."""
    rng = np.random.default_rng(seed)
    t = np.arange(0, Nq, 128)
    fixed = np.unique(np.concatenate([t, t + 1, t + 126, t + 127, [Nq - 2, Nq - 1]]))
    fixed = fixed[(fixed >= 0) & (fixed < Nq)]
    rows = []
    for bh in range(B * H):
        rand = rng.choice(Nq, size=min(Nq, n_random), replace=False)
        rows.append(bh * Nq + np.unique(np.concatenate([fixed, rand])))
    return np.concatenate(rows).astype(np.int64)


@pytest.mark.parametrize("name", ["long_prefill_causal", "long_prefill", "long_prefill_peaky",
                                  "long_ctx_16k"])
def test_full_size_every_row(name):
    """The benchmark's workloads at full size, every output compared with the oracle."""
    w = WORKLOADS[name]
    q, k, v, o, lse = _run(w)
    o_ref, l_ref = _oracle_full(w, q, k, v)
    compare(o, lse, o_ref, l_ref)
    assert (o.abs().amax() <= v.abs().amax().float() + 1e-3).item(), "O outside the hull of V"


@pytest.mark.parametrize("name", ["long_prefill_causal", "long_prefill_peaky"])
def test_full_size_every_row_16bit_out(name):
    """The benchmark's launch configuration (16-bit O), every output compared."""
    w = WORKLOADS[name]
    q, k, v, o, lse = _run(w, out_dtype=w.dtype)
    o_ref, l_ref = _oracle_full(w, q, k, v)
    compare(o, lse, o_ref, l_ref, rel_o=REL_O16[w.dtype])


def test_full_size_32k_sampled():
    """N = 32768: every head's tile-boundary rows and 256 random rows per head (the oracle
    would need minutes for all of them); properties that hold at any size on every output."""
    w = WORKLOADS["long_ctx_32k"]
    q, k, v, o, lse = _run(w)
    rows = boundary_and_random_rows(w.B, w.H, w.Nq, 256, seed=w.index)
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, w.causal,
                                    rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, w.d)[idx], lse.reshape(-1)[idx], o_ref, l_ref)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert (o.abs().amax() <= v.abs().amax().float() + 1e-3).item(), "O outside the hull of V"


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_full_size_every_head(out_dtype):
    """The decode workload (B=16, H=32, Nkv=32768): all 512 heads against the oracle."""
    w = WORKLOADS["decode"]
    q, k, v, o, lse = _run(w, out_dtype=out_dtype)
    key = ("decode", w.name)
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE.clear()
        _ORACLE_CACHE[key] = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, False)
    o_ref, l_ref = _ORACLE_CACHE[key]
    rel = REL_O16[w.dtype] if out_dtype != torch.float32 else 0.0
    compare(o, lse, o_ref, l_ref, rel_o=rel)


def test_decode_small_full_compare():
    """Decode on a size the oracle finishes in full: several heads, a ragged key tail."""
    from exact_io_aware_59_b200.inputs import make_qkv

    q, k, v = make_qkv(3, 5, 1, 1000, 128, torch.bfloat16, 777)
    o, lse = binding.attention(q.cuda(), k.cuda(), v.cuda(), scale=0.09)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q, k, v, 0.09, False)
    compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("growth", [12.0, 20.0, 26.0, 40.0, -20.0])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_running_max_growing_along_keys(growth, causal, d, dtype):
    """Scores that rise (or fall) by `growth` log2 units per 128-key tile, plus noise.
    The kernel hands each tile's P out in two halves of 64 keys, the first as soon as it is
    known not to move the reference max.  Rising by 20 or 26 per tile, the first half
    stays within the lazy threshold (15) of the previous tile's max and goes out, and the
    second half moves it: O is rescaled after the first half's product and the second half
    is redone.  Rising by 40, the first half already moves it (the whole tile is redone in
    two passes, O rescaled before any of it goes out).  Rising by 12, the reference max
    lags the true one without moving for a tile, so p reaches ~2^12 (close to the fp16
    limit for the lag); falling leaves the first tile's max in charge."""
    B, H, N = 1, 2, 1000
    scale = scale_for(d)
    g = growth / (128 * scale * math.log2(math.e))
    q = randn((B, H, N, d), 71, torch.float32, 0.3)
    k = randn((B, H, N, d), 72, torch.float32, 0.3)
    v = randn((B, H, N, d), 73, dtype)
    q[..., 0] = 1.0
    k[..., 0] = g * torch.arange(N, dtype=torch.float32)
    q, k = q.to(dtype), k.to(dtype)
    o, lse = binding.attention(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q, k, v, scale, causal)
    compare(o, lse, o_ref, l_ref)

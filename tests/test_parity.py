"""GPU parity: the CUDA path against the fp64 CPU oracle on every named workload.

Small workloads are compared on every output; the full-size ones (the same launch
configuration the benchmark times) on sampled rows that the oracle computes one by one.
Tolerances: max|dO| <= 1e-2, mean|dO| <= 1e-3, max|dLSE| <= 1e-3 (fp32 O).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import WORKLOADS, randn, workload_qkv
from fa_testlib import REL_O16, compare, has_b200, sample_rows, scale_for

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


@pytest.mark.parametrize("name", ["long_prefill_causal", "long_prefill", "long_prefill_peaky",
                                  "long_ctx_16k", "long_ctx_32k"])
def test_full_size_sampled(name):
    w = WORKLOADS[name]
    q, k, v, o, lse = _run(w)
    rows = sample_rows(w.B, w.H, w.Nq, per_head=40, seed=w.index)
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, w.causal,
                                    rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, w.d)[idx], lse.reshape(-1)[idx], o_ref, l_ref)
    # properties that hold at any size, on every output
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert (o.abs().amax() <= v.abs().amax().float() + 1e-3).item(), "O outside the hull of V"


@pytest.mark.parametrize("name", ["long_prefill_causal", "long_prefill_peaky"])
def test_full_size_sampled_16bit_out(name):
    """The benchmark's launch configuration: 16-bit O."""
    w = WORKLOADS[name]
    q, k, v, o, lse = _run(w, out_dtype=w.dtype)
    rows = sample_rows(w.B, w.H, w.Nq, per_head=40, seed=w.index + 50)
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, w.causal,
                                    rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, w.d)[idx], lse.reshape(-1)[idx], o_ref, l_ref, rel_o=REL_O16[w.dtype])


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_full_size_sampled_heads(out_dtype):
    w = WORKLOADS["decode"]
    q, k, v, o, lse = _run(w, out_dtype=out_dtype)
    BH = w.B * w.H
    heads = np.unique(np.concatenate([[0, 1, BH // 2, BH - 1],
                                      np.random.default_rng(5).choice(BH, 20, replace=False)]))
    sel = torch.from_numpy(heads).cuda()
    qs = q.reshape(BH, 1, w.Nq, w.d)[sel].reshape(1, -1, w.Nq, w.d).cpu()
    ks = k.reshape(BH, 1, w.Nkv, w.d)[sel].reshape(1, -1, w.Nkv, w.d).cpu()
    vs = v.reshape(BH, 1, w.Nkv, w.d)[sel].reshape(1, -1, w.Nkv, w.d).cpu()
    o_ref, l_ref = oracle.attention(qs, ks, vs, w.softmax_scale, False)
    rel = REL_O16[w.dtype] if out_dtype != torch.float32 else 0.0
    compare(o.reshape(BH, w.d)[sel], lse.reshape(BH)[sel], o_ref.reshape(-1, w.d),
            l_ref.reshape(-1), rel_o=rel)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_decode_small_full_compare():
    """Decode on a size the oracle finishes in full: several heads, a ragged key tail."""
    from exact_io_aware_59_b200.inputs import make_qkv

    q, k, v = make_qkv(3, 5, 1, 1000, 128, torch.bfloat16, 777)
    o, lse = binding.attention(q.cuda(), k.cuda(), v.cuda(), scale=0.09)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q, k, v, 0.09, False)
    compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("growth", [12.0, 20.0, -20.0])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_running_max_growing_along_keys(growth, causal, d, dtype):
    """Scores that rise (or fall) by `growth` log2 units per 128-key tile, plus noise.
    Rising by 20 moves every row's reference max on every tile (rescale of O, and the
    early exponentiation against the old max is redone); rising by 12 makes the reference
    max lag the true one without moving it, so p reaches ~2^12 (close to the fp16 limit
    for the lag); falling leaves the first tile's max in charge."""
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

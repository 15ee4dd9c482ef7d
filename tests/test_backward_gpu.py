"""GPU parity of the attention backward (fa_bwd) against the fp64 oracle
(oracle.attention_backward, pinned on the CPU against autograd, finite differences,
column sums and closed forms).

The forward outputs O and LSE fed to fa_bwd come from fa_fwd (16-bit O, as a training
step stores it); the oracle recomputes everything from Q, K, V and dO in fp64.

Tolerance, from the arithmetic: P and dS enter the tensor-core products rounded to the
inputs' 16-bit type, O is stored in it, and dQ, dK, dV are rounded to it at the end, so
every output element carries a few 16-bit roundings of terms no larger than the largest
output of its tensor (bf16 unit roundoff u = 2^-8, fp16 2^-11).  Errors are measured
relative to the largest |reference| of each tensor: max |err| <= 4u and mean |err| <= u/4.
(Measured on a B200: max |err| 1.0u for bf16 and 1.3u for fp16, mean at most 0.09u.)
The measured errors are printed (pytest -s) for the record.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_grad_out, make_qkv
from fa_testlib import has_b200

pytestmark = pytest.mark.gpu

U16 = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


@pytest.fixture(autouse=True)
def _device_clean():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    binding.fa_device_status(clear=True)
    yield
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0, "a kernel wait timed out"


def _run(q, k, v, g, causal, scale):
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, g))
    o, lse = binding.attention(qc, kc, vc, causal=causal, scale=scale, out_dtype=q.dtype)
    dq, dk, dv = binding.attention_backward(qc, kc, vc, o, lse, gc, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check(ours, refs, dtype, heads=None, what=""):
    u = U16[dtype]
    for name, x, r in zip(("dq", "dk", "dv"), ours, refs):
        x = x.to(torch.float64).numpy()
        if heads is not None:
            B, H = x.shape[:2]
            x = x.reshape(B * H, *x.shape[2:])[heads]
            r = r.reshape(B * H, *r.shape[2:])[heads]
        assert np.all(np.isfinite(x)), f"{what} {name}: non-finite"
        err = np.abs(x - r)
        print(f"[bwd] {what} {name}: max|err|/max|ref| {err.max() / max(np.abs(r).max(), 1e-30):.2e} "
              f"mean|err|/max|ref| {err.mean() / max(np.abs(r).max(), 1e-30):.2e}")
        # An exactly-zero reference (one key: dS = 0) is measured on an absolute 1e-3
        # scale: D (an fp32 sum over d) and dP (a tensor-core sum) round differently, which
        # leaves |dS| near 1e-7 instead of 0.
        scale = max(np.abs(r).max(), 1e-3)
        assert err.max() <= 4 * u * scale, f"{what} {name}: max err {err.max():.3e} vs max|ref| {scale:.3e}"
        assert err.mean() <= u / 4 * scale, f"{what} {name}: mean err {err.mean():.3e} vs max|ref| {scale:.3e}"


CASES = [
    # B, H, Nq, Nkv, causal, dtype
    (1, 2, 256, 256, False, torch.bfloat16),
    (1, 2, 256, 256, True, torch.bfloat16),
    (2, 3, 200, 200, True, torch.bfloat16),     # ragged last query and key tiles
    (1, 2, 130, 300, True, torch.bfloat16),     # Nq < Nkv: bottom-right diagonal
    (1, 2, 130, 300, False, torch.float16),
    (1, 2, 300, 130, True, torch.bfloat16),     # Nq > Nkv: the first rows see no key
    (1, 1, 1, 1, False, torch.bfloat16),        # one query, one key
    (1, 1, 64, 1000, False, torch.float16),     # one query tile, many key tiles
    (1, 2, 192, 320, True, torch.float16),      # fp16 with the bottom-right diagonal
]


@pytest.mark.parametrize("B,H,Nq,Nkv,causal,dtype", CASES)
def test_backward_matches_oracle(B, H, Nq, Nkv, causal, dtype):
    q, k, v = make_qkv(B, H, Nq, Nkv, 128, dtype, 3100 + Nq + Nkv)
    g = make_grad_out(B, H, Nq, 128, dtype, 3103 + Nq + Nkv)
    scale = 128 ** -0.5
    ours = _run(q, k, v, g, causal, scale)
    refs = oracle.attention_backward(q, k, v, g, scale, causal)
    _check(ours, refs, dtype, what=f"{B}x{H}x{Nq}x{Nkv} causal={causal}")


def test_backward_peaky_scores():
    """Q with std 4: sharper softmax rows, larger dS."""
    B, H, N = 1, 2, 384
    q, k, v = make_qkv(B, H, N, N, 128, torch.bfloat16, 3300, q_std=4.0)
    g = make_grad_out(B, H, N, 128, torch.bfloat16, 3303)
    ours = _run(q, k, v, g, True, 128 ** -0.5)
    refs = oracle.attention_backward(q, k, v, g, 128 ** -0.5, True)
    _check(ours, refs, torch.bfloat16, what="peaky")


def test_backward_full_size_sampled_heads():
    """The long causal prefill shape (1 x 32 x 8192 x 128, bf16), in the launch
    configuration the benchmark times; the oracle checks heads 0 and 31 in full."""
    B, H, N = 1, 32, 8192
    q, k, v = make_qkv(B, H, N, N, 128, torch.bfloat16, 3000)
    g = make_grad_out(B, H, N, 128, torch.bfloat16, 3003)
    ours = _run(q, k, v, g, True, 128 ** -0.5)
    heads = [0, 31]
    refs = oracle.attention_backward(q, k, v, g, 128 ** -0.5, True, heads=heads)
    _check(ours, refs, torch.bfloat16, heads=heads, what="full size")


def test_backward_zero_upstream_gradient_is_exactly_zero():
    B, H, N = 1, 2, 200
    q, k, v = make_qkv(B, H, N, N, 128, torch.bfloat16, 3400)
    g = torch.zeros(B, H, N, 128, dtype=torch.bfloat16)
    for t in _run(q, k, v, g, True, 128 ** -0.5):
        assert torch.count_nonzero(t) == 0


def test_backward_uniform_attention_closed_form():
    """K = 0: every score is 0 and P = 1/Nkv exactly (Nkv a power of two), so dQ is exactly
    0 and dV_j = sum_i dO_i / Nkv for every key j (one fp32 sum, rounded once)."""
    B, H, Nq, Nkv = 1, 2, 192, 256
    q, _, v = make_qkv(B, H, Nq, Nkv, 128, torch.bfloat16, 3500)
    k = torch.zeros(B, H, Nkv, 128, dtype=torch.bfloat16)
    g = make_grad_out(B, H, Nq, 128, torch.bfloat16, 3503)
    dq, dk, dv = _run(q, k, v, g, False, 128 ** -0.5)
    assert torch.count_nonzero(dq) == 0
    ref = (g.to(torch.float64).sum(dim=2, keepdim=True) / Nkv).expand(B, H, Nkv, 128)
    err = (dv.to(torch.float64) - ref).abs().max().item()
    assert err <= 2.0 ** -8 * ref.abs().max().item() * 2


def test_backward_dk_dv_deterministic():
    """dK and dV are sums kept in one CTA's TMEM: two runs give identical bits.  (dQ is
    summed across CTAs at L2 in arrival order and may differ in the last bits.)"""
    B, H, N = 1, 4, 640
    q, k, v = make_qkv(B, H, N, N, 128, torch.bfloat16, 3600)
    g = make_grad_out(B, H, N, 128, torch.bfloat16, 3603)
    a = _run(q, k, v, g, True, 128 ** -0.5)
    b = _run(q, k, v, g, True, 128 ** -0.5)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 2.0 ** -7 * a[0].float().abs().max().item()


def test_backward_workspace_reuse_and_size():
    """A caller-owned workspace of exactly fa_bwd_workspace_bytes, used twice."""
    B, H, Nq, Nkv = 1, 2, 100, 260
    q, k, v = make_qkv(B, H, Nq, Nkv, 128, torch.bfloat16, 3700)
    g = make_grad_out(B, H, Nq, 128, torch.bfloat16, 3703)
    nbytes = binding.fa_bwd_workspace_bytes(B, H, Nq, 128)
    assert nbytes == B * H * 128 * (4 + 4 + 512)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, g))
    o, lse = binding.attention(qc, kc, vc, causal=True, out_dtype=torch.bfloat16)
    r1 = binding.attention_backward(qc, kc, vc, o, lse, gc, causal=True, workspace=ws)
    r2 = binding.attention_backward(qc, kc, vc, o, lse, gc, causal=True, workspace=ws)
    torch.cuda.synchronize()
    refs = oracle.attention_backward(q, k, v, g, 128 ** -0.5, True)
    _check([t.cpu() for t in r2], refs, torch.bfloat16, what="reuse")
    assert torch.equal(r1[1], r2[1]) and torch.equal(r1[2], r2[2])


CASES_D64 = [
    # B, H, Nq, Nkv, causal, dtype
    (1, 2, 256, 256, False, torch.float16),
    (2, 3, 200, 200, True, torch.float16),      # ragged last query and key tiles
    (1, 2, 130, 300, True, torch.bfloat16),     # Nq < Nkv: bottom-right diagonal
    (1, 2, 300, 130, True, torch.float16),      # Nq > Nkv: the first rows see no key
]


@pytest.mark.parametrize("B,H,Nq,Nkv,causal,dtype", CASES_D64)
def test_backward_d64_matches_oracle(B, H, Nq, Nkv, causal, dtype):
    """d = 64: K^T for the dQ product is padded to 128 rows with a zero block."""
    q, k, v = make_qkv(B, H, Nq, Nkv, 64, dtype, 3800 + Nq + Nkv)
    g = make_grad_out(B, H, Nq, 64, dtype, 3803 + Nq + Nkv)
    scale = 64 ** -0.5
    ours = _run(q, k, v, g, causal, scale)
    refs = oracle.attention_backward(q, k, v, g, scale, causal)
    _check(ours, refs, dtype, what=f"d64 {B}x{H}x{Nq}x{Nkv} causal={causal}")


def test_backward_prefill_mha_every_head():
    """The prefill MHA workload (B=2, H=8, N=2048, d=64, fp16, causal), every head."""
    from exact_io_aware_59_b200.inputs import WORKLOADS, workload_qkv
    w = WORKLOADS["prefill_mha"]
    q, k, v = workload_qkv(w)
    g = make_grad_out(w.B, w.H, w.Nq, w.d, w.dtype, 1000 * w.index + 3)
    ours = _run(q, k, v, g, True, w.softmax_scale)
    refs = oracle.attention_backward(q, k, v, g, w.softmax_scale, True)
    _check(ours, refs, w.dtype, what="prefill_mha")

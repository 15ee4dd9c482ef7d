"""GPU parity of the packed variable-length backward (fa_bwd_varlen) against the fp64
oracle applied sequence by sequence (oracle.attention_backward on each sequence's tokens,
the oracle that test_backward_gpu.py checks fa_bwd against; each sequence of a packed batch
is an independent problem, as oracle.varlen_attention treats the forward).

The forward outputs O and LSE come from fa_fwd_varlen in the inputs' 16-bit type, as a
training step stores them.  Tolerance as for fa_bwd (relative to the largest |reference|
of each gradient of each sequence): max |err| <= 4u and mean |err| <= u/4, u the 16-bit
unit roundoff."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import randn
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


def _batch(lq, lk, H, d, dtype, seed):
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    q = randn((int(cq[-1]), H, d), seed, dtype)
    k = randn((int(ck[-1]), H, d), seed + 1, dtype)
    v = randn((int(ck[-1]), H, d), seed + 2, dtype)
    g = randn((int(cq[-1]), H, d), seed + 3, dtype)
    return q, k, v, g, cq, ck


def _run(q, k, v, g, cq, ck, lq, lk, causal, scale):
    qc, kc, vc, gc, cqc, ckc = (t.cuda() for t in (q, k, v, g, cq, ck))
    o, lse = binding.varlen_attention(qc, kc, vc, cqc, ckc, max(lq), max(lk), causal=causal,
                                      scale=scale, out_dtype=q.dtype)
    dq, dk, dv = binding.varlen_attention_backward(qc, kc, vc, o, lse, gc, cqc, ckc, max(lq),
                                                   max(lk), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check_sequences(ours, q, k, v, g, cq, ck, causal, scale, dtype):
    """Each sequence against the oracle's backward on its own tokens ([1, H, L, d])."""
    u = U16[dtype]
    dq, dk, dv = ours
    heads_first = lambda t: t.permute(1, 0, 2).unsqueeze(0)  # noqa: E731  [L,H,d] -> [1,H,L,d]
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 == q0 and k1 == k0:
            continue
        if k1 == k0:  # no keys: no gradient reaches the queries
            assert torch.count_nonzero(dq[q0:q1]) == 0
            continue
        if q1 == q0:  # no queries: the keys get no gradient
            assert torch.count_nonzero(dk[k0:k1]) == 0 and torch.count_nonzero(dv[k0:k1]) == 0
            continue
        refs = oracle.attention_backward(heads_first(q[q0:q1]), heads_first(k[k0:k1]),
                                         heads_first(v[k0:k1]), heads_first(g[q0:q1]), scale,
                                         causal)
        for name, x, r in zip(("dq", "dk", "dv"), (dq[q0:q1], dk[k0:k1], dv[k0:k1]), refs):
            x = heads_first(x).to(torch.float64).numpy()
            assert np.all(np.isfinite(x)), f"sequence {b} {name}: non-finite"
            err = np.abs(x - r)
            ref_scale = max(np.abs(r).max(), 1e-3)
            assert err.max() <= 4 * u * ref_scale, f"sequence {b} {name}: max err {err.max():.3e}"
            assert err.mean() <= u / 4 * ref_scale, f"sequence {b} {name}: mean err {err.mean():.3e}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float16)])
def test_varlen_backward_matches_oracle(causal, d, dtype):
    lq = [1, 127, 128, 129, 300, 0, 257, 64]
    lk = [1, 127, 128, 129, 300, 5, 257, 64]
    q, k, v, g, cq, ck = _batch(lq, lk, 3, d, dtype, 2100 + d)
    ours = _run(q, k, v, g, cq, ck, lq, lk, causal, d ** -0.5)
    _check_sequences(ours, q, k, v, g, cq, ck, causal, d ** -0.5, dtype)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_backward_queries_and_keys_differ(causal):
    """Fewer queries than keys (bottom-right causal alignment per sequence), more queries
    than keys (the first rows see no key), a sequence with keys but no queries and one with
    queries but no keys."""
    lq = [100, 7, 250, 0, 3, 40]
    lk = [1000, 0, 130, 90, 900, 20]
    q, k, v, g, cq, ck = _batch(lq, lk, 2, 128, torch.bfloat16, 2300)
    ours = _run(q, k, v, g, cq, ck, lq, lk, causal, 0.09)
    _check_sequences(ours, q, k, v, g, cq, ck, causal, 0.09, torch.bfloat16)


def test_varlen_backward_equal_lengths_is_the_batched_backward():
    """Equal lengths: the same tiles, products and reductions as fa_bwd on the [B,H,N,d]
    layout; dK and dV are summed in a fixed order, so they must agree bit for bit (dQ is
    summed in arrival order, so only within rounding).  The batched forward runs with
    Q-tile pairs (a one-CTA grid), as the packed forward does, so O and LSE agree too."""
    B, H, L, d = 3, 4, 700, 128
    q, k, v, g, cq, ck = _batch([L] * B, [L] * B, H, d, torch.bfloat16, 2500)
    ours = _run(q, k, v, g, cq, ck, [L] * B, [L] * B, True, 0.1)
    to_b = lambda t: t.reshape(B, L, H, d).permute(0, 2, 1, 3).contiguous().cuda()  # noqa: E731
    qb, kb, vb, gb = (to_b(t) for t in (q, k, v, g))
    o, lse = binding.attention(qb, kb, vb, causal=True, scale=0.1, out_dtype=torch.bfloat16,
                               num_ctas=1, num_splits=1)
    dqb, dkb, dvb = binding.attention_backward(qb, kb, vb, o, lse, gb, causal=True, scale=0.1)
    torch.cuda.synchronize()
    back = lambda t: t.permute(0, 2, 1, 3).reshape(B * L, H, d).cpu()  # noqa: E731
    assert torch.equal(ours[1], back(dkb)) and torch.equal(ours[2], back(dvb))
    diff = (ours[0].float() - back(dqb).float()).abs().max().item()
    assert diff <= 4 * U16[torch.bfloat16] * back(dqb).float().abs().max().item()


def test_varlen_backward_long_ragged_sampled_sequences():
    """A ragged batch up to 3000 tokens per sequence (d = 128, bf16, causal): the two
    longest sequences and the shortest against the oracle."""
    lq = [3000, 1, 2049, 700, 130]
    q, k, v, g, cq, ck = _batch(lq, lq, 2, 128, torch.bfloat16, 2700)
    dq, dk, dv = _run(q, k, v, g, cq, ck, lq, lq, True, 128 ** -0.5)
    keep = [0, 2, 1]
    sub = lambda t, c: torch.cat([t[int(c[b]):int(c[b + 1])] for b in keep])  # noqa: E731
    cs = torch.tensor(np.concatenate([[0], np.cumsum([lq[b] for b in keep])]), dtype=torch.int32)
    _check_sequences((sub(dq, cq), sub(dk, ck), sub(dv, ck)), sub(q, cq), sub(k, ck), sub(v, ck),
                     sub(g, cq), cs, cs, True, 128 ** -0.5, torch.bfloat16)


def test_varlen_backward_bad_offsets_are_flagged():
    """Offsets past total or longer than max_seqlen are clamped by the plan kernel's
    checks and reported in the status word; nothing faults."""
    lq = [50, 60]
    q, k, v, g, cq, ck = _batch(lq, lq, 2, 64, torch.float16, 2900)
    qc, kc, vc, gc = (t.cuda() for t in (q, k, v, g))
    o, lse = binding.varlen_attention(qc, kc, vc, cq.cuda(), ck.cuda(), 60, 60, causal=True,
                                      scale=0.1, out_dtype=torch.float16)
    torch.cuda.synchronize()
    binding.fa_device_status(clear=True)
    bad = cq.clone()
    bad[1] = 90  # sequence 0 claims 90 tokens with max_seqlen 60
    binding.varlen_attention_backward(qc, kc, vc, o, lse, gc, bad.cuda(), ck.cuda(), 60, 60,
                                      causal=True, scale=0.1)
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) & binding.FA_DEV_BAD_INPUT

"""GPU parity of the packed variable-length prefill (fa_fwd_varlen) against the fp64
oracle (oracle.varlen_attention: attention() sequence by sequence, pinned on the CPU)."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_qkv, randn
from fa_testlib import REL_O16, compare, has_b200

pytestmark = pytest.mark.gpu


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
    return q, k, v, cq, ck


def _run(q, k, v, cq, ck, lq, lk, causal, scale, **kw):
    o, lse = binding.varlen_attention(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(),
                                      max(lq), max(lk), causal=causal, scale=scale, **kw)
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_varlen_matches_oracle(causal, d, dtype):
    lq = [1, 127, 128, 129, 300, 0, 257, 64]
    lk = [1, 127, 128, 129, 300, 5, 257, 64]
    H = 3
    q, k, v, cq, ck = _batch(lq, lk, H, d, dtype, 900 + d)
    o, lse = _run(q, k, v, cq, ck, lq, lk, causal, d ** -0.5)
    o_ref, l_ref = oracle.varlen_attention(q, k, v, cq.tolist(), ck.tolist(), d ** -0.5, causal)
    compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_queries_and_keys_differ(causal):
    """Chunked-prefill shapes: fewer queries than keys (and a sequence with no keys at
    all, whose queries get O = 0, LSE = -inf), causal alignment bottom-right per sequence."""
    lq = [100, 7, 250, 3]
    lk = [1000, 0, 260, 900]
    q, k, v, cq, ck = _batch(lq, lk, 2, 128, torch.bfloat16, 950)
    o, lse = _run(q, k, v, cq, ck, lq, lk, causal, 0.09, out_dtype=torch.bfloat16)
    o_ref, l_ref = oracle.varlen_attention(q, k, v, cq.tolist(), ck.tolist(), 0.09, causal)
    compare(o, lse, o_ref, l_ref, rel_o=REL_O16[torch.bfloat16])


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equal_lengths_is_the_batched_kernel(causal):
    """Equal lengths: the same tiles in the same order as the unsplit prefill on the
    [B,H,N,d] layout with Q-tile pairs (a grid smaller than the pair count), so the packed
    call must give the batched call's result bit for bit."""
    B, H, L, d = 3, 4, 700, 128
    q, k, v = make_qkv(B, H, L, L, d, torch.bfloat16, 960, device="cuda")
    o_b, l_b = binding.attention(q, k, v, causal=causal, scale=0.1, num_ctas=1, num_splits=1)
    pack = lambda x: x.permute(0, 2, 1, 3).reshape(B * L, H, d).contiguous()
    cu = torch.arange(0, (B + 1) * L, L, dtype=torch.int32, device="cuda")
    o_v, l_v = binding.varlen_attention(pack(q), pack(k), pack(v), cu, cu, L, L, causal=causal,
                                        scale=0.1)
    torch.cuda.synchronize()
    assert torch.equal(o_v, pack(o_b)) and torch.equal(l_v, l_b.permute(0, 2, 1).reshape(B * L, H))


def test_varlen_long_ragged_sampled():
    """A ragged batch up to 6000 tokens per sequence (d=128, bf16, causal), checked on
    sampled query tokens of every sequence."""
    lq = [6000, 1, 4096, 2500, 130, 3333]
    q, k, v, cq, ck = _batch(lq, lq, 4, 128, torch.bfloat16, 970)
    o, lse = _run(q, k, v, cq, ck, lq, lq, True, 128 ** -0.5)
    rng = np.random.default_rng(1)
    for b in range(len(lq)):
        n = lq[b]
        picks = sorted(set([0, n - 1, min(n - 1, 127), min(n - 1, 128)]) |
                       set(rng.integers(0, n, size=min(n, 12)).tolist()))
        # a one-sequence packed batch per sampled token range keeps the oracle small
        for t in picks:
            L = t + 1  # causal: the token sees keys 0..t of its sequence
            qs = q[int(cq[b]) + t: int(cq[b]) + t + 1]
            ks = k[int(ck[b]): int(ck[b]) + L]
            vs = v[int(ck[b]): int(ck[b]) + L]
            o_ref, l_ref = oracle.varlen_attention(qs, ks, vs, [0, 1], [0, L], 128 ** -0.5, False)
            compare(o[int(cq[b]) + t], lse[int(cq[b]) + t], o_ref[0], l_ref[0])


def test_varlen_bad_offsets_are_flagged():
    """Offsets that run past total or exceed max_seqlen are clamped by the kernel's own
    checks and reported in the status word; nothing faults."""
    lq = [50, 60]
    q, k, v, cq, ck = _batch(lq, lq, 2, 64, torch.float16, 990)
    cq_bad = cq.clone()
    cq_bad[1] = 90            # sequence 0 claims 90 tokens with max_seqlen 60
    o, lse = binding.varlen_attention(q.cuda(), k.cuda(), v.cuda(), cq_bad.cuda(), ck.cuda(),
                                      60, 60, causal=True, scale=0.1)
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) & binding.FA_DEV_BAD_INPUT


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_many_ragged_sequences(causal):
    """Forty sequences of 0 to 700 tokens (queries and keys of different lengths): the
    plan kernel's work list (bounds-checked ranges, items heaviest first) covers every query
    row exactly once; every output compared with the oracle."""
    rng = np.random.default_rng(2024 + causal)
    lq = rng.integers(0, 700, size=40).tolist()
    lk = [max(0, n + int(x)) for n, x in zip(lq, rng.integers(-50, 200, size=40))]
    lq[3], lk[3] = 0, 0
    lq[7], lk[7] = 1, 1
    q, k, v, cq, ck = _batch(lq, lk, 2, 64, torch.float16, 1200)
    o, lse = _run(q, k, v, cq, ck, lq, lk, causal, 0.125)
    o_ref, l_ref = oracle.varlen_attention(q, k, v, cq.tolist(), ck.tolist(), 0.125, causal)
    compare(o, lse, o_ref, l_ref)


def test_varlen_claimed_units_repeat_bitwise():
    """A packed batch's units are claimed from a work counter, so which CTA runs which unit
    changes from call to call; a unit's rows depend on its inputs alone, so repeated calls
    must agree bit for bit (here about 600 units for 148 CTAs)."""
    rng = np.random.default_rng(77)
    lq = rng.integers(1, 1500, size=24).tolist()
    q, k, v, cq, ck = _batch(lq, lq, 8, 128, torch.bfloat16, 1300)
    outs = [_run(q, k, v, cq, ck, lq, lq, True, 0.088) for _ in range(3)]
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])
    rows = np.concatenate([np.arange(int(cq[b]), int(cq[b]) + n)[:: max(1, n // 6)]
                           for b, n in enumerate(lq)])
    o_ref, l_ref = oracle.varlen_attention(q, k, v, cq.tolist(), ck.tolist(), 0.088, True)
    compare(outs[0][0][rows], outs[0][1][rows], o_ref[rows], l_ref[rows])


def test_varlen_benchmark_batch_sampled():
    """The benchmark's packed batch in the benchmark's launch configuration: 16 sequences
    of seeded log-uniform lengths in [512, 8192], H = 32, d = 128, bf16 in and out,
    causal, the inputs bench.py times.  Checked against the oracle on the first and last
    query token of every sequence, the tokens on both sides of its first Q-tile boundary
    and 16 random tokens."""
    from exact_io_aware_59_b200.inputs import varlen_inputs, varlen_lengths

    lens = varlen_lengths(16, 512, 8192, 4242)
    H, d, scale = 32, 128, 128 ** -0.5
    q, k, v, cu = varlen_inputs(lens, H, d, torch.bfloat16, 8000, device="cuda")
    o, lse = _run(q, k, v, cu, cu, lens, lens, True, scale, out_dtype=torch.bfloat16)
    rng = np.random.default_rng(4242)
    for b, n in enumerate(lens):
        c0 = int(cu[b])
        picks = sorted({0, n - 1, 127, 128} | set(rng.integers(0, n, size=16).tolist()))
        for t in picks:
            L = t + 1  # causal: token t sees keys 0..t of its sequence
            o_ref, l_ref = oracle.varlen_attention(
                q[c0 + t: c0 + t + 1].cpu(), k[c0: c0 + L].cpu(), v[c0: c0 + L].cpu(), [0, 1],
                [0, L], scale, False)
            compare(o[c0 + t], lse[c0 + t], o_ref[0], l_ref[0], rel_o=REL_O16[torch.bfloat16])

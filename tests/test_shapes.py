"""GPU parity on ragged and edge shapes, with guard bands around every output.

Covers: Nq and Nkv not multiples of the 128-row tile (tails), Nq != Nkv with the causal
mask aligned bottom-right, causal rows that see no key (Nq > Nkv), one query row through
the prefill path, head dims 64 and 128, fp16 and bf16, fp32 and 16-bit O, a persistent
grid smaller than the work (num_ctas), prefill with its K/V range split into parts
(num_splits; the small shapes above also take the split when the library chooses it) and
decode with several split counts.
"""
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_qkv
from fa_testlib import REL_O16, compare, has_b200

pytestmark = pytest.mark.gpu

GUARD = 64  # elements of canary on each side of O and LSE (keeps 16-byte alignment)
CANARY = 1234.5


@pytest.fixture(autouse=True)
def _device_clean():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    binding.fa_device_status(clear=True)
    yield
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0, "a kernel wait timed out"


def _guarded(n, dtype):
    buf = torch.full((n + 2 * GUARD,), CANARY, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + n]


def _check_guard(buf, n):
    assert (buf[:GUARD] == CANARY).all() and (buf[GUARD + n:] == CANARY).all(), \
        "write outside the output buffer"


def _run_case(B, H, Nq, Nkv, d, dtype, causal, out_dtype=torch.float32, scale=None,
              num_ctas=0, num_splits=0, path="auto", seed=1):
    q, k, v = make_qkv(B, H, Nq, Nkv, d, dtype, seed)
    scale = d ** -0.5 if scale is None else scale
    n_o = B * H * Nq * d
    obuf, o = _guarded(n_o, out_dtype)
    lbuf, lse = _guarded(B * H * Nq, torch.float32)
    binding.attention(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale,
                      out=o.view(B, H, Nq, d), lse=lse.view(B, H, Nq), num_ctas=num_ctas,
                      num_splits=num_splits, path=path)
    torch.cuda.synchronize()
    _check_guard(obuf, n_o)
    _check_guard(lbuf, B * H * Nq)
    o_ref, l_ref = oracle.attention(q, k, v, scale, causal)
    rel = REL_O16[dtype] if out_dtype != torch.float32 else 0.0
    return compare(o.view(B, H, Nq, d), lse.view(B, H, Nq), o_ref, l_ref, rel_o=rel)


RAGGED = [
    # B, H, Nq, Nkv
    (1, 1, 2, 2),
    (1, 2, 17, 17),
    (2, 1, 127, 127),
    (1, 1, 129, 129),
    (1, 3, 255, 257),
    (1, 2, 300, 1000),   # Nq < Nkv: bottom-right causal
    (1, 2, 1000, 300),   # Nq > Nkv: early causal rows see nothing
    (1, 1, 383, 130),
    (2, 2, 513, 513),
]


@pytest.mark.parametrize("shape", RAGGED)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_ragged_prefill(shape, causal, d, dtype):
    _run_case(*shape, d, dtype, causal)


@pytest.mark.parametrize("d,dtype", [(64, torch.bfloat16), (128, torch.float16)])
@pytest.mark.parametrize("causal", [False, True])
def test_other_dtype_pairs(d, dtype, causal):
    _run_case(2, 3, 333, 333, d, dtype, causal)


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_16bit_output(d, dtype):
    _run_case(1, 3, 400, 400, d, dtype, True, out_dtype=dtype)


@pytest.mark.parametrize("num_ctas", [1, 3, 7])
def test_persistent_grid_smaller_than_work(num_ctas):
    _run_case(2, 3, 700, 700, 128, torch.bfloat16, True, num_ctas=num_ctas)


# A causal launch whose Q-tile pairs would all get their own CTA makes each Q tile a unit
# instead, its even K/V tiles on one softmax warpgroup and its odd ones on the other, the two
# partial results merged at the end.  A grid one CTA short of the pairs runs the ordinary
# pairs.  Both must match the oracle, and each other within the same tolerance.  A grid of
# exactly the pair count runs the per-tile units with some CTAs taking two of them.
# Shapes: odd tile counts, Nq != Nkv (bottom-right mask; rows that see no key), a single
# query row, a single K/V tile, the benchmark's d=64 MHA shape.
@pytest.mark.parametrize("shape", [(1, 2, 640, 640, 64, torch.bfloat16),
                                   (2, 3, 1000, 1200, 128, torch.float16),
                                   (1, 3, 773, 773, 128, torch.bfloat16),
                                   (1, 2, 1, 300, 64, torch.bfloat16),
                                   (1, 2, 900, 200, 64, torch.float16),
                                   (2, 2, 100, 100, 128, torch.bfloat16),
                                   (2, 8, 2048, 2048, 64, torch.float16)])
def test_causal_small_launch_interleaved_kv(shape):
    B, H, Nq, Nkv, d, dtype = shape
    units = B * H * (((Nq + 127) // 128 + 1) // 2)
    assert units <= torch.cuda.get_device_properties(0).multi_processor_count
    q, k, v = make_qkv(B, H, Nq, Nkv, d, dtype, 21)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o_ref, l_ref = oracle.attention(q, k, v, d ** -0.5, True)
    o_i, l_i = binding.attention(qc, kc, vc, causal=True, num_ctas=0, num_splits=1)
    compare(o_i, l_i, o_ref, l_ref)
    o_g, l_g = binding.attention(qc, kc, vc, causal=True, num_ctas=units, num_splits=1)
    compare(o_g, l_g, o_ref, l_ref)
    if units > 1:
        o_a, l_a = binding.attention(qc, kc, vc, causal=True, num_ctas=units - 1, num_splits=1)
        compare(o_a, l_a, o_ref, l_ref)
        compare(o_i, l_i, o_a.float().cpu().double().numpy(), l_a.cpu().double().numpy())


# Without the causal mask every pair takes the same number of steps, so a non-causal launch
# runs per-tile interleaved-K/V units only when every Q tile gets its own CTA (a grid of at
# least twice the pair count); a grid one CTA short of that runs the pairs.
@pytest.mark.parametrize("shape", [(1, 2, 640, 640, 64, torch.bfloat16),
                                   (2, 3, 1000, 1200, 128, torch.float16),
                                   (1, 1, 100, 300, 128, torch.bfloat16),
                                   (2, 4, 2048, 2048, 64, torch.float16)])
def test_noncausal_small_launch_interleaved_kv(shape):
    B, H, Nq, Nkv, d, dtype = shape
    pairs = B * H * (((Nq + 127) // 128 + 1) // 2)
    assert 2 * pairs <= torch.cuda.get_device_properties(0).multi_processor_count
    q, k, v = make_qkv(B, H, Nq, Nkv, d, dtype, 23)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o_ref, l_ref = oracle.attention(q, k, v, d ** -0.5, False)
    o_i, l_i = binding.attention(qc, kc, vc, causal=False, num_ctas=0, num_splits=1)
    compare(o_i, l_i, o_ref, l_ref)
    o_g, l_g = binding.attention(qc, kc, vc, causal=False, num_ctas=2 * pairs, num_splits=1)
    torch.cuda.synchronize()
    assert torch.equal(o_g, o_i) and torch.equal(l_g, l_i)
    o_a, l_a = binding.attention(qc, kc, vc, causal=False, num_ctas=2 * pairs - 1, num_splits=1)
    compare(o_a, l_a, o_ref, l_ref)
    compare(o_i, l_i, o_a.float().cpu().double().numpy(), l_a.cpu().double().numpy())


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_interleaved_kv_16bit_output_negative_scale(d, dtype):
    # the per-tile units' merge and store path with 16-bit output (guard bands around O and
    # LSE), a negative scale (the row max taken from the minimum score), and a ragged tail
    _run_case(1, 2, 700, 700, d, dtype, True, out_dtype=dtype, scale=-0.3)
    _run_case(2, 3, 333, 333, d, dtype, True, out_dtype=dtype)


@pytest.mark.parametrize("num_splits", [1, 2, 3, 4, 7, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_prefill_kv_split_counts(num_splits, causal):
    # 9 key tiles: 7 parts leave some pairs' parts empty, 64 is clamped to the tile count
    _run_case(1, 2, 700, 1100, 128, torch.bfloat16, causal, num_splits=num_splits)


@pytest.mark.parametrize("shape", [(1, 2, 1000, 300), (2, 1, 300, 1000), (1, 1, 129, 640)])
@pytest.mark.parametrize("num_ctas", [0, 1, 5])
def test_prefill_kv_split_ragged_small_grid(shape, num_ctas):
    # causal rows that see no key (Nq > Nkv), bottom-right alignment (Nq < Nkv), and a
    # persistent grid smaller than the split work
    _run_case(*shape, 64, torch.float16, True, num_ctas=num_ctas, num_splits=3)


@pytest.mark.parametrize("d,dtype", [(64, torch.bfloat16), (128, torch.float16)])
def test_prefill_kv_split_16bit_output_and_negative_scale(d, dtype):
    _run_case(1, 3, 500, 900, d, dtype, True, out_dtype=dtype, num_splits=4)
    _run_case(1, 2, 400, 800, d, dtype, False, scale=-0.3, num_splits=2)


@pytest.mark.parametrize("Nkv", [1, 5, 64, 65, 1000])
def test_prefill_path_single_query(Nkv):
    _run_case(2, 2, 1, Nkv, 128, torch.bfloat16, True, path="prefill")


@pytest.mark.parametrize("Nkv", [1, 7, 63, 64, 65, 129, 4097])
@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_decode_shapes(Nkv, d, dtype):
    _run_case(2, 3, 1, Nkv, d, dtype, False)


@pytest.mark.parametrize("num_splits", [1, 2, 5, 16, 64, 1000])
def test_decode_split_counts(num_splits):
    _run_case(2, 4, 1, 3000, 128, torch.bfloat16, False, num_splits=num_splits)


def test_decode_16bit_output():
    _run_case(3, 2, 1, 2000, 128, torch.bfloat16, False, out_dtype=torch.bfloat16)


def test_large_negative_and_zero_scale():
    _run_case(1, 2, 260, 260, 128, torch.bfloat16, True, scale=0.0)
    _run_case(1, 2, 260, 260, 128, torch.bfloat16, False, scale=-0.3)
    _run_case(2, 2, 1, 900, 128, torch.bfloat16, False, scale=-0.3)

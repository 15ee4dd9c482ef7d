"""Properties of the CUDA path that hold exactly or at any size (GPU)."""
import numpy as np
import pytest
import torch

from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_qkv, randn
from fa_testlib import MAX_ABS_LSE, MAX_ABS_O, has_b200

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    binding.fa_device_status(clear=True)
    yield
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0, "a kernel wait timed out"


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_causal_row0_is_v0_exactly(d, dtype):
    q, k, v = make_qkv(2, 4, 600, 600, d, dtype, 3, device="cuda")
    o, lse = binding.attention(q, k, v, causal=True, scale=0.2)
    torch.cuda.synchronize()
    assert torch.equal(o[:, :, 0, :], v[:, :, 0, :].float())
    s00 = 0.2 * (q[:, :, 0, :].double() * k[:, :, 0, :].double()).sum(-1)
    assert (lse[:, :, 0].double() - s00).abs().max().item() <= 1e-4


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_visible_v(causal):
    B, H, N, d = 1, 2, 700, 128
    q, k, v = make_qkv(B, H, N, N, d, torch.bfloat16, 8, device="cuda")
    k = k[:, :, :1, :].expand(B, H, N, d).contiguous()
    o, lse = binding.attention(q, k, v, causal=causal, scale=0.3)
    torch.cuda.synchronize()
    vf = v.double()
    if causal:
        ref = vf.cumsum(2) / torch.arange(1, N + 1, device="cuda", dtype=torch.float64)[:, None]
        cnt = torch.arange(1, N + 1, device="cuda", dtype=torch.float64)
    else:
        ref = vf.mean(2, keepdim=True).expand_as(vf)
        cnt = torch.full((N,), float(N), device="cuda", dtype=torch.float64)
    assert (o.double() - ref).abs().max().item() <= MAX_ABS_O
    s = 0.3 * (q.double() * k[:, :, :1, :].double()).sum(-1)
    assert (lse.double() - (s + cnt.log())).abs().max().item() <= MAX_ABS_LSE


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance_integer_inputs(causal):
    """Integer-valued inputs make Q K^T exact in fp32; adding the integer vector u to
    every key shifts row i's scores by scale * q_i.u: O is unchanged, LSE moves by it."""
    B, H, N, d = 1, 2, 520, 128
    g = torch.Generator(device="cpu").manual_seed(9)
    q = torch.randint(-2, 3, (B, H, N, d), generator=g).to(torch.bfloat16).cuda()
    k = torch.randint(-2, 3, (B, H, N, d), generator=g).to(torch.bfloat16).cuda()
    v = randn((B, H, N, d), 10, torch.bfloat16, device="cuda")
    u = torch.randint(-1, 2, (d,), generator=g).to(torch.bfloat16).cuda()
    scale = 0.05
    o1, l1 = binding.attention(q, k, v, causal=causal, scale=scale)
    o2, l2 = binding.attention(q, (k + u).contiguous(), v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert (o1 - o2).abs().max().item() <= 2e-3
    shift = scale * (q.double() * u.double()).sum(-1)
    assert ((l2.double() - l1.double()) - shift).abs().max().item() <= MAX_ABS_LSE


def test_bitwise_deterministic():
    q, k, v = make_qkv(1, 8, 1500, 1500, 128, torch.bfloat16, 4, device="cuda")
    a = binding.attention(q, k, v, causal=True)
    b = binding.attention(q, k, v, causal=True)
    qd, kd, vd = make_qkv(4, 8, 1, 5000, 128, torch.bfloat16, 5, device="cuda")
    c = binding.attention(qd, kd, vd)
    e = binding.attention(qd, kd, vd)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(c[0], e[0]) and torch.equal(c[1], e[1])


def test_decode_split_counts_agree():
    q, k, v = make_qkv(4, 8, 1, 20000, 128, torch.bfloat16, 6, q_std=3.0, device="cuda")
    outs = [binding.attention(q, k, v, num_splits=s) for s in (1, 4, 16, 64, 0)]
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert (o - outs[0][0]).abs().max().item() <= 1e-4
        assert (l - outs[0][1]).abs().max().item() <= 1e-4


@pytest.mark.parametrize("num_splits", [1, 3])
def test_prefill_grid_sizes_agree_bitwise(num_splits):
    """Each Q tile (each part of its K/V range, when split) is computed by one CTA in a
    fixed order and the parts are merged in a fixed order, so the grid size must not change
    a single bit.  Unsplit causal launches with at least one CTA per Q-tile pair (24 here)
    run per-tile units whose K/V tiles two warpgroups share; among those grids too the
    result is fixed, and it differs from the paired one only in rounding."""
    q, k, v = make_qkv(2, 3, 900, 900, 128, torch.bfloat16, 7, device="cuda")
    ref = binding.attention(q, k, v, causal=True, num_ctas=1, num_splits=num_splits)
    for n in (5, 23) if num_splits == 1 else (0, 5, 200):
        o, l = binding.attention(q, k, v, causal=True, num_ctas=n, num_splits=num_splits)
        torch.cuda.synchronize()
        assert torch.equal(o, ref[0]) and torch.equal(l, ref[1])
    if num_splits == 1:
        ref_i = binding.attention(q, k, v, causal=True, num_ctas=0, num_splits=1)
        for n in (24, 31, 200):
            o, l = binding.attention(q, k, v, causal=True, num_ctas=n, num_splits=1)
            torch.cuda.synchronize()
            assert torch.equal(o, ref_i[0]) and torch.equal(l, ref_i[1])
        assert (ref_i[0] - ref[0]).abs().max().item() <= MAX_ABS_O
        assert (ref_i[1] - ref[1]).abs().max().item() <= MAX_ABS_LSE


def test_prefill_split_agrees_with_unsplit():
    """Splitting the K/V range changes only the rounding of the merge."""
    q, k, v = make_qkv(1, 4, 2048, 2048, 64, torch.float16, 8, q_std=3.0, device="cuda")
    ref = binding.attention(q, k, v, causal=True, num_splits=1)
    for s in (2, 4, 0):
        o, l = binding.attention(q, k, v, causal=True, num_splits=s)
        torch.cuda.synchronize()
        assert (o - ref[0]).abs().max().item() <= MAX_ABS_O
        assert (l - ref[1]).abs().max().item() <= MAX_ABS_LSE


def test_no_score_matrix_in_memory():
    """The n x n matrix never reaches HBM: at N = 16384 one head's fp32 scores alone would
    be 1 GiB, yet a call needs nothing beyond O, LSE and (for this small problem, whose
    K/V range is split) O(N d) partials from the library's pool, which a repeated call
    reuses."""
    q, k, v = make_qkv(1, 2, 16384, 16384, 128, torch.bfloat16, 11, device="cuda")
    o = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    binding.attention(q, k, v, causal=True, out=o, lse=lse)  # warm: library state
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    binding.attention(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (64 << 20)


def test_device_wait_timeout_is_reported_not_hung():
    """A kernel whose wait can never finish gives up after about 1 s, sets the status
    word and returns; the context stays usable."""
    assert binding.fa_selftest_wait_timeout(None) == binding.FA_OK
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 8  # FA_DEV_TIMEOUT_DECODE
    assert binding.fa_device_status(clear=True) == 0
    q, k, v = make_qkv(1, 1, 128, 128, 64, torch.float16, 1, device="cuda")
    o, _ = binding.attention(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()

"""GPU parity of the FP8-Q/K prefill (fa_fwd_fp8) against the fp64 oracle
(oracle.fp8_qk_attention: attention() of the dequantised E4M3 tensors, pinned on the CPU).
P stays in V's 16-bit type, so the bf16 tolerances apply unchanged."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import randn
from fa_testlib import REL_O16, compare, has_b200, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    binding.fa_device_status(clear=True)
    yield
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0, "a kernel wait timed out"


def _quantise(x):
    """Per-tensor scale to the E4M3 range, then round to E4M3 codes."""
    s = float(x.abs().max()) / 448.0
    return (x / s).to(torch.float8_e4m3fn).view(torch.uint8), s


def _inputs(B, H, Nq, Nkv, vdtype, seed, std=1.0):
    qf = randn((B, H, Nq, 128), seed, torch.float32, std)
    kf = randn((B, H, Nkv, 128), seed + 1, torch.float32, std)
    v = randn((B, H, Nkv, 128), seed + 2, vdtype)
    q8, qs = _quantise(qf)
    k8, ks = _quantise(kf)
    return q8, qs, k8, ks, v


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("vdtype", [torch.bfloat16, torch.float16])
def test_fp8_matches_oracle(causal, vdtype):
    B, H, Nq, Nkv = 2, 3, 300, 333
    q8, qs, k8, ks, v = _inputs(B, H, Nq, Nkv, vdtype, 1200)
    o, lse = binding.fp8_attention(q8.cuda(), k8.cuda(), v.cuda(), qs, ks, causal=causal,
                                   scale=128 ** -0.5)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.fp8_qk_attention(q8, k8, v, qs, ks, 128 ** -0.5, causal)
    compare(o, lse, o_ref, l_ref)


def test_fp8_16bit_out_peaky():
    """Larger scores (Q std 4 before quantisation), 16-bit O."""
    B, H, N = 1, 2, 520
    q8, qs, k8, ks, v = _inputs(B, H, N, N, torch.bfloat16, 1300, std=4.0)
    o, lse = binding.fp8_attention(q8.cuda(), k8.cuda(), v.cuda(), qs, ks, causal=True,
                                   scale=128 ** -0.5, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.fp8_qk_attention(q8, k8, v, qs, ks, 128 ** -0.5, True)
    compare(o, lse, o_ref, l_ref, rel_o=REL_O16[torch.bfloat16])


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_equals_bf16_path_on_exact_values(causal):
    """Small integers are exact in E4M3 and bf16 and their dot products are exact in
    fp32, so S, and with it the whole result, must equal fa_fwd's bit for bit (with Q-tile
    pairs: a one-CTA grid, since the FP8 path always pairs)."""
    B, H, N = 1, 2, 384
    g = torch.Generator().manual_seed(31)
    qi = torch.randint(-3, 4, (B, H, N, 128), generator=g).float()
    ki = torch.randint(-3, 4, (B, H, N, 128), generator=g).float()
    v = randn((B, H, N, 128), 1400, torch.bfloat16)
    q8 = qi.to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = ki.to(torch.float8_e4m3fn).view(torch.uint8)
    o8, l8 = binding.fp8_attention(q8.cuda(), k8.cuda(), v.cuda(), 1.0, 1.0, causal=causal,
                                   scale=0.02)
    o16, l16 = binding.attention(qi.to(torch.bfloat16).cuda(), ki.to(torch.bfloat16).cuda(),
                                 v.cuda(), causal=causal, scale=0.02, num_ctas=1, num_splits=1)
    torch.cuda.synchronize()
    assert torch.equal(o8, o16) and torch.equal(l8, l16)


def test_fp8_full_size_sampled():
    """The long causal prefill shape (B=1, H=32, N=8192) with E4M3 Q and K, sampled rows."""
    B, H, N = 1, 32, 8192
    qf = randn((B, H, N, 128), 1500, torch.float32, device="cuda")
    kf = randn((B, H, N, 128), 1501, torch.float32, device="cuda")
    v = randn((B, H, N, 128), 1502, torch.bfloat16, device="cuda")
    q8, qs = _quantise(qf)
    k8, ks = _quantise(kf)
    del qf, kf
    o, lse = binding.fp8_attention(q8, k8, v, qs, ks, causal=True, scale=128 ** -0.5)
    torch.cuda.synchronize()
    rows = sample_rows(B, H, N, per_head=24, seed=15)
    o_ref, l_ref = oracle.fp8_qk_attention(q8.cpu(), k8.cpu(), v.cpu(), qs, ks, 128 ** -0.5,
                                           True, rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, 128)[idx], lse.reshape(-1)[idx], o_ref, l_ref)


@pytest.mark.parametrize("N", [1, 300, 1024])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_matches_oracle_bitwise(N, dtype):
    """fa_quantize_e4m3 against the oracle's per-tile quantisation (written from the E4M3
    format): identical scales and identical codes, byte for byte (both take the scale and
    the division in fp32 and round to nearest even)."""
    x = randn((2, 3, N, 128), 1400 + N, dtype, 3.0)
    x[0, 1, : min(N, 128)] = 0                  # an all-zero tile: scale 1, codes 0
    if N > 200:
        x[1, 2, 150] *= 50                      # one tile dominated by a single row
    codes, scales = binding.quantize_e4m3(x.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.e4m3_quantize_tiles(x.reshape(6, N, 128))
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy().reshape(6, N, 128), c_ref)


def test_quantize_many_tiles_per_sm_bitwise():
    """A launch of several waves (48 heads of 4,173 rows: 33 tiles each, the last one 77 rows
    high, about eleven tiles per SM): scales and codes equal the oracle's byte for byte."""
    x = randn((4, 12, 4173, 128), 1700, torch.bfloat16, 2.0)
    x[1, 3, 4096:] *= 1e-3                      # a ragged last tile at another scale
    codes, scales = binding.quantize_e4m3(x.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.e4m3_quantize_tiles(x.reshape(48, 4173, 128))
    assert np.array_equal(scales.cpu().numpy().reshape(s_ref.shape), s_ref)
    assert np.array_equal(codes.cpu().numpy().reshape(c_ref.shape), c_ref)


def _tiles_of_every_value_up_to(amax_bits, dtype):
    """[T, 128, 128] tiles of the 16-bit type: for each amax bit pattern a, every
    non-negative value with bits 0..a (alternate ones negated), 16,383 to a tile, each
    tile also holding a itself, so that its scale is amax / 448; zeros fill the rest."""
    tiles = []
    for a in amax_bits:
        vals = np.arange(a + 1, dtype=np.uint16)
        vals[1::2] |= 0x8000
        for g in range(0, a + 1, 16383):
            t = np.zeros(16384, dtype=np.uint16)
            part = vals[g:g + 16383]
            t[:part.size] = part
            t[16383] = a
            tiles.append(t)
    bits = torch.from_numpy(np.stack(tiles).view(np.int16)).reshape(-1, 128, 128)
    return bits.view(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_every_value_below_sampled_amax(dtype):
    """The codes of every value at or below a tile's amax, for amax sampled over the whole
    16-bit range (around the smallest scale, 2^-100, that takes the reciprocal-and-correction
    quotient; subnormal and largest finite amax), equal the oracle's byte for byte: the
    oracle divides each element by the scale in fp32."""
    top = 0x7F7F if dtype == torch.bfloat16 else 0x7BFF
    rng = np.random.default_rng(1600)
    fixed = [1, 2, 3, 0x7F, 0x80, 0x0B2A, 0x0400, top]
    if dtype == torch.bfloat16:
        fixed += list(range(0x11D8, 0x11E9))       # scale just below and above 2^-100
    amax_bits = sorted(set(fixed + rng.integers(1, top + 1, 150).tolist()))
    x = _tiles_of_every_value_up_to(amax_bits, dtype)
    codes, scales = binding.quantize_e4m3(x.reshape(1, -1, 128, 128).cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.e4m3_quantize_tiles(x)
    assert np.array_equal(scales.cpu().numpy().reshape(-1), s_ref.reshape(-1))
    got = codes.cpu().numpy().reshape(c_ref.shape)
    bad = np.argwhere(got != c_ref)
    assert bad.size == 0, f"{len(bad)} codes differ, first at tile/row/col {bad[0].tolist()}"


def _quant_reference(q, k, v, scale, causal, rows=None):
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    q8, qs = oracle.e4m3_quantize_tiles(q.reshape(B * H, Nq, d))
    k8, ks = oracle.e4m3_quantize_tiles(k.reshape(B * H, Nkv, d))
    return oracle.fp8_tile_scaled_attention(q8.reshape(B, H, Nq, d), qs, k8.reshape(B, H, Nkv, d),
                                            ks, v, scale, causal, rows=rows)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fp8_quant_matches_oracle(causal, dtype):
    """fa_fwd_fp8_quant (Q and K quantised on the fly, one scale per 128-row tile) against
    the oracle's quantisation and attention of the dequantised tensors; ragged tiles."""
    B, H, Nq, Nkv = 2, 3, 300, 333
    q = randn((B, H, Nq, 128), 1500, dtype, 2.0)
    k = randn((B, H, Nkv, 128), 1501, dtype)
    v = randn((B, H, Nkv, 128), 1502, dtype)
    o, lse = binding.fp8_quant_attention(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    o_ref, l_ref = _quant_reference(q, k, v, 128 ** -0.5, causal)
    compare(o, lse, o_ref, l_ref)


def test_fp8_quant_full_size_every_row():
    """The benchmark's configuration (B=1, H=32, N=8192, causal, bf16 O), every output."""
    from exact_io_aware_59_b200.inputs import WORKLOADS, workload_qkv
    w = WORKLOADS["long_prefill_causal"]
    q, k, v = workload_qkv(w, device="cuda")
    o, lse = binding.fp8_quant_attention(q, k, v, causal=True, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    o_ref, l_ref = _quant_reference(q.cpu(), k.cpu(), v.cpu(), w.softmax_scale, True)
    compare(o, lse, o_ref, l_ref, rel_o=REL_O16[torch.bfloat16])

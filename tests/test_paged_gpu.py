"""GPU parity of the paged-KV decode (fa_fwd_decode_paged) against the fp64 oracle.

The oracle gathers each sequence's keys through the block table and runs the two-pass
attention (oracle.paged_decode_attention, pinned on the CPU against contiguous keys).
Tolerances as for the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import randn
from fa_testlib import REL_O16, compare, has_b200

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")
    binding.fa_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def _make_paged(B, H, d, page_size, lens, num_pages, dtype, seed):
    """Random caches; sequence b owns ceil(len/page_size) distinct pages in random order.
    Table entries past a sequence's pages point at other valid pages."""
    rng = np.random.default_rng(seed)
    per = [(L + page_size - 1) // page_size for L in lens]
    P = max(1, max(per))
    assert sum(per) <= num_pages
    perm = rng.permutation(num_pages)
    table = rng.integers(0, num_pages, size=(B, P)).astype(np.int32)
    pos = 0
    for b, n in enumerate(per):
        table[b, :n] = perm[pos:pos + n]
        pos += n
    q = randn((B, H, d), seed, dtype)
    kc = randn((num_pages, H, page_size, d), seed + 1, dtype)
    vc = randn((num_pages, H, page_size, d), seed + 2, dtype)
    return q, kc, vc, torch.from_numpy(table), torch.tensor(lens, dtype=torch.int32)


def _run(q, kc, vc, table, lens, scale, **kw):
    o, lse = binding.paged_decode(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), lens.cuda(),
                                  scale=scale, **kw)
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0
    return o, lse


@pytest.mark.parametrize("page_size", [16, 64, 256])
@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_paged_decode_matches_oracle(page_size, d, dtype):
    lens = [0, 1, 15, 16, 17, 63, 64, 65, 700, 2047]
    B, H = len(lens), 4
    q, kc, vc, table, sl = _make_paged(B, H, d, page_size, lens, 256, dtype, 40 + page_size)
    o, lse = _run(q, kc, vc, table, sl, d ** -0.5)
    o_ref, l_ref = oracle.paged_decode_attention(q, kc, vc, table, lens, d ** -0.5)
    compare(o, lse, o_ref, l_ref)


@pytest.mark.parametrize("num_splits", [1, 7, 0])
def test_paged_decode_16bit_out_and_splits(num_splits):
    lens = [3000, 1, 0, 4096, 129]
    B, H, d, ps = len(lens), 8, 128, 32
    q, kc, vc, table, sl = _make_paged(B, H, d, ps, lens, 400, torch.bfloat16, 77)
    o, lse = _run(q, kc, vc, table, sl, 0.1, out_dtype=torch.bfloat16, num_splits=num_splits)
    assert o.dtype == torch.bfloat16
    o_ref, l_ref = oracle.paged_decode_attention(q, kc, vc, table, lens, 0.1)
    compare(o, lse, o_ref, l_ref, rel_o=REL_O16[torch.bfloat16])


def test_one_page_per_sequence_is_the_contiguous_decode():
    """With one page per sequence the cache [B,H,L,d] is the contiguous K/V layout, so the
    paged call must give fa_fwd_decode's result bit for bit."""
    B, H, L, d = 4, 8, 1000, 128
    q, kc, vc, _, _ = _make_paged(B, H, d, 1024, [L] * B, B, torch.bfloat16, 91)
    table = torch.arange(B, dtype=torch.int32).reshape(B, 1)
    sl = torch.full((B,), L, dtype=torch.int32)
    o_p, l_p = _run(q, kc, vc, table, sl, 0.2)
    k = kc[:, :, :L].contiguous().cuda()
    v = vc[:, :, :L].contiguous().cuda()
    o_c, l_c = binding.attention(q.reshape(B, H, 1, d).cuda(), k, v, scale=0.2, path="decode")
    torch.cuda.synchronize()
    assert torch.equal(o_p, o_c.reshape(B, H, d)) and torch.equal(l_p, l_c.reshape(B, H))


def test_paged_decode_full_size_sampled():
    """The decode workload's shape (B=16, H=32, 32768 keys, d=128, bf16) in 64-key pages
    spread over the pool in random order; two sequences checked against the oracle."""
    B, H, L, d, ps = 16, 32, 32768, 128, 64
    P = L // ps
    g = torch.Generator(device="cuda").manual_seed(5005)
    perm = torch.randperm(B * P, generator=g, device="cuda").to(torch.int32)
    table = perm.reshape(B, P).contiguous()
    kc = torch.randn(B * P, H, ps, d, generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn(B * P, H, ps, d, generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn(B, H, d, generator=g, device="cuda").to(torch.bfloat16)
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    o, lse = binding.paged_decode(q, kc, vc, table, sl, scale=d ** -0.5)
    torch.cuda.synchronize()
    assert binding.fa_device_status(clear=True) == 0
    for b in (0, B - 1):
        kb = kc[table[b].long()].permute(1, 0, 2, 3).reshape(1, H, L, d).cpu()
        vb = vc[table[b].long()].permute(1, 0, 2, 3).reshape(1, H, L, d).cpu()
        o_ref, l_ref = oracle.attention(q[b].reshape(1, H, 1, d).cpu(), kb, vb, d ** -0.5, False)
        compare(o[b], lse[b], o_ref[0, :, 0], l_ref[0, :, 0])


def test_out_of_range_table_and_lengths_are_flagged():
    """A table entry outside [0, num_pages) and a length beyond the table's capacity are
    caught by the kernel's own bounds checks: the status word says so, nothing faults."""
    B, H, d, ps = 3, 2, 64, 16
    q, kc, vc, table, sl = _make_paged(B, H, d, ps, [40, 40, 40], 16, torch.float16, 13)
    table[0, 1] = 16          # one past the last page
    table[1, 0] = -3
    sl[2] = 40 + 10 * ps      # more keys than the table row holds
    o, lse = binding.paged_decode(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), sl.cuda(), scale=0.1)
    torch.cuda.synchronize()
    status = binding.fa_device_status(clear=True)
    assert status & binding.FA_DEV_BAD_INPUT
    assert torch.isfinite(o).all()

"""fa_fwd_decode_noalloc: the decode entry point for callers that cannot allocate device
memory (for example a runtime whose device memory is all handed to its own pool, or a
plug-in whose host forbids device allocations after start-up).  It keeps the split
partials in the library's fixed static device array instead of workspace from the
library's memory pool.

Checked here, through the C ABI: on two calls in a row (the second finds the first call's
partials still in the shared array) its output matches fa_fwd_decode's within the parity
tolerances, and the fp64 CPU oracle's (every head of the first call, sampled heads of the
second); it allocates nothing once the array is set up; and a request too large for the
array is refused before anything is enqueued.  This file is collected last on purpose
and does not depend on the other test files.
"""
import ctypes

import pytest
import torch

import numpy as np

import oracle
from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200.inputs import make_qkv
from fa_testlib import MAX_ABS_LSE, MAX_ABS_O, MEAN_ABS_O, REL_O16, compare, has_b200

pytestmark = pytest.mark.gpu


def _call(fn, q, k, v, o, lse, scale, num_splits=0):
    B, H, _, d = q.shape
    Nkv = k.shape[2]
    ic = binding.FA_BF16 if q.dtype == torch.bfloat16 else binding.FA_F16
    oc = binding._dtype_code(o.dtype)
    stream = torch.cuda.current_stream().cuda_stream
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H,
              Nkv, d, ctypes.c_float(scale), stream, ic, oc, num_splits)


def _close(o1, l1, o2, l2):
    d_o = (o1.double() - o2.double()).abs()
    assert d_o.max().item() <= MAX_ABS_O and d_o.mean().item() <= MEAN_ABS_O
    assert (l1.double() - l2.double()).abs().max().item() <= MAX_ABS_LSE


@pytest.fixture(autouse=True)
def _needs_b200():
    if not has_b200():
        pytest.skip("needs a B200 (sm_100a)")


@pytest.mark.parametrize("d,dtype,out_dtype", [(128, torch.bfloat16, torch.float32),
                                               (64, torch.float16, torch.float16)])
def test_noalloc_matches_fa_fwd_decode_twice(d, dtype, out_dtype):
    lib = binding.library()
    shapes = [(4, 8, 5000, 11), (16, 32, 32768, 12)]   # second call: other shape, other data
    for B, H, Nkv, seed in shapes:
        q, k, v = make_qkv(B, H, 1, Nkv, d, dtype, 1000 * seed, device="cuda")
        scale = d ** -0.5
        o_ref = torch.empty((B, H, 1, d), dtype=out_dtype, device="cuda")
        l_ref = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
        o_new = torch.full_like(o_ref, float("nan"))
        l_new = torch.full_like(l_ref, float("nan"))
        assert _call(lib.fa_fwd_decode, q, k, v, o_ref, l_ref, scale) == binding.FA_OK
        assert _call(lib.fa_fwd_decode_noalloc, q, k, v, o_new, l_new, scale) == binding.FA_OK
        torch.cuda.synchronize()
        assert torch.isfinite(o_new).all() and torch.isfinite(l_new).all()
        _close(o_new, l_new, o_ref, l_ref)
        # against the oracle: every head of the small call, 16 heads of the large one
        BH = B * H
        heads = np.arange(BH) if BH <= 64 else np.unique(np.concatenate(
            [[0, BH - 1], np.random.default_rng(seed).choice(BH, 14, replace=False)]))
        sel = torch.from_numpy(heads).cuda()
        pick = lambda t, n: t.reshape(BH, n, d)[sel].reshape(1, -1, n, d).cpu()  # noqa: E731
        o_or, l_or = oracle.attention(pick(q, 1), pick(k, Nkv), pick(v, Nkv), scale, False)
        rel = 0.0 if out_dtype == torch.float32 else REL_O16[dtype]
        compare(o_new.reshape(BH, d)[sel], l_new.reshape(BH)[sel], o_or.reshape(-1, d),
                l_or.reshape(-1), rel_o=rel)
        del q, k, v
        torch.cuda.empty_cache()


def test_noalloc_allocates_nothing():
    lib = binding.library()
    q, k, v = make_qkv(8, 16, 1, 3000, 128, torch.bfloat16, 4040, device="cuda")
    o = torch.empty((8, 16, 1, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((8, 16, 1), dtype=torch.float32, device="cuda")
    assert _call(lib.fa_fwd_decode_noalloc, q, k, v, o, lse, 0.1) == binding.FA_OK  # set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        assert _call(lib.fa_fwd_decode_noalloc, q, k, v, o, lse, 0.1) == binding.FA_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_refuses_requests_larger_than_its_array():
    lib = binding.library()
    B, H, Nkv, d = 1, 4096, 64, 128   # 4096 heads: partials need ~35 MB > 8 MiB
    q, k, v = make_qkv(B, H, 1, Nkv, d, torch.bfloat16, 77, device="cuda")
    o = torch.full((B, H, 1, d), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((B, H, 1), 7.0, dtype=torch.float32, device="cuda")
    assert binding.fa_decode_workspace_bytes(B, H, Nkv, d, 0) > (8 << 20)
    assert _call(lib.fa_fwd_decode_noalloc, q, k, v, o, lse, 0.1) == binding.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (o == 7.0).all() and (lse == 7.0).all()   # nothing was enqueued
    assert _call(lib.fa_fwd_decode_noalloc, q, k, v, o, lse, 0.1, num_splits=-1) == \
        binding.FA_ERR_INVALID_ARG

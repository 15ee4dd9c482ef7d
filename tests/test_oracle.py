"""Pins for the fp64 CPU oracle, against facts the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a closed form, an
invariant, brute force written independently (numpy exp/sum with an explicit mask), a
library routine (torch CPU fp64 SDPA), or a byte count printed on the pages.
"""
import csv
import math
import os

import numpy as np
import pytest
import torch

from exact_io_aware_59_b200.inputs import make_qkv, randn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(t):
    return t.to(torch.float64).numpy()


def _visible_mask(Nq, Nkv, causal):
    """Boolean [Nq, Nkv]: query i sees key j (bottom-right alignment when causal)."""
    i = np.arange(Nq)[:, None]
    j = np.arange(Nkv)[None, :]
    return (j <= i + (Nkv - Nq)) if causal else np.ones((Nq, Nkv), dtype=bool)


def _brute(q, k, v, scale, causal):
    """exp(S) / sum exp(S) with no max subtraction; fine for |S| well below 700."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    mask = _visible_mask(Nq, Nkv, causal)
    o = np.zeros((B, H, Nq, d))
    lse = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        for h in range(H):
            s = scale * np.einsum("ic,jc->ij", q[b, h], k[b, h])
            e = np.where(mask, np.exp(s), 0.0)
            z = e.sum(axis=1)
            seen = z > 0
            o[b, h] = np.where(seen[:, None], e / np.where(seen, z, 1)[:, None], 0) @ v[b, h]
            lse[b, h] = np.where(seen, np.log(np.where(seen, z, 1)), -np.inf)
    return o, lse


SHAPES = [
    # B, H, Nq, Nkv, d
    (1, 1, 1, 1, 8),
    (1, 2, 5, 5, 16),
    (2, 3, 17, 17, 32),
    (1, 2, 9, 23, 16),   # Nq < Nkv
    (1, 2, 23, 9, 16),   # Nq > Nkv: causal rows 0..13 see nothing
    (1, 1, 130, 130, 64),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_bruteforce_tiny(oracle_mod, shape, causal, dtype):
    B, H, Nq, Nkv, d = shape
    q, k, v = make_qkv(B, H, Nq, Nkv, d, dtype, 11 + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle_mod.attention(q, k, v, scale, causal)
    ob, lb = _brute(q, k, v, scale, causal)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_fp64(oracle_mod, causal):
    """Library special case: torch's CPU fp64 math SDPA (square causal = its is_causal)."""
    B, H, N, d = 2, 3, 40, 32
    q, k, v = make_qkv(B, H, N, N, d, torch.bfloat16, 99)
    scale = 0.3
    o, _ = oracle_mod.attention(q, k, v, scale, causal)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), is_causal=causal, scale=scale
    ).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_matches_torch_sdpa_bottom_right_mask(oracle_mod):
    B, H, Nq, Nkv, d = 1, 2, 12, 31, 16
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.float16, 5)
    mask = torch.from_numpy(_visible_mask(Nq, Nkv, True))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), attn_mask=mask, scale=0.25
    ).numpy()
    o, _ = oracle_mod.attention(q, k, v, 0.25, True)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_normalised(oracle_mod, causal):
    """Softmax rows sum to one: with V all ones every visible row of O is exactly 1."""
    B, H, Nq, Nkv, d = 1, 2, 37, 37, 16
    q, k, _ = make_qkv(B, H, Nq, Nkv, d, torch.float16, 3, q_std=3.0)
    v = torch.ones(B, H, Nkv, d, dtype=torch.float16)
    o, _ = oracle_mod.attention(q, k, v, 1.0, causal)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-12)


def test_causal_row0_is_v0(oracle_mod):
    """The causal mask leaves query 0 only key 0: O_0 = V_0 exactly, LSE_0 = s_00."""
    B, H, N, d = 2, 2, 29, 32
    q, k, v = make_qkv(B, H, N, N, d, torch.bfloat16, 21, q_std=4.0)
    scale = 0.177
    o, lse = oracle_mod.attention(q, k, v, scale, True)
    assert np.array_equal(o[:, :, 0, :], _f64(v)[:, :, 0, :])
    s00 = scale * np.einsum("bhc,bhc->bh", _f64(q)[:, :, 0], _f64(k)[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s00, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_visible_v(oracle_mod, causal):
    B, H, Nq, Nkv, d = 1, 2, 19, 26, 16
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.float16, 8)
    k = k[:, :, :1, :].expand(B, H, Nkv, d).contiguous()
    scale = 0.5
    o, lse = oracle_mod.attention(q, k, v, scale, causal)
    vis = _visible_mask(Nq, Nkv, causal)
    vf, qf, kf = _f64(v), _f64(q), _f64(k)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                J = np.nonzero(vis[i])[0]
                np.testing.assert_allclose(o[b, h, i], vf[b, h, J].mean(axis=0), atol=1e-12)
                s = scale * qf[b, h, i] @ kf[b, h, 0]
                assert lse[b, h, i] == pytest.approx(s + math.log(len(J)), abs=1e-12)


def test_scale_zero_gives_mean(oracle_mod):
    B, H, Nq, Nkv, d = 2, 1, 11, 11, 8
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.bfloat16, 4)
    o, lse = oracle_mod.attention(q, k, v, 0.0, True)
    vf = _f64(v)
    for i in range(Nq):
        np.testing.assert_allclose(o[:, :, i], vf[:, :, : i + 1].mean(axis=2), atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], math.log(i + 1), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance(oracle_mod, causal):
    """Adding u to every key adds scale*q_i.u to row i's scores: O is unchanged and LSE
    moves by exactly that amount (the max subtraction must cancel it)."""
    B, H, Nq, Nkv, d = 1, 2, 13, 21, 16
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.float64, 6)
    u = randn((d,), 77, torch.float64, std=3.0)
    scale = 0.4
    o, lse = oracle_mod.attention(q, k, v, scale, causal)
    o2, lse2 = oracle_mod.attention(q, k + u, v, scale, causal)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-11)
    shift = scale * np.einsum("bhic,c->bhi", _f64(q), _f64(u))
    fin = np.isfinite(lse)
    np.testing.assert_allclose((lse2 - lse)[fin], shift[fin], rtol=0, atol=1e-10)


def test_large_scores_stay_finite(oracle_mod):
    """Scores near 1e4 overflow a softmax without max subtraction; the oracle must not."""
    B, H, N, d = 1, 1, 16, 8
    q, k, v = make_qkv(B, H, N, N, d, torch.float64, 12)
    o, lse = oracle_mod.attention(q * 100, k * 100, v, 1.0, False)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    qf, kf = _f64(q) * 100, _f64(k) * 100
    s = qf[0, 0] @ kf[0, 0].T
    # row-wise argmax dominates: O equals V at the argmax within float rounding
    top = s.argmax(axis=1)
    gap = np.sort(s, axis=1)[:, -1] - np.sort(s, axis=1)[:, -2]
    sure = gap > 60
    np.testing.assert_allclose(o[0, 0][sure], _f64(v)[0, 0][top[sure]], atol=1e-12)


def test_fully_masked_rows(oracle_mod):
    """Causal with Nq > Nkv: query i sees keys j <= i - (Nq - Nkv); rows before that see
    nothing and give O = 0, LSE = -inf."""
    q, k, v = make_qkv(1, 1, 10, 4, 8, torch.float16, 2)
    o, lse = oracle_mod.attention(q, k, v, 1.0, True)
    assert (o[0, 0, :6] == 0).all() and np.isneginf(lse[0, 0, :6]).all()
    assert np.isfinite(lse[0, 0, 6:]).all()
    np.testing.assert_array_equal(o[0, 0, 6], _f64(v)[0, 0, 0])


def test_sixteen_bit_decoding_is_exact(oracle_mod):
    """The C oracle decodes fp16/bf16 bit patterns itself; it must agree bit for bit
    with the same values passed as fp64 (subnormals, extremes and signed zero too)."""
    special = [0.0, -0.0, 6.0e-8, -6.0e-8, 1.0e-5, 65504.0, -65504.0, 0.333, 1024.5]
    for dtype in (torch.float16, torch.bfloat16):
        q, k, v = make_qkv(1, 2, 9, 9, 16, dtype, 31)
        vals = torch.tensor(special, dtype=dtype)
        v.view(-1)[: len(special)] = vals
        k.view(-1)[-len(special):] = vals * 0.001
        o16, l16 = oracle_mod.attention(q, k, v, 0.1, False)
        o64, l64 = oracle_mod.attention(q.double(), k.double(), v.double(), 0.1, False)
        assert np.array_equal(o16, o64) and np.array_equal(l16, l64)


def test_rows_subset_and_threads(oracle_mod):
    B, H, Nq, Nkv, d = 2, 2, 33, 40, 16
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.bfloat16, 13)
    o, lse = oracle_mod.attention(q, k, v, 0.2, True, nthreads=1)
    o4, lse4 = oracle_mod.attention(q, k, v, 0.2, True, nthreads=4)
    assert np.array_equal(o, o4) and np.array_equal(lse, lse4)
    rows = [0, 5, 32, 33, 70, B * H * Nq - 1]
    orow, lrow = oracle_mod.attention(q, k, v, 0.2, True, rows=rows)
    of, lf = o.reshape(-1, d), lse.reshape(-1)
    assert np.array_equal(orow, of[rows]) and np.array_equal(lrow, lf[rows])


@pytest.mark.parametrize("tau", [0.0, 8.0, 15.0])
@pytest.mark.parametrize("causal", [False, True])
def test_online_blockwise_equals_two_pass(oracle_mod, tau, causal):
    """The tiled online softmax (the method) reaches the two-pass definition."""
    rng = np.random.default_rng(int(tau) * 10 + causal)
    for trial in range(4):
        Nq, Nkv = int(rng.integers(1, 70)), int(rng.integers(1, 90))
        if causal and trial == 0:
            Nq, Nkv = 64, 64
        q, k, v = make_qkv(1, 2, Nq, Nkv, 16, torch.float64, 100 + trial, q_std=3.0)
        blocks = tuple(int(b) for b in rng.integers(1, 33, size=5))
        o2, l2 = oracle_mod.attention(q, k, v, 0.7, causal)
        o1, l1 = oracle_mod.online_softmax_attention(q, k, v, 0.7, causal, blocks, tau)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
        assert np.array_equal(np.isneginf(l1), np.isneginf(l2))
        fin = np.isfinite(l2)
        np.testing.assert_allclose(l1[fin], l2[fin], rtol=0, atol=1e-12)


def test_split_combine_equals_unsplit(oracle_mod):
    """Split-KV: partial results over any partition of the keys, merged by LSE, equal
    the result over all keys (one part may be empty)."""
    rng = np.random.default_rng(5)
    B, H, Nq, Nkv, d = 2, 2, 1, 300, 32
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.bfloat16, 55, q_std=2.0)
    o_full, l_full = oracle_mod.attention(q, k, v, 0.3, False)
    for S in (1, 2, 5, 16):
        cuts = np.sort(rng.choice(np.arange(1, Nkv), size=S - 1, replace=False))
        bounds = [0, *cuts.tolist(), Nkv]
        parts_o, parts_l = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            o_s, l_s = oracle_mod.attention(q, k[:, :, a:b], v[:, :, a:b], 0.3, False)
            parts_o.append(o_s)
            parts_l.append(l_s)
        parts_o.append(np.zeros_like(parts_o[0]))
        parts_l.append(np.full_like(parts_l[0], -np.inf))
        o, l = oracle_mod.lse_combine(parts_o, parts_l)
        np.testing.assert_allclose(o, o_full, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, l_full, rtol=0, atol=1e-12)
    o, l = oracle_mod.lse_combine([np.zeros((3, 4))] * 2, [np.full(3, -np.inf)] * 2)
    assert (o == 0).all() and np.isneginf(l).all()


def test_golden_byte_counts(oracle_mod):
    with open(os.path.join(GOLDEN, "byte_counts.txt")) as f:
        rows = [r for r in csv.reader((line for line in f if not line.startswith("#")),
                                     delimiter="|")]
    assert len(rows) == 7
    for kind, n, d, eb, term, val, unit, _cite in rows:
        n, d, eb, val = int(n), int(d), int(eb), int(val)
        if kind == "score_matrix":
            assert oracle_mod.score_matrix_bytes(n, eb) == val
        else:
            t = oracle_mod.standard_attention_traffic(n, d, eb)
            if term == "total":
                printed = [int(r[5]) for r in rows if r[0] == kind and r[4] != "total"]
                assert sum(printed) == val
                assert abs(t["total"] / 1e6 - val) < 2
            else:
                assert round(t[term] / 1e6) == val


# ---------------------------------------------------------------- paged KV cache (decode)
def _scatter_pages(K, V, page_size, num_pages, rng, dtype):
    """Writes contiguous K, V [B,H,Lmax,d] into pages [num_pages,H,page_size,d] in a random
    page order (unused pages and slots hold other random values); returns the caches and
    the block table."""
    B, H, Lmax, d = K.shape
    P = (Lmax + page_size - 1) // page_size
    perm = rng.permutation(num_pages)[: B * P].reshape(B, P)
    kc = torch.randn(num_pages, H, page_size, d).to(dtype)
    vc = torch.randn(num_pages, H, page_size, d).to(dtype)
    for b in range(B):
        for i in range(P):
            n = min(page_size, Lmax - i * page_size)
            kc[perm[b, i], :, :n] = K[b, :, i * page_size: i * page_size + n]
            vc[perm[b, i], :, :n] = V[b, :, i * page_size: i * page_size + n]
    return kc, vc, torch.from_numpy(perm.astype(np.int32))


@pytest.mark.parametrize("page_size", [16, 64])
def test_paged_decode_equals_contiguous(oracle_mod, page_size):
    """Pages in a random order, ragged lengths (0, 1, a page, a page + 1, full): the
    paged oracle equals attention() over each sequence's contiguous keys."""
    rng = np.random.default_rng(page_size)
    B, H, Lmax, d = 6, 3, 200, 32
    q = make_qkv(B, H, 1, 1, d, torch.bfloat16, 500)[0][:, :, 0]
    _, K, V = make_qkv(B, H, 1, Lmax, d, torch.bfloat16, 510)
    kc, vc, bt = _scatter_pages(K, V, page_size, 96, rng, torch.bfloat16)
    lens = [0, 1, page_size, page_size + 1, 137, Lmax]
    o, lse = oracle_mod.paged_decode_attention(q, kc, vc, bt, lens, 0.3)
    for b, L in enumerate(lens):
        if L == 0:
            assert (o[b] == 0).all() and np.isneginf(lse[b]).all()
            continue
        o_ref, l_ref = oracle_mod.attention(q[b].reshape(1, H, 1, d), K[b:b + 1, :, :L].contiguous(),
                                            V[b:b + 1, :, :L].contiguous(), 0.3, False)
        np.testing.assert_allclose(o[b], o_ref[0, :, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], l_ref[0, :, 0], rtol=0, atol=1e-12)


def test_paged_decode_pin_sees_a_wrong_page():
    """Negative control for the pin above: pointing one block-table entry at a page the
    sequence does not own changes the result, so a mis-indexed page would be caught.
    (Reordering a sequence's own pages would not: without a mask the keys form a set.)"""
    import oracle
    rng = np.random.default_rng(3)
    B, H, Lmax, d, ps = 1, 2, 128, 16, 16
    q = make_qkv(B, H, 1, 1, d, torch.bfloat16, 520)[0][:, :, 0]
    _, K, V = make_qkv(B, H, 1, Lmax, d, torch.bfloat16, 530)
    kc, vc, bt = _scatter_pages(K, V, ps, 16, rng, torch.bfloat16)
    unused = sorted(set(range(16)) - set(bt[0].tolist()))[0]
    bt2 = bt.clone()
    bt2[0, 2] = unused
    o1, _ = oracle.paged_decode_attention(q, kc, vc, bt, [Lmax - 20], 1.0)
    o2, _ = oracle.paged_decode_attention(q, kc, vc, bt2, [Lmax - 20], 1.0)
    assert np.isfinite(o1).all() and not np.allclose(o1, o2, atol=1e-6)


# ---------------------------------------------------------------- varlen (packed batches)
def _pack(x):
    """[B,H,L,d] -> token-major [B*L,H,d]."""
    B, H, L, d = x.shape
    return x.permute(0, 2, 1, 3).reshape(B * L, H, d).contiguous()


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equal_lengths_is_the_batched_oracle(oracle_mod, causal):
    """Equal lengths: the packed token-major batch gives attention() of the [B,H,L,d]
    batch, row for row (pins the token-major indexing and the per-sequence split)."""
    B, H, L, d = 3, 2, 50, 16
    q, k, v = make_qkv(B, H, L, L, d, torch.float16, 600)
    cu = [0, L, 2 * L, 3 * L]
    o, lse = oracle_mod.varlen_attention(_pack(q), _pack(k), _pack(v), cu, cu, 0.4, causal)
    o_ref, l_ref = oracle_mod.attention(q, k, v, 0.4, causal)
    np.testing.assert_array_equal(o, o_ref.transpose(0, 2, 1, 3).reshape(B * L, H, d))
    np.testing.assert_array_equal(lse, l_ref.transpose(0, 2, 1).reshape(B * L, H))


def test_varlen_sequences_are_isolated(oracle_mod):
    """Changing one sequence's keys and values changes only that sequence's rows; ragged
    and empty sequences, Nq != Nkv with bottom-right causal alignment."""
    H, d = 2, 16
    lq, lk = [5, 0, 40, 7, 3], [9, 4, 40, 0, 12]
    cq = np.concatenate([[0], np.cumsum(lq)]).tolist()
    ck = np.concatenate([[0], np.cumsum(lk)]).tolist()
    q = randn((cq[-1], H, d), 700, torch.bfloat16)
    k = randn((ck[-1], H, d), 701, torch.bfloat16)
    v = randn((ck[-1], H, d), 702, torch.bfloat16)
    o1, l1 = oracle_mod.varlen_attention(q, k, v, cq, ck, 0.5, True)
    k2, v2 = k.clone(), v.clone()
    k2[ck[2]:ck[3]] = randn((lk[2], H, d), 703, torch.bfloat16)
    v2[ck[2]:ck[3]] = randn((lk[2], H, d), 704, torch.bfloat16)
    o2, l2 = oracle_mod.varlen_attention(q, k2, v2, cq, ck, 0.5, True)
    other = np.r_[0:cq[2], cq[3]:cq[-1]]
    np.testing.assert_array_equal(o1[other], o2[other])
    np.testing.assert_array_equal(l1[other], l2[other])
    assert not np.allclose(o1[cq[2]:cq[3]], o2[cq[2]:cq[3]])
    # sequence 3 has no keys: O = 0, LSE = -inf
    assert (o1[cq[3]:cq[4]] == 0).all() and np.isneginf(l1[cq[3]:cq[4]]).all()
    # sequence 4: 3 queries, 12 keys, causal bottom-right: query i sees keys <= i + 9
    qb = q[cq[4]:cq[5]].permute(1, 0, 2).reshape(1, H, 3, d)
    kb = k[ck[4]:ck[5]].permute(1, 0, 2).reshape(1, H, 12, d)
    vb = v[ck[4]:ck[5]].permute(1, 0, 2).reshape(1, H, 12, d)
    s = torch.einsum("bhqd,bhkd->bhqk", qb.double(), kb.double()) * 0.5
    s = s.masked_fill(torch.arange(12)[None, :] > torch.arange(3)[:, None] + 9, float("-inf"))
    ref = torch.softmax(s, -1) @ vb.double()
    np.testing.assert_allclose(o1[cq[4]:cq[5]], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 (E4M3) queries and keys
def test_e4m3_decode_matches_torch_for_every_code(oracle_mod):
    """All 256 E4M3 codes decode to the values of torch.float8_e4m3fn (a library
    routine), NaN codes included."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ours = oracle_mod.e4m3_to_f64(codes)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref)) and np.isnan(ours).sum() == 2
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[fin], ref[fin])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0


def test_fp8_attention_is_attention_of_the_dequantised_tensors(oracle_mod):
    """The FP8 reference equals attention() on q_scale * Q and k_scale * K given as fp64,
    and the scales act as one factor on the scores (q_scale*k_scale*scale fixed)."""
    B, H, N, d = 1, 2, 40, 32
    qf = randn((B, H, N, d), 800, torch.float32, 3.0)
    kf = randn((B, H, N, d), 801, torch.float32, 3.0)
    v = randn((B, H, N, d), 802, torch.bfloat16)
    q8 = qf.to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = kf.to(torch.float8_e4m3fn).view(torch.uint8)
    o, lse = oracle_mod.fp8_qk_attention(q8, k8, v, 0.5, 0.25, 0.1, True)
    qd = q8.view(torch.float8_e4m3fn).to(torch.float64) * 0.5
    kd = k8.view(torch.float8_e4m3fn).to(torch.float64) * 0.25
    o_ref, l_ref = oracle_mod.attention(qd, kd, v.to(torch.float64), 0.1, True)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, l_ref)
    o2, l2 = oracle_mod.fp8_qk_attention(q8, k8, v, 1.0, 1.0, 0.1 * 0.5 * 0.25, True)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, lse, rtol=0, atol=1e-12)


def _e4m3_nearest_brute(x):
    """Nearest finite E4M3 value by exhaustive search over the 254 finite codes, ties to
    the code with the even mantissa; magnitudes beyond 448 saturate."""
    import oracle
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes)
    fin = ~np.isnan(vals)
    codes, vals = codes[fin], vals[fin]
    out = np.empty(x.shape, dtype=np.uint8)
    for i, xi in enumerate(np.asarray(x, dtype=np.float64).ravel()):
        xi = min(max(xi, -448.0), 448.0)
        dist = np.abs(vals - xi)
        best = np.flatnonzero(dist == dist.min())
        best = best[np.signbit(vals[best]) == np.signbit(xi)]   # -0.0 keeps its sign too
        even = [b for b in best if codes[b] & 1 == 0]
        out.ravel()[i] = codes[even[0] if even else best[0]]
    return out


def test_e4m3_encode_is_nearest_even_by_brute_force(oracle_mod):
    """The encoder against an exhaustive nearest-value search: random values over the whole
    range (subnormals and saturation included) and every midpoint between neighbours."""
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-520, 520, 3000), rng.uniform(-0.02, 0.02, 2000),
                        rng.normal(0, 3, 2000)]).astype(np.float32)
    vals = np.unique(oracle_mod.e4m3_to_f64(np.arange(0, 127, dtype=np.uint8)))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)   # exact in fp32
    x = np.concatenate([x, mids, -mids, [0.0, -0.0, 448.0, -448.0, 464.0, 1e6]]).astype(np.float32)
    assert np.array_equal(oracle_mod.e4m3_encode(x), _e4m3_nearest_brute(x))


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    """Within the finite range the encoder equals torch's float8_e4m3fn conversion (a library
    routine, round to nearest even), and every finite code round-trips."""
    x = randn((200000,), 905, torch.float32, 40.0).clamp(-448, 448)
    ours = oracle_mod.e4m3_encode(x.numpy())
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle_mod.e4m3_to_f64(codes)
    fin = ~np.isnan(vals)
    assert np.array_equal(oracle_mod.e4m3_encode(vals[fin].astype(np.float32)), codes[fin])


def test_e4m3_quantize_tiles_scale_and_error(oracle_mod):
    """Per-tile quantisation: every tile's largest magnitude maps to 448 exactly, an all-zero
    tile keeps scale 1 and codes 0, and decode(code) * scale is within half a spacing of x."""
    x = randn((3, 300, 16), 906, torch.bfloat16).float()
    x[1, 128:256] = 0.0
    codes, scales = oracle_mod.e4m3_quantize_tiles(x)
    assert scales.shape == (3, 3) and scales.dtype == np.float32
    dec = oracle_mod.e4m3_to_f64(codes)
    for b in range(3):
        for t in range(3):
            blk = dec[b, t * 128:(t + 1) * 128]
            if b == 1 and t == 1:
                assert scales[b, t] == 1.0 and (codes[b, 128:256] == 0).all()
                continue
            assert np.abs(blk).max() == 448.0
            xs = x[b, t * 128:(t + 1) * 128].numpy().astype(np.float64)
            rel = np.abs(blk * scales[b, t] - xs) / np.maximum(np.abs(xs), 2.0 ** -6 * scales[b, t])
            assert rel.max() <= 2.0 ** -4 + 1e-6   # half of the 3-bit mantissa spacing


def test_fp8_tile_scaled_attention_is_attention_of_the_dequantised_tensors(oracle_mod):
    B, H, N, d = 1, 2, 300, 32
    q = randn((B, H, N, d), 907, torch.bfloat16)
    k = randn((B, H, N, d), 908, torch.bfloat16)
    v = randn((B, H, N, d), 909, torch.bfloat16)
    q8, qs = oracle_mod.e4m3_quantize_tiles(q.reshape(B * H, N, d))
    k8, ks = oracle_mod.e4m3_quantize_tiles(k.reshape(B * H, N, d))
    q8, k8 = q8.reshape(B, H, N, d), k8.reshape(B, H, N, d)
    o, lse = oracle_mod.fp8_tile_scaled_attention(q8, qs, k8, ks, v, 0.2, True)
    qd = oracle_mod.e4m3_to_f64(q8) * np.repeat(qs, 128, axis=1)[:, :N].reshape(B, H, N, 1)
    kd = oracle_mod.e4m3_to_f64(k8) * np.repeat(ks, 128, axis=1)[:, :N].reshape(B, H, N, 1)
    o_ref, l_ref = oracle_mod.attention(torch.from_numpy(qd), torch.from_numpy(kd),
                                        v.to(torch.float64), 0.2, True)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, l_ref)
    # and it is close to the unquantised attention (E4M3 keeps 3 mantissa bits)
    o16, _ = oracle_mod.attention(q, k, v, 0.2, True)
    assert np.abs(o - o16).max() < 0.1


# ---------------------------------------------------------------- backward pass
def _bwd_inputs(B, H, Nq, Nkv, d, seed, dtype=torch.float64):
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.float32, seed)
    g = randn((B, H, Nq, d), seed + 3, torch.float32)
    return q.to(dtype), k.to(dtype), v.to(dtype), g.to(dtype)


@pytest.mark.parametrize("causal,Nq,Nkv", [(False, 6, 9), (True, 6, 9), (True, 9, 9),
                                           (False, 9, 4)])
def test_backward_matches_autograd_of_the_definition(oracle_mod, causal, Nq, Nkv):
    """torch autograd (fp64) of softmax(scale Q K^T + mask) V, a library derivation of the
    same gradients, agrees with the written-out formulas."""
    B, H, d = 2, 2, 5
    q, k, v, g = _bwd_inputs(B, H, Nq, Nkv, d, 41)
    scale = 0.37
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    s = scale * qa @ ka.transpose(-1, -2)
    if causal:
        s = s.masked_fill(~torch.from_numpy(_visible_mask(Nq, Nkv, True)), float("-inf"))
    (torch.softmax(s, dim=-1) @ va).backward(g)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, scale, causal)
    for ours, ref in ((dq, qa.grad), (dk, ka.grad), (dv, va.grad)):
        np.testing.assert_allclose(ours, ref.numpy(), rtol=0, atol=1e-12)


def test_backward_matches_finite_differences_of_the_forward_oracle(oracle_mod):
    """Central differences of L = sum(dO * O), O from the C forward oracle, against the
    backward formulas: every element of Q, K and V on a tiny causal case with Nq != Nkv."""
    B, H, Nq, Nkv, d = 1, 2, 3, 4, 3
    q, k, v, g = _bwd_inputs(B, H, Nq, Nkv, d, 57)
    scale, eps = 0.61, 1e-6
    gf = _f64(g)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, scale, True)

    def loss(qq, kk, vv):
        o, _ = oracle_mod.attention(qq, kk, vv, scale, True)
        return float((o * gf).sum())

    for which, grad in ((0, dq), (1, dk), (2, dv)):
        base = [q.clone(), k.clone(), v.clone()]
        t = base[which]
        for idx in np.ndindex(*t.shape):
            plus = [x.clone() for x in base]
            minus = [x.clone() for x in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert grad[idx] == pytest.approx(fd, abs=1e-7), (which, idx)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_column_sums(oracle_mod, causal):
    """Rows of P sum to 1, so the dV rows sum to the dO rows summed over queries; rows of
    dS sum to 0, so the dK rows sum to zero.  (Causal with Nq <= Nkv: every query sees a
    key.)  A dropped D term or an unnormalised P breaks one of these."""
    B, H, Nq, Nkv, d = 2, 3, 21, 33, 8
    q, k, v, g = _bwd_inputs(B, H, Nq, Nkv, d, 63)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, 0.3, causal)
    np.testing.assert_allclose(dv.sum(axis=2), _f64(g).sum(axis=2), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, rtol=0, atol=1e-11)


def test_backward_key_shift_invariance(oracle_mod):
    """Adding one vector c to every key adds q_i . c to a whole row of scores, which the
    softmax ignores: dQ, dK and dV do not change."""
    B, H, Nq, Nkv, d = 1, 2, 13, 17, 6
    q, k, v, g = _bwd_inputs(B, H, Nq, Nkv, d, 71)
    c = torch.linspace(-1.0, 2.0, d, dtype=torch.float64)
    a = oracle_mod.attention_backward(q, k, v, g, 0.45, True)
    b = oracle_mod.attention_backward(q, k + c, v, g, 0.45, True)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-11)


def test_backward_uniform_attention_closed_form(oracle_mod):
    """K = 0 makes every score 0 and P = 1/Nkv: then dV_j = sum_i dO_i / Nkv,
    dQ = 0, and dK_j = scale/Nkv * sum_i (dO_i . (V_j - mean V)) Q_i."""
    B, H, Nq, Nkv, d = 1, 1, 7, 5, 4
    q, _, v, g = _bwd_inputs(B, H, Nq, Nkv, d, 83)
    k = torch.zeros(B, H, Nkv, d, dtype=torch.float64)
    scale = 0.8
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, scale, False)
    Q, V, G = _f64(q)[0, 0], _f64(v)[0, 0], _f64(g)[0, 0]
    np.testing.assert_allclose(dq, 0.0, atol=0)
    np.testing.assert_allclose(dv[0, 0], np.tile(G.sum(axis=0) / Nkv, (Nkv, 1)), atol=1e-13)
    vbar = V.mean(axis=0)
    for j in range(Nkv):
        ref = sum(scale / Nkv * float(G[i] @ (V[j] - vbar)) * Q[i] for i in range(Nq))
        np.testing.assert_allclose(dk[0, 0, j], ref, atol=1e-13)


def test_backward_single_key_and_masked_rows(oracle_mod):
    """One key: P = 1, so dV = sum of dO and dS = 0 (dQ = dK = 0).  Causal with Nq > Nkv:
    the first Nq - Nkv queries see no key and get dQ = 0; the rest equal the gradient of
    the visible block alone."""
    q, k, v, g = _bwd_inputs(1, 2, 6, 1, 4, 91)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, 0.5, False)
    np.testing.assert_allclose(dv[:, :, 0], _f64(g).sum(axis=2), atol=1e-13)
    assert np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13
    q, k, v, g = _bwd_inputs(1, 2, 9, 5, 4, 97)
    dq, dk, dv = oracle_mod.attention_backward(q, k, v, g, 0.5, True)
    assert np.all(dq[:, :, :4] == 0)
    sub = oracle_mod.attention_backward(q[:, :, 4:], k, v, g[:, :, 4:], 0.5, True)
    np.testing.assert_allclose(dq[:, :, 4:], sub[0], atol=1e-13)
    np.testing.assert_allclose(dk, sub[1], atol=1e-13)
    np.testing.assert_allclose(dv, sub[2], atol=1e-13)


def test_backward_heads_subset(oracle_mod):
    q, k, v, g = _bwd_inputs(2, 2, 5, 7, 3, 101)
    full = oracle_mod.attention_backward(q, k, v, g, 0.4, True)
    part = oracle_mod.attention_backward(q, k, v, g, 0.4, True, heads=[2])
    for x, y in zip(full, part):
        np.testing.assert_array_equal(x[1, 0], y[1, 0])
        assert np.all(y[0] == 0) and np.all(y[1, 1] == 0)

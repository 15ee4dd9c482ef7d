"""The benchmark's FLOP counts against brute force: visible (query, key) pairs under the
bottom-right causal mask, 4·d FLOP per pair forward and 10·d per pair backward."""
import numpy as np
import pytest
import torch

import bench
from exact_io_aware_59_b200.inputs import WORKLOADS, Workload


def _brute_pairs(Nq, Nkv):
    i = np.arange(Nq)[:, None]
    j = np.arange(Nkv)[None, :]
    return int((j <= i + (Nkv - Nq)).sum())


@pytest.mark.parametrize("Nq,Nkv", [(1, 1), (1, 7), (7, 1), (5, 5), (13, 40), (40, 13), (128, 128),
                                    (200, 130), (130, 200), (1, 32768), (3, 2)])
def test_causal_pairs_is_the_visible_count(Nq, Nkv):
    assert bench.causal_pairs(Nq, Nkv) == _brute_pairs(Nq, Nkv)


def test_causal_pairs_random_shapes():
    rng = np.random.default_rng(7)
    for _ in range(200):
        Nq, Nkv = (int(x) for x in rng.integers(1, 300, size=2))
        assert bench.causal_pairs(Nq, Nkv) == _brute_pairs(Nq, Nkv)


def test_flops_of_the_headline_shape():
    w = WORKLOADS["long_prefill_causal"]
    pairs = 8192 * 8193 // 2
    assert bench.attention_flops(w) == 4 * 128 * 32 * pairs == 549822922752
    assert bench.backward_flops(w) == 10 * 128 * 32 * pairs
    wn = WORKLOADS["long_prefill"]
    assert bench.attention_flops(wn) == 4 * 128 * 32 * 8192 * 8192


def test_backward_is_two_and_a_half_forwards():
    w = Workload("x", 9, 2, 3, 37, 53, 64, torch.bfloat16, True)
    assert 2 * bench.backward_flops(w) == 5 * bench.attention_flops(w)


def test_decode_algorithmic_bytes():
    """Q, K, V read once and O (16-bit) and LSE written once: the decode roofline's unit."""
    w = WORKLOADS["decode"]
    BH = 16 * 32
    expect = BH * (128 * 2 + 2 * 32768 * 128 * 2 + 128 * 2 + 4)
    assert bench.algorithmic_bytes(w, 2) == expect == 8590198784

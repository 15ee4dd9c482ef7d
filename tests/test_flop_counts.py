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


def test_bench_line_keeps_every_config_in_its_last_1500_characters():
    """The per-config records go last in the printed line and stay short enough that the
    end of the line (what a log tail keeps) holds every one of them."""
    import json

    clk = {"sm_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    names = ["mha_d64", "noncausal_8k", "peaky_8k", "causal_16k", "causal_32k", "decode",
             "decode_paged", "fp8_8k", "fp8q_8k", "bwd_8k", "varlen"]
    configs = {n: bench.compact(1234.56789, "TFLOP/s", 0.123456789, 2000, 0.6789012,
                                0.7890123, clk) for n in names}
    line = {"metric": bench.METRIC, "value": 1.0, "configs": configs}
    tail = json.dumps(line, separators=(",", ":"))[-1500:]
    for n in names:
        assert f'"{n}":' in tail, n

"""Plants plausible mistakes in copies of the oracle's C source (on the CPU) and checks
that the pins catch every one: a dropped term, a wrong sign or index, a transposed
operand, a misaligned mask, a wrong 16-bit decode."""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

from exact_io_aware_59_b200.inputs import make_qkv

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "attn_oracle.c")

MUTANTS = {
    "scale_dropped": ("s[j] = J->scale * acc;", "s[j] = acc;"),
    "mask_top_left": ("int64_t lim = i + (Nkv - Nq);", "int64_t lim = i;"),
    "mask_off_by_one_low": ("int64_t lim = i + (Nkv - Nq);", "int64_t lim = i + (Nkv - Nq) - 1;"),
    "mask_off_by_one_high": ("int64_t lim = i + (Nkv - Nq);", "int64_t lim = i + (Nkv - Nq) + 1;"),
    "max_sign": ("s[j] = exp(s[j] - m);", "s[j] = exp(s[j] + m);"),
    "lse_without_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "v_is_k": ("out[c] += p * elem(J->v,", "out[c] += p * elem(J->k,"),
    "kv_offset_uses_nq": ("const size_t kv0 = (size_t)(bh * Nkv * d);",
                          "const size_t kv0 = (size_t)(bh * Nq * d);"),
    "q_row_of_first_head": ("elem(J->q, J->dtype, (size_t)(grow * d + c))",
                            "elem(J->q, J->dtype, (size_t)(i * d + c))"),
    "k_transposed": ("acc += qrow[c] * elem(J->k, J->dtype, kv0 + (size_t)(j * d + c));",
                     "acc += qrow[c] * elem(J->k, J->dtype, kv0 + (size_t)(c * d + j % d));"),
    "half_exponent_bias": ("r = ldexp((double)(man + 1024), e - 25);",
                           "r = ldexp((double)(man + 1024), e - 24);"),
    "half_subnormal": ("r = ldexp((double)man, -24);", "r = ldexp((double)man, -25);"),
    "bf16_shift": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    "no_normalisation": ("const double p = s[j] / l;", "const double p = s[j];"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           str(path), "-o", str(so), "-lm"])
    return str(so)


def _pins_hold(oracle_mod, lib):
    """A compact version of the pins in test_oracle.py; True when all of them hold."""
    def run(q, k, v, scale, causal):
        return oracle_mod.attention(q, k, v, scale, causal, lib=lib)

    # brute force, several heads, Nq != Nkv both ways, both 16-bit types
    for (B, H, Nq, Nkv, d), dtype in [((1, 2, 9, 23, 16), torch.float16),
                                      ((2, 2, 23, 9, 16), torch.bfloat16),
                                      ((1, 3, 17, 17, 32), torch.float16)]:
        for causal in (False, True):
            q, k, v = make_qkv(B, H, Nq, Nkv, d, dtype, 3 + d)
            o, lse = run(q, k, v, 1 / math.sqrt(d), causal)
            qf, kf, vf = (t.double().numpy() for t in (q, k, v))
            i = np.arange(Nq)[:, None]
            j = np.arange(Nkv)[None, :]
            mask = (j <= i + Nkv - Nq) if causal else np.ones((Nq, Nkv), bool)
            s = np.einsum("bhic,bhjc->bhij", qf, kf) / math.sqrt(d)
            e = np.where(mask, np.exp(s), 0)
            z = e.sum(-1)
            ob = np.einsum("bhij,bhjc->bhic", e / np.where(z > 0, z, 1)[..., None], vf)
            with np.errstate(divide="ignore"):
                lb = np.where(z > 0, np.log(np.where(z > 0, z, 1)), -np.inf)
            if not np.allclose(o, ob, rtol=0, atol=1e-12):
                return False
            if not np.array_equal(np.isneginf(lse), np.isneginf(lb)):
                return False
            fin = np.isfinite(lb)
            if not np.allclose(lse[fin], lb[fin], rtol=0, atol=1e-12):
                return False
    # 16-bit decoding: subnormal and extreme fp16 values against the fp64 path
    special = torch.tensor([6.0e-8, -1.0e-5, 65504.0, 0.333], dtype=torch.float16)
    q, k, v = make_qkv(1, 1, 4, 6, 8, torch.float16, 9)
    v.view(-1)[:4] = special
    o16, _ = run(q, k, v, 0.1, False)
    o64, _ = run(q.double(), k.double(), v.double(), 0.1, False)
    return bool(np.array_equal(o16, o64))


def test_unmutated_oracle_passes_compact_pins(oracle_mod):
    assert _pins_hold(oracle_mod, None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(oracle_mod, tmp_path, name):
    old, new = MUTANTS[name]
    lib = oracle_mod.load_library(_build_mutant(tmp_path, name, old, new))
    assert not _pins_hold(oracle_mod, lib), f"mutant {name} survived the pins"

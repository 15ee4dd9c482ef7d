"""Derives the coefficients of the FMA-pipe exp2 used by the prefill softmax.

2^x = 2^j * 2^f with j = round(x) and f in [-1/2, 1/2]; 2^f is approximated by the
degree-4 polynomial c0 + c1 f + ... + c4 f^4 that minimises the maximum relative error on
a dense grid of [-1/2, 1/2], found by linear programming (minimise t subject to
|p(f_i) / 2^f_i - 1| <= t).  The result, rounded to fp32, is what csrc/fa_device.cuh uses
(kExp2C0..kExp2C4); tests/test_exp2_poly.py re-derives it and checks the two agree.

    python -m exact_io_aware_59_b200.exp2_poly
"""
from __future__ import annotations

import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc", "fa_device.cuh")


def minimax_coefficients(degree: int = 4, points: int = 4001):
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    n = degree + 1
    A = np.vstack([f ** k for k in range(n)]).T / y[:, None]
    ones = np.ones((len(f), 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([np.ones(len(f)), -np.ones(len(f))])
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (n + 1), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return res.x[:n].astype(np.float32), float(res.x[-1])


def header_coefficients():
    text = open(HEADER).read()
    vals = dict(re.findall(r"constexpr float kExp2C(\d) = ([0-9.eE+-]+)f;", text))
    return np.array([float(vals[str(k)]) for k in range(len(vals))], dtype=np.float32)


def exp2_emulated(x, c):
    """The device routine step by step in float32 (clamp, magic-number rounding, Horner,
    exponent add) for checking on the host."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + np.float32(c[k])).astype(np.float32)
    bits = (t.view(np.uint32).astype(np.uint64) * (1 << 23) + p.view(np.uint32)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, err = minimax_coefficients()
    print("coefficients (fp32):", [float(v) for v in c], "max relative error", err)

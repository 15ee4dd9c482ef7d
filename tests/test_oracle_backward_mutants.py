"""Plants plausible mistakes in copies of the backward oracle (oracle.attention_backward,
on the CPU) and checks that its pins catch every one: a dropped term, a wrong sign, a
wrong operand, a missing scale, an unnormalised softmax, a misaligned mask."""
import inspect
import textwrap

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_59_b200.inputs import make_qkv, randn

MUTANTS = {
    "drop_D": ("dS = P * (dP - D)", "dS = P * dP"),
    "dS_sign": ("dS = P * (dP - D)", "dS = P * (D - dP)"),
    "D_without_P": ("D = (P * dP).sum(axis=1, keepdims=True)", "D = dP.sum(axis=1, keepdims=True)"),
    "dq_without_scale": ("dq[b, h] = scale * (dS @ K)", "dq[b, h] = dS @ K"),
    "dq_uses_V": ("dq[b, h] = scale * (dS @ K)", "dq[b, h] = scale * (dS @ V)"),
    "dk_uses_P": ("dk[b, h] = scale * (dS.T @ Q)", "dk[b, h] = scale * (P.T @ Q)"),
    "dv_uses_dS": ("dv[b, h] = P.T @ G", "dv[b, h] = (P * (G @ V.T)).T @ G"),
    "unnormalised": ("P = e / np.where(z > 0, z, 1.0)", "P = e"),
    "mask_top_left": ("np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)",
                      "np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None]"),
    "mask_off_by_one": ("np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)",
                        "np.arange(Nkv)[None, :] < np.arange(Nq)[:, None] + (Nkv - Nq)"),
}


def _mutant(old, new):
    src = textwrap.dedent(inspect.getsource(oracle.attention_backward))
    assert src.count(old) == 1, old
    ns = {"np": np, "_f64": oracle._f64}
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["attention_backward"]


def _inputs(B, H, Nq, Nkv, d, seed):
    q, k, v = make_qkv(B, H, Nq, Nkv, d, torch.float32, seed)
    g = randn((B, H, Nq, d), seed + 3, torch.float32)
    return q.double(), k.double(), v.double(), g.double()


def _pin_autograd(f):
    for causal, Nq, Nkv in ((True, 6, 9), (False, 9, 4)):
        q, k, v, g = _inputs(1, 2, Nq, Nkv, 5, 41)
        qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
        s = 0.37 * qa @ ka.transpose(-1, -2)
        if causal:
            vis = np.arange(Nkv)[None, :] <= np.arange(Nq)[:, None] + (Nkv - Nq)
            s = s.masked_fill(~torch.from_numpy(vis), float("-inf"))
        (torch.softmax(s, dim=-1) @ va).backward(g)
        ours = f(q, k, v, g, 0.37, causal)
        for x, r in zip(ours, (qa.grad, ka.grad, va.grad)):
            if not np.allclose(x, r.numpy(), rtol=0, atol=1e-10):
                return False
    return True


def _pin_finite_differences(f):
    q, k, v, g = _inputs(1, 1, 3, 4, 2, 57)
    scale, eps = 0.61, 1e-6
    grads = f(q, k, v, g, scale, True)
    gf = g.numpy()

    def loss(qq, kk, vv):
        o, _ = oracle.attention(qq, kk, vv, scale, True)
        return float((o * gf).sum())

    for which in range(3):
        base = [q.clone(), k.clone(), v.clone()]
        for idx in np.ndindex(*base[which].shape):
            plus = [x.clone() for x in base]
            minus = [x.clone() for x in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            if abs(grads[which][idx] - (loss(*plus) - loss(*minus)) / (2 * eps)) > 1e-6:
                return False
    return True


def _pin_column_sums(f):
    q, k, v, g = _inputs(1, 2, 7, 11, 4, 63)
    for causal in (False, True):
        dq, dk, dv = f(q, k, v, g, 0.3, causal)
        if not (np.allclose(dv.sum(axis=2), g.numpy().sum(axis=2), atol=1e-11)
                and np.allclose(dk.sum(axis=2), 0.0, atol=1e-11)):
            return False
    return True


def _pin_uniform(f):
    q, _, v, g = _inputs(1, 1, 5, 4, 3, 83)
    k = torch.zeros(1, 1, 4, 3, dtype=torch.float64)
    dq, dk, dv = f(q, k, v, g, 0.8, False)
    G, V, Q = g.numpy()[0, 0], v.numpy()[0, 0], q.numpy()[0, 0]
    ref_dk = np.stack([sum(0.8 / 4 * float(G[i] @ (V[j] - V.mean(axis=0))) * Q[i] for i in range(5))
                       for j in range(4)])
    return (np.allclose(dq, 0.0, atol=1e-13) and np.allclose(dv[0, 0], G.sum(axis=0) / 4, atol=1e-13)
            and np.allclose(dk[0, 0], ref_dk, atol=1e-13))


PINS = (_pin_autograd, _pin_finite_differences, _pin_column_sums, _pin_uniform)


def _caught(f):
    for pin in PINS:
        try:
            if not pin(f):
                return pin.__name__
        except Exception as e:  # a shape error is a catch too
            return f"{pin.__name__} raised {type(e).__name__}"
    return None


def test_unmutated_backward_oracle_passes_every_pin():
    assert _caught(oracle.attention_backward) is None


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_pins_catch_mutant(name):
    old, new = MUTANTS[name]
    assert _caught(_mutant(old, new)) is not None, f"mutant {name} passed every pin"

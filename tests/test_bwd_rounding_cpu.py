"""The backward pass's rounding scheme, emulated in numpy on the CPU.

The kernels round their MMA operands to bf16 (the inputs q, k, v, dO are
bf16 already; the squares and dS are rounded where they are formed) and take
the difference dO.v - dO.o in fp32 before scaling by 1/D.  This test applies
the same roundings to a case with tiny denominators and checks the result
against the fp64 gradient oracle: that scheme stays inside the 2e-2 gate,
while rounding dN = dO / D to bf16 before the dP product (an earlier design)
does not.  No GPU is involved; the kernels' own parity tests are in
tests/test_bwd_gpu.py.
"""
import numpy as np

import workloads
from oracle import backward as obw

rb = workloads.round_bf16


def _forward(q, k, v, mask):
    S = np.einsum("bhtp,bhsp->bhts", q, k).astype(np.float32)
    W = np.where(mask, rb((S * S).astype(np.float32)), 0)
    N = np.einsum("bhts,bhse->bhte", W, v).astype(np.float32)
    D = W.sum(-1).astype(np.float32)
    o = rb((N / D[..., None]).astype(np.float32))
    return S, D, o


def _grads_fp32_cancellation(q, k, v, dO):
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    S, D, o = _forward(q, k, v, mask)
    delta = np.einsum("bhte,bhte->bht", dO, o).astype(np.float32)
    r = np.where(D > 0, 2 / D, 0).astype(np.float32)
    dP = np.einsum("bhte,bhse->bhts", dO, v).astype(np.float32)
    u = S * r[..., None]
    dS = np.where(mask, rb((u * (dP - delta[..., None])).astype(np.float32)), 0)
    Wp = np.where(mask, rb((S * u).astype(np.float32)), 0)
    return (np.einsum("bhts,bhsp->bhtp", dS, k), np.einsum("bhts,bhtp->bhsp", dS, q),
            0.5 * np.einsum("bhts,bhte->bhse", Wp, dO))


def _grads_rounded_dn(q, k, v, dO):
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    S, D, o = _forward(q, k, v, mask)
    dN = rb((dO / D[..., None]).astype(np.float32))
    dD = (-np.einsum("bhte,bhte->bht", dO, o) / D).astype(np.float32)
    dP = np.einsum("bhte,bhse->bhts", dN, v).astype(np.float32)
    dS = np.where(mask, rb((2 * S * (dP + dD[..., None])).astype(np.float32)), 0)
    return np.einsum("bhts,bhsp->bhtp", dS, k), np.einsum("bhts,bhtp->bhsp", dS, q)


def _err(g, r):
    return max(np.linalg.norm(g[0, h] - r[0, h]) / np.linalg.norm(r[0, h]) for h in range(g.shape[1]))


def test_fp32_cancellation_keeps_tiny_denominators_inside_the_gate():
    q, k, v = workloads.normal_qkv(1, 2, 300, 16, 64, seed=0, dtype="bf16")
    dO = rb(np.random.default_rng(3).standard_normal(v.shape).astype(np.float32))
    ref = obw.backward(q, k, v, dO)
    _, D, _ = _forward(q, k, v, np.tril(np.ones((300, 300), dtype=bool)))
    assert D.min() < 1e-5  # this seeded input has a row with a tiny denominator
    got = _grads_fp32_cancellation(q, k, v, dO)
    assert max(_err(g, r) for g, r in zip(got, ref)) < 2e-2
    old = _grads_rounded_dn(q, k, v, dO)
    assert max(_err(g, r) for g, r in zip(old, ref[:2])) > 0.1

"""fp64 gradients of the KATA forward pass (test infrastructure only).

Only the test suite and the benchmark's CPU leg may import this module; it
shares nothing with the CUDA path.

For one (batch, head) pair, with S_ts = q_t . k_s, w_ts = S_ts^2 (s <= t),
N_t = sum_s w_ts v_s, D_t = sum_s w_ts and o_t = N_t / D_t (o_t = 0 when
D_t = 0) -- the operation of the gist.science technical summary, sec. 2.1
"Output Gating" and sec. 2.2 "PSD Kegel (Rank-One)" -- the gradients of a
loss with upstream gradient dO follow by the chain rule:

    dN_t  = dO_t / D_t                   dD_t = -(dO_t . o_t) / D_t
    dw_ts = dN_t . v_s + dD_t            (s <= t)
    dv_s  = sum_{t >= s} w_ts dN_t
    dS_ts = 2 S_ts dw_ts
    dq_t  = sum_{s <= t} dS_ts k_s       dk_s = sum_{t >= s} dS_ts q_t

and a row with D_t = 0 (its output is the constant 0) passes no gradient.
The pages print no backward pass; this is the derivative of the forward
they define, written out step by step (the pages claim the kernels are
competitive on the training step: arXiv abstract).
"""
from __future__ import annotations

import numpy as np


def forward_with_d(q, k, v):
    """o [B,H,T,dv] and D [B,H,T] in fp64 by the defining sums (T x T matrices)."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    S = np.einsum("bhtp,bhsp->bhts", q, k)
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    W = np.where(mask, S * S, 0.0)
    N = np.einsum("bhts,bhse->bhte", W, v)
    D = W.sum(axis=-1)
    safe = np.where(D > 0, D, 1.0)
    o = np.where((D > 0)[..., None], N / safe[..., None], 0.0)
    return o, D


def backward(q, k, v, dO):
    """(dq, dk, dv) in fp64 for the upstream gradient dO [B,H,T,dv]."""
    q, k, v, dO = (np.asarray(x, np.float64) for x in (q, k, v, dO))
    o, D = forward_with_d(q, k, v)
    live = D > 0
    safe = np.where(live, D, 1.0)
    dN = np.where(live[..., None], dO / safe[..., None], 0.0)
    dD = np.where(live, -np.einsum("bhte,bhte->bht", dO, o) / safe, 0.0)
    S = np.einsum("bhtp,bhsp->bhts", q, k)
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    W = np.where(mask, S * S, 0.0)
    dW = np.where(mask, np.einsum("bhte,bhse->bhts", dN, v) + dD[..., None], 0.0)
    dv = np.einsum("bhts,bhte->bhse", W, dN)
    dS = 2.0 * S * dW
    dq = np.einsum("bhts,bhsp->bhtp", dS, k)
    dk = np.einsum("bhts,bhtp->bhsp", dS, q)
    return dq, dk, dv


def forward_mg_with_d(q, k, v, groups: int):
    """KATA-Mg forward (g PSD factors over a head of width d, weight
    sum_j (q_t^j . k_s^j)^2) with its denominators, fp64, T x T matrices."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    d = q.shape[-1]
    p = d // groups
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    W = np.zeros(q.shape[:2] + (T, T))
    for j in range(groups):
        Sj = np.einsum("bhtp,bhsp->bhts", q[..., j * p:(j + 1) * p], k[..., j * p:(j + 1) * p])
        W += Sj * Sj
    W = np.where(mask, W, 0.0)
    N = np.einsum("bhts,bhse->bhte", W, v)
    D = W.sum(axis=-1)
    safe = np.where(D > 0, D, 1.0)
    o = np.where((D > 0)[..., None], N / safe[..., None], 0.0)
    return o, D


def backward_mg(q, k, v, dO, groups: int):
    """(dq, dk, dv) of the KATA-Mg forward, fp64: the single-factor chain rule
    with w = sum_j S_j^2, so dS_j = 2 S_j dw and each group's dq^j, dk^j come
    from its own scores."""
    q, k, v, dO = (np.asarray(x, np.float64) for x in (q, k, v, dO))
    d = q.shape[-1]
    p = d // groups
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    o, D = forward_mg_with_d(q, k, v, groups)
    live = D > 0
    safe = np.where(live, D, 1.0)
    dN = np.where(live[..., None], dO / safe[..., None], 0.0)
    dD = np.where(live, -np.einsum("bhte,bhte->bht", dO, o) / safe, 0.0)
    dW = np.where(mask, np.einsum("bhte,bhse->bhts", dN, v) + dD[..., None], 0.0)
    W = np.zeros(q.shape[:2] + (T, T))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    for j in range(groups):
        sl = slice(j * p, (j + 1) * p)
        Sj = np.einsum("bhtp,bhsp->bhts", q[..., sl], k[..., sl])
        W += np.where(mask, Sj * Sj, 0.0)
        dSj = 2.0 * Sj * dW
        dq[..., sl] = np.einsum("bhts,bhsp->bhtp", dSj, k[..., sl])
        dk[..., sl] = np.einsum("bhts,bhtp->bhsp", dSj, q[..., sl])
    dv = np.einsum("bhts,bhte->bhse", W, dN)
    return dq, dk, dv


def forward_sg_with_d(q, k, v, groups: int):
    """KATA-Sigma-g forward (weight sum_{j,l} (q_t^j . k_s^l)^2, every query
    group against every key group) with its denominators, fp64."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    d = q.shape[-1]
    p = d // groups
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    W = np.zeros(q.shape[:2] + (T, T))
    for j in range(groups):
        for l in range(groups):
            S = np.einsum("bhtp,bhsp->bhts", q[..., j * p:(j + 1) * p], k[..., l * p:(l + 1) * p])
            W += S * S
    W = np.where(mask, W, 0.0)
    N = np.einsum("bhts,bhse->bhte", W, v)
    D = W.sum(axis=-1)
    safe = np.where(D > 0, D, 1.0)
    o = np.where((D > 0)[..., None], N / safe[..., None], 0.0)
    return o, D


def backward_sg(q, k, v, dO, groups: int):
    """(dq, dk, dv) of the KATA-Sigma-g forward, fp64: the single-factor chain
    rule with w = sum_{j,l} S_jl^2, S_jl = q^j . k^l, so dS_jl = 2 S_jl dw;
    dq^j sums over the key groups l, dk^l over the query groups j."""
    q, k, v, dO = (np.asarray(x, np.float64) for x in (q, k, v, dO))
    d = q.shape[-1]
    p = d // groups
    T = q.shape[2]
    mask = np.tril(np.ones((T, T), dtype=bool))
    o, D = forward_sg_with_d(q, k, v, groups)
    live = D > 0
    safe = np.where(live, D, 1.0)
    dN = np.where(live[..., None], dO / safe[..., None], 0.0)
    dD = np.where(live, -np.einsum("bhte,bhte->bht", dO, o) / safe, 0.0)
    dW = np.where(mask, np.einsum("bhte,bhse->bhts", dN, v) + dD[..., None], 0.0)
    W = np.zeros(q.shape[:2] + (T, T))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    for j in range(groups):
        sj = slice(j * p, (j + 1) * p)
        for l in range(groups):
            sl = slice(l * p, (l + 1) * p)
            S = np.einsum("bhtp,bhsp->bhts", q[..., sj], k[..., sl])
            W += np.where(mask, S * S, 0.0)
            dS = 2.0 * S * dW
            dq[..., sj] += np.einsum("bhts,bhsp->bhtp", dS, k[..., sl])
            dk[..., sl] += np.einsum("bhts,bhtp->bhsp", dS, q[..., sj])
    dv = np.einsum("bhts,bhte->bhse", W, dN)
    return dq, dk, dv

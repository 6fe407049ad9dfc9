"""fp64 oracle of KATA-Sigma-g, the summed-factor feature map (test
infrastructure only; shares nothing with the CUDA path).

The head's d coordinates split into g consecutive groups of width p = d/g,
u = [u^1 | ... | u^g], and the feature is the SUM of the group maps,

    psi_S(u) = sum_j vec(u^j u^j^T)                        (p x p, symmetric)
    w_ts = <psi_S(q_t), psi_S(k_s)> = sum_{j,l} (q_t^j . k_s^l)^2

with one value vector and one denominator (arXiv abstract and gist.science
sec. 2.3 "Varianten": KATA-Sigma-g, summed PSD factors; ai.info summary, Main
Findings: state (d/g)(d/g+1)/2 * dv, the full map at g = 1).  Two forms: the
defining double sum, and the recurrence on the explicit p^2 feature; and one
step of that recurrence from a given state (decode).
"""
from __future__ import annotations

import numpy as np


def _groups(x, groups):
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    if groups < 1 or d % groups:
        raise ValueError("groups must divide the head width")
    return x.reshape(x.shape[:-1] + (groups, d // groups))


def direct_sg(q, k, v, groups: int):
    """o [B,H,T,dv] from w_ts = sum_{j,l} (q_t^j . k_s^l)^2, causal, D = 0 -> 0."""
    qg, kg = _groups(q, groups), _groups(k, groups)
    v = np.asarray(v, np.float64)
    T = qg.shape[2]
    # dots[b,h,t,s,j,l] = q_t^j . k_s^l
    dots = np.einsum("bhtjp,bhslp->bhtsjl", qg, kg)
    W = np.where(np.tril(np.ones((T, T), dtype=bool)), (dots * dots).sum(axis=(-1, -2)), 0.0)
    N = np.einsum("bhts,bhse->bhte", W, v)
    D = W.sum(axis=-1)
    safe = np.where(D > 0, D, 1.0)
    return np.where((D > 0)[..., None], N / safe[..., None], 0.0)


def features_sg(u, groups: int):
    """psi_S(u) = sum_j vec(u^j u^j^T), [..., p*p]."""
    ug = _groups(u, groups)
    p = ug.shape[-1]
    return np.einsum("...ja,...jb->...ab", ug, ug).reshape(ug.shape[:-2] + (p * p,))


def recurrent_sg(q, k, v, groups: int):
    """The same output through the state S_t = S_{t-1} + psi_S(k_t) v_t^T,
    z_t = z_{t-1} + psi_S(k_t), o_t = psi_S(q_t)^T S_t / psi_S(q_t)^T z_t."""
    fq, fk = features_sg(q, groups), features_sg(k, groups)
    v = np.asarray(v, np.float64)
    B, H, T, P = fk.shape
    o = np.zeros(v.shape)
    S = np.zeros((B, H, P, v.shape[-1]))
    z = np.zeros((B, H, P))
    for t in range(T):
        S += fk[:, :, t, :, None] * v[:, :, t, None, :]
        z += fk[:, :, t]
        num = np.einsum("bhp,bhpe->bhe", fq[:, :, t], S)
        den = np.einsum("bhp,bhp->bh", fq[:, :, t], z)
        safe = np.where(den > 0, den, 1.0)
        o[:, :, t] = np.where((den > 0)[..., None], num / safe[..., None], 0.0)
    return o


def decode_step_sg(q, k, v, S, z, groups: int):
    """One recurrent step on the summed-feature state: S' = S + psi_S(k) v^T,
    z' = z + psi_S(k), o = psi_S(q)^T S' / psi_S(q)^T z' (0 where that is 0).

    q, k [B,H,d]; v [B,H,dv]; S [B,H,p*p,dv], z [B,H,p*p] with p = d/groups
    (row a*p + b holds sum_j u^j_a u^j_b).  Returns (o, S', z')."""
    fq, fk = features_sg(q, groups), features_sg(k, groups)
    v = np.asarray(v, np.float64)
    S2 = np.asarray(S, np.float64) + fk[..., :, None] * v[..., None, :]
    z2 = np.asarray(z, np.float64) + fk
    num = np.einsum("bhp,bhpe->bhe", fq, S2)
    den = np.einsum("bhp,bhp->bh", fq, z2)
    safe = np.where(den > 0, den, 1.0)
    return np.where((den > 0)[..., None], num / safe[..., None], 0.0), S2, z2

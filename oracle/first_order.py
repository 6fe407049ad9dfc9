"""fp64 oracle of first-order (linear) attention, the feature psi(u) = u
(test infrastructure only; shares nothing with the CUDA path and never
calls it).

    o_t = sum_{s<=t} (q_t . k_s) v_s / sum_{s<=t} (q_t . k_s)

This is the comparator of the pages' scan claim: an associative scan of the
first-order feature lowers the inter-chunk recurrence depth to O(log(T/C))
and averages ~2.4x the throughput of a matched sequential linear-attention
baseline (arXiv abstract; review page, Figure 3 caption; gist.science
sec. 2.3).  It is the KATA recurrence (ai.info summary, Methodology in Plain
English) with psi(u) = u in place of vec(u u^T).  Two forms:

* :func:`direct_linear` -- the defining double sum;
* :func:`recurrent_linear` -- the state recurrence
  S_t = S_{t-1} + k_t v_t^T, z_t = z_{t-1} + k_t,
  o_t = q_t^T S_t / q_t^T z_t, with optional initial and final state.

Readings: inclusive causal sum (s <= t), as for the KATA paths; the
denominator is not sign-constrained (u itself is not a nonnegative feature),
so o_t = N_t / D_t for any D_t != 0 and o_t = 0 only where D_t is exactly 0.

Its pins live in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import numpy as np


def _div(N, D):
    nz = D != 0
    safe = np.where(nz, D, 1.0)
    return np.where(nz[..., None], N / safe[..., None], 0.0)


def direct_linear(q, k, v):
    """o [B,H,T,dv] from w_ts = q_t . k_s for s <= t (the double sum)."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    T = q.shape[2]
    W = np.einsum("bhtd,bhsd->bhts", q, k)
    W = np.where(np.tril(np.ones((T, T), dtype=bool)), W, 0.0)
    N = np.einsum("bhts,bhse->bhte", W, v)
    return _div(N, W.sum(axis=-1))


def recurrent_linear(q, k, v, S0=None, z0=None, return_state=False):
    """The same output through the state recurrence, token by token.

    S0 [B,H,d,dv] and z0 [B,H,d] give the state before token 0 (zero when
    omitted); with return_state the state after the last token is returned
    too."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    B, H, T, d = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, d, dv)) if S0 is None else np.array(S0, np.float64)
    z = np.zeros((B, H, d)) if z0 is None else np.array(z0, np.float64)
    o = np.zeros((B, H, T, dv))
    for t in range(T):
        S += k[:, :, t, :, None] * v[:, :, t, None, :]
        z += k[:, :, t]
        N = np.einsum("bhd,bhde->bhe", q[:, :, t], S)
        D = np.einsum("bhd,bhd->bh", q[:, :, t], z)
        o[:, :, t] = _div(N, D)
    if return_state:
        return o, S, z
    return o

"""Seeded synthetic inputs for the KATA forward pass.

This module only draws and shapes random inputs; it holds none of the
method's arithmetic.  Both the oracle tests and the CUDA-path tests and the
benchmark take their inputs from here, so that the two sides see the same
values.

Recipes (shapes follow the pages' workloads: the 340M model's 16 heads at
context 2048 in the KATA repository README, long contexts up to 131k tokens
in the arXiv abstract, and the overwrite task's "each key written twice"
structure in the README's benchmark section):

* ``normal``: q, k ~ N(0, 1) then L2-normalised per token; v ~ N(0, 1).
* ``recall``: keys from a code of ``code_size`` unit vectors (i.i.d. N(0, I)
  normalised); within each block of 2*code_size tokens every codeword appears
  exactly twice at randomly permuted positions (overwrite pattern); query t is
  a noisy copy of an earlier key, normalise(k_s + sigma * N(0, I)) with s
  uniform over 0..t-1 (s = 0 for t = 0); v ~ N(0, 1).

Values are returned as float32 numpy arrays.  For ``dtype="bf16"`` every value
is rounded once to the nearest bfloat16 (ties to even), so the float32 array
holds exactly the values the device sees and the oracle upcasts them exactly.
"""
from __future__ import annotations

import numpy as np

# Configurations used by the tests and the benchmark.  Seeds are the index of
# the configuration in this list.
CONFIGS = {
    "tiny": dict(B=1, H=1, T=256, p=16, dv=16, C=64, dtype="f32", kind="normal", seed=0),
    "layer340m_ctx2k": dict(B=8, H=16, T=2048, p=16, dv=64, C=64, dtype="bf16", kind="normal", seed=1),
    "long_ctx131k": dict(B=1, H=16, T=131072, p=16, dv=64, C=64, dtype="bf16", kind="normal", seed=2),
    "recall_p32": dict(B=4, H=16, T=8192, p=32, dv=64, C=64, dtype="bf16", kind="recall", seed=3),
}

# KATA-Mg configurations: the 340M model's heads (hidden size 1024 over 16
# heads, d = 64) split into `groups` PSD factors -- 2 as in the README's model
# config (spd_num_groups=2, p = 32) and 4 (p = 16) -- at context 2048, in the
# README attention call's [B, T, H, d] layout.  q, k are L2-normalised over
# the whole head row.
MG_CONFIGS = {
    "mg2_ctx2k": dict(B=8, H=16, T=2048, d=64, groups=2, dv=64, dtype="bf16", layout="bthd", seed=5),
    "mg4_ctx2k": dict(B=8, H=16, T=2048, d=64, groups=4, dv=64, dtype="bf16", layout="bthd", seed=6),
}
SWEEP_B = (1, 4, 16)
SWEEP_T = (1024, 4096, 16384, 65536, 131072)
DECODE = dict(B=64, H=16, p=16, dv=64, dtype="bf16", seed=4)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    # keep NaN payloads quiet and unchanged in sign
    nan = np.isnan(x)
    if nan.any():
        out = out.copy()
        out[nan] = np.float32("nan")
    return out


def _cast(x: np.ndarray, dtype: str) -> np.ndarray:
    x = x.astype(np.float32)
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return x
    raise ValueError("dtype must be 'bf16' or 'f32'")


def _l2n(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    n[n == 0] = 1.0
    return (x / n).astype(np.float32)


def normal_qkv(B, H, T, p, dv, seed=0, dtype="bf16"):
    """q, k L2-normalised N(0,1) per token; v ~ N(0,1).  Returns float32 arrays."""
    rng = np.random.default_rng(seed)
    q = _l2n(rng.standard_normal((B, H, T, p), dtype=np.float32))
    k = _l2n(rng.standard_normal((B, H, T, p), dtype=np.float32))
    v = rng.standard_normal((B, H, T, dv), dtype=np.float32)
    return _cast(q, dtype), _cast(k, dtype), _cast(v, dtype)


def nonneg_qkv(B, H, T, p, dv, seed=0, dtype="bf16"):
    """q, k = |N(0,1)| per coordinate, L2-normalised per token (nonnegative
    unit vectors, so every q_t . k_s >= 0); v ~ N(0,1).  Inputs for the
    first-order feature, whose denominators are only sign-definite on such
    inputs.  Returns float32 arrays."""
    rng = np.random.default_rng(seed)
    q = _l2n(np.abs(rng.standard_normal((B, H, T, p), dtype=np.float32)))
    k = _l2n(np.abs(rng.standard_normal((B, H, T, p), dtype=np.float32)))
    v = rng.standard_normal((B, H, T, dv), dtype=np.float32)
    return _cast(q, dtype), _cast(k, dtype), _cast(v, dtype)


def recall_qkv(B, H, T, p, dv, seed=0, dtype="bf16", code_size=512, sigma=0.05):
    """Recall-shaped keys (overwrite pattern) and noisy-copy queries."""
    rng = np.random.default_rng(seed)
    k = np.empty((B, H, T, p), np.float32)
    q = np.empty((B, H, T, p), np.float32)
    block = 2 * code_size
    for b in range(B):
        for h in range(H):
            code = _l2n(rng.standard_normal((code_size, p), dtype=np.float32))
            idx = np.empty(T, np.int64)
            for start in range(0, T, block):
                n = min(block, T - start)
                perm = rng.permutation(np.repeat(np.arange(code_size), 2))[:n]
                idx[start:start + n] = perm
            k[b, h] = code[idx]
            # query t copies key s, s uniform over 0..t-1 (s = 0 at t = 0)
            t = np.arange(T)
            s = np.floor(rng.random(T) * np.maximum(t, 1)).astype(np.int64)
            noise = sigma * rng.standard_normal((T, p), dtype=np.float32)
            q[b, h] = _l2n(k[b, h][s] + noise)
    v = rng.standard_normal((B, H, T, dv), dtype=np.float32)
    return _cast(q, dtype), _cast(k, dtype), _cast(v, dtype)


def make_inputs(cfg: dict, T=None, B=None):
    """Inputs for a configuration dict (see CONFIGS); T or B may be overridden."""
    B = cfg["B"] if B is None else B
    T = cfg["T"] if T is None else T
    if cfg.get("kind", "normal") == "recall":
        return recall_qkv(B, cfg["H"], T, cfg["p"], cfg["dv"], cfg["seed"], cfg["dtype"])
    return normal_qkv(B, cfg["H"], T, cfg["p"], cfg["dv"], cfg["seed"], cfg["dtype"])


def decode_inputs(B, H, p, dv, seed=4, dtype="bf16"):
    """One decode step's q, k, v [B,H,p|dv] plus a random starting state.

    The starting state is a generic random one with the structure a real
    state has: S [B,H,p*p,dv] is symmetric under the swap of the two psi
    indices (i,j) <-> (j,i), and z [B,H,p*p] is the flattening of a random
    positive-definite p x p matrix G G^T / p + 0.1 I, so psi(q)^T z > 0 for
    every q != 0.  Both are float32.
    """
    rng = np.random.default_rng(seed)
    q = _cast(_l2n(rng.standard_normal((B, H, p), dtype=np.float32)), dtype)
    k = _cast(_l2n(rng.standard_normal((B, H, p), dtype=np.float32)), dtype)
    v = _cast(rng.standard_normal((B, H, dv), dtype=np.float32), dtype)
    A = rng.standard_normal((B, H, p, p, dv), dtype=np.float32)
    S = (0.5 * (A + A.transpose(0, 1, 3, 2, 4))).reshape(B, H, p * p, dv).astype(np.float32)
    G = rng.standard_normal((B, H, p, p)).astype(np.float64)
    Z = np.matmul(G, G.transpose(0, 1, 3, 2)) / p + 0.1 * np.eye(p)
    z = Z.reshape(B, H, p * p).astype(np.float32)
    return q, k, v, S, z


def decode_inputs_mg(B, H, d, groups, dv, seed=7, dtype="bf16"):
    """One KATA-Mg decode step's q, k [B,H,d], v [B,H,dv] and a random
    starting state S [B,H,groups*p*p,dv], z [B,H,groups*p*p] (p = d/groups):
    one block per group, each built as in :func:`decode_inputs` (symmetric in
    the two indices, positive-definite normaliser)."""
    rng = np.random.default_rng(seed)
    p = d // groups
    q = _cast(_l2n(rng.standard_normal((B, H, d), dtype=np.float32)), dtype)
    k = _cast(_l2n(rng.standard_normal((B, H, d), dtype=np.float32)), dtype)
    v = _cast(rng.standard_normal((B, H, dv), dtype=np.float32), dtype)
    Ss, zs = [], []
    for _ in range(groups):
        A = rng.standard_normal((B, H, p, p, dv), dtype=np.float32)
        Ss.append((0.5 * (A + A.transpose(0, 1, 3, 2, 4))).reshape(B, H, p * p, dv))
        Gm = rng.standard_normal((B, H, p, p)).astype(np.float64)
        Z = np.matmul(Gm, Gm.transpose(0, 1, 3, 2)) / p + 0.1 * np.eye(p)
        zs.append(Z.reshape(B, H, p * p))
    S = np.concatenate(Ss, axis=2).astype(np.float32)
    z = np.concatenate(zs, axis=2).astype(np.float32)
    return q, k, v, S, z

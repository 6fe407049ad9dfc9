"""Shared helpers for the parity tests: tolerances, the error metric and
conversions between numpy inputs and device tensors."""
import numpy as np

# Gates on the per-row relative error below: fp32 inputs 1e-4; bf16 inputs
# with fp32 accumulation 2e-2.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def row_rel_err(o, o_ref, v):
    """Max over rows (b,h,t) of ||o_t - o_ref_t||_inf / max(||o_ref_t||_inf, 1e-3 ||v_(b,h)||_inf).

    An elementwise relative error is undefined where the reference output is
    near zero; the floor ties the scale to the values being averaged.
    """
    o = np.asarray(o, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    v = np.asarray(v, np.float64)
    num = np.abs(o - o_ref).max(axis=-1)
    vmax = np.abs(v).reshape(v.shape[0], v.shape[1], -1).max(axis=-1)  # [B,H]
    floor = 1e-3 * vmax[:, :, None]
    den = np.maximum(np.abs(o_ref).max(axis=-1), floor)
    return float((num / den).max())


def rows_rel_err(o_rows, ref_rows, vmax_rows):
    num = np.abs(np.asarray(o_rows, np.float64) - ref_rows).max(axis=-1)
    den = np.maximum(np.abs(ref_rows).max(axis=-1), 1e-3 * vmax_rows)
    return float((num / den).max())


def to_dev(x, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    return t.to(device="cuda", dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)


def to_np(t):
    return t.float().cpu().numpy()


def sample_rows(T, C, n_random, rng):
    """Row indices for sampled parity at long T: random rows plus chunk/tile edges."""
    fixed = [0, 1, C - 1, C, C + 1, 127, 128, 129, T // 2, T - 2, T - 1]
    rnd = rng.integers(0, T, size=n_random).tolist()
    return np.array(sorted({t for t in fixed + rnd if 0 <= t < T}), np.int64)

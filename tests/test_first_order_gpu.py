"""Parity of the first-order (psi(u) = u) chunked forward and its matched
sequential baseline with the fp64 oracle (oracle/first_order.py, pinned in
tests/test_oracle.py), element by element on seeded inputs.

Inputs are nonnegative unit q, k (workloads.nonneg_qkv), where every weight
is >= 0 and the per-row metric of the KATA tests applies; one case with
signed inputs checks each row against a bound derived from the arithmetic
(the denominator may then come close to 0)."""
import numpy as np
import pytest

import workloads
from helpers import TOL, row_rel_err, rows_rel_err, sample_rows, to_dev, to_np
from oracle import first_order as ofo

pytestmark = pytest.mark.gpu

D, DV = 16, 64


@pytest.fixture(scope="module")
def kata():
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return K


def _state_bound(k, v, T):
    # the state is a sum of exact bf16 x bf16 products in fp32: the error of
    # each entry is at most (T + 4) 2^-24 sum_t |k_t| |v_t|
    eps = (T + 4) * 2.0 ** -24
    return eps * np.einsum("bhtd,bhte->bhde", np.abs(k), np.abs(v)), eps * np.abs(k).sum(axis=2)


# T = 1, a ragged chunk, exactly one and a bit more than one 128-token tile,
# one super-chunk per (b,h) (B8 H16 T700), a few (B2 H8 T3000: 8 super-chunks)
# and many (B1 H2 T20000: the scan over 53 records)
@pytest.mark.parametrize("B,H,T", [(1, 1, 1), (2, 3, 77), (1, 2, 128), (1, 2, 129), (8, 16, 700), (2, 8, 3000),
                                   (1, 2, 20000)])
@pytest.mark.parametrize("form", ["scan", "sequential"])
def test_first_order_matches_oracle(kata, B, H, T, form):
    import torch
    q, k, v = workloads.nonneg_qkv(B, H, T, D, DV, seed=700 + T, dtype="bf16")
    o_ref, S_ref, z_ref = ofo.recurrent_linear(q, k, v, return_state=True)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    fn = kata.kata_fwd_linear_chunked if form == "scan" else kata.kata_fwd_linear_chunked_sequential
    o, S, z = fn(qd, kd, vd, return_state=True)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    assert row_rel_err(to_np(o), o_ref, v) <= TOL["bf16"]
    bS, bz = _state_bound(k, v, T)
    assert np.all(np.abs(S.cpu().numpy() - S_ref) <= bS + 1e-6)
    assert np.all(np.abs(z.cpu().numpy() - z_ref) <= bz + 1e-6)


@pytest.mark.parametrize("B,H,T,t0", [(8, 16, 700, 300), (2, 8, 3000, 1100), (1, 2, 20000, 7000)])
def test_first_order_state_in_and_out(kata, B, H, T, t0):
    import torch
    q, k, v = workloads.nonneg_qkv(B, H, T, D, DV, seed=710 + T, dtype="bf16")
    o_ref = ofo.recurrent_linear(q, k, v)
    _, S1, z1 = ofo.recurrent_linear(q[:, :, :t0], k[:, :, :t0], v[:, :, :t0], return_state=True)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    # split on the device: the second part resumes from the first's state
    oa, Sa, za = kata.kata_fwd_linear_chunked(qd[:, :, :t0].contiguous(), kd[:, :, :t0].contiguous(),
                                              vd[:, :, :t0].contiguous(), return_state=True)
    ob = kata.kata_fwd_linear_chunked(qd[:, :, t0:].contiguous(), kd[:, :, t0:].contiguous(),
                                      vd[:, :, t0:].contiguous(), S0=Sa, z0=za)
    torch.cuda.synchronize()
    assert row_rel_err(np.concatenate([to_np(oa), to_np(ob)], axis=2), o_ref, v) <= TOL["bf16"]
    # resume from the oracle's state, in both forms
    S0 = torch.from_numpy(S1.astype(np.float32)).cuda()
    z0 = torch.from_numpy(z1.astype(np.float32)).cuda()
    for fn in (kata.kata_fwd_linear_chunked, kata.kata_fwd_linear_chunked_sequential):
        o2 = fn(qd[:, :, t0:].contiguous(), kd[:, :, t0:].contiguous(), vd[:, :, t0:].contiguous(), S0=S0, z0=z0)
        torch.cuda.synchronize()
        assert row_rel_err(to_np(o2), o_ref[:, :, t0:], v) <= TOL["bf16"]
    assert kata.kata_get_status() == 0


def test_first_order_signed_inputs_within_derived_bound(kata):
    """Signed q, k: each row's error is bounded by the rounding the kernels do
    (the weights and the state copy rounded to bf16, 2^-8 relative each, fp32
    sums) scaled by how far the denominator is from cancelling:
      |o_t - o_ref_t| <= 2^-6 (sum_s |q_t||k_s| |v_s| + |o_ref_t| sum_s |q_t||k_s|) / |D_t|
    with |.| elementwise products summed over coordinates (an upper bound of
    |q_t . k_s|)."""
    import torch
    B, H, T = 2, 4, 1500
    q, k, v = workloads.normal_qkv(B, H, T, D, DV, seed=720, dtype="bf16")
    o_ref = ofo.direct_linear(q, k, v)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    qa, ka, va = np.abs(q).astype(np.float64), np.abs(k).astype(np.float64), np.abs(v).astype(np.float64)
    Wa = np.tril(np.einsum("bhtd,bhsd->bhts", qa, ka))
    Na = np.einsum("bhts,bhse->bhte", Wa, va).max(axis=-1)
    Da = Wa.sum(-1)
    Dt = np.tril(np.einsum("bhtd,bhsd->bhts", q.astype(np.float64), k.astype(np.float64))).sum(-1)
    for fn in (kata.kata_fwd_linear_chunked, kata.kata_fwd_linear_chunked_sequential):
        o = to_np(fn(qd, kd, vd))
        torch.cuda.synchronize()
        err = np.abs(o - o_ref).max(axis=-1)
        bound = 2.0 ** -6 * (Na + np.abs(o_ref).max(axis=-1) * Da) / np.maximum(np.abs(Dt), 1e-30)
        assert np.all(err <= bound + 1e-6)


def test_first_order_full_size_sampled_rows(kata):
    """B1 H16 T131072 (the long-context configuration) in both forms, on
    sampled rows computed one by one from the definition."""
    import torch
    B, H, T = 1, 16, 131072
    q, k, v = workloads.nonneg_qkv(B, H, T, D, DV, seed=730, dtype="bf16")
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    o_scan = to_np(kata.kata_fwd_linear_chunked(qd, kd, vd))
    o_seq = to_np(kata.kata_fwd_linear_chunked_sequential(qd, kd, vd))
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    rng = np.random.default_rng(731)
    rows = sample_rows(T, 64, 24, rng)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    for h in (0, 7, 15):
        ref = np.empty((len(rows), DV))
        for i, t in enumerate(rows):
            w = k64[0, h, :t + 1] @ q64[0, h, t]
            ref[i] = (w @ v64[0, h, :t + 1]) / w.sum()
        vmax = np.full(len(rows), np.abs(v[0, h]).max())
        assert rows_rel_err(o_scan[0, h, rows], ref, vmax) <= TOL["bf16"]
        assert rows_rel_err(o_seq[0, h, rows], ref, vmax) <= TOL["bf16"]


def test_first_order_argument_errors(kata):
    import torch
    from kernelized_feature_map_b200 import _abi
    q = torch.zeros((1, 1, 8, 32), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_abi.KataError) as e:
        kata.kata_fwd_linear_chunked(q, q, v)  # d = 32
    assert e.value.status == _abi.KATA_ERR_UNSUPPORTED
    qf = torch.zeros((1, 1, 8, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(_abi.KataError) as e:
        kata.kata_fwd_linear_chunked_sequential(qf, qf, v.float())  # fp32
    assert e.value.status == _abi.KATA_ERR_UNSUPPORTED

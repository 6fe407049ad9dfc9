"""GPU parity of the KATA-Mg entry points (g PSD factors per head) against
the fp64 Mg oracle on the same seeded inputs: the flash-style forward in both
layouts and the decode step.  Gate as for the single-factor paths: per-row
relative error 2e-2 for bf16 inputs, 1e-4 for fp32 (tests/helpers.py)."""
import numpy as np
import pytest

import oracle
import workloads
from helpers import TOL, row_rel_err, rows_rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kata():
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return K


def _bthd(x):
    return np.ascontiguousarray(np.asarray(x).transpose(0, 2, 1, 3))


def _run_mg(K, q, k, v, groups, layout):
    import torch
    if layout == "bthd":
        o = K.kata_fwd_mg_quadratic(to_dev(_bthd(q), "bf16"), to_dev(_bthd(k), "bf16"), to_dev(_bthd(v), "bf16"),
                                    groups, layout="bthd")
        out = _bthd(to_np(o))
    else:
        o = K.kata_fwd_mg_quadratic(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), groups)
        out = to_np(o)
    torch.cuda.synchronize()
    assert K.kata_get_status() == 0
    return out


MG_SHAPES = [
    # B, H, T, d, groups, dv -- T spans several 128-row tiles and ends ragged
    (2, 2, 1000, 64, 4, 64),
    (1, 3, 777, 64, 2, 64),
    (2, 2, 600, 32, 2, 64),
    (1, 2, 385, 16, 1, 16),
    (1, 1, 129, 32, 1, 64),
]


@pytest.mark.parametrize("layout", ["bhtd", "bthd"])
@pytest.mark.parametrize("shape", MG_SHAPES)
def test_mg_flash_matches_oracle(kata, shape, layout):
    B, H, T, d, g, dv = shape
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=200 + T + g, dtype="bf16")
    ref = oracle.direct_mg(q, k, v, g)
    err = row_rel_err(_run_mg(kata, q, k, v, g, layout), ref, v)
    assert err <= TOL["bf16"], (shape, layout, err)


def test_mg_layouts_agree_bitwise_and_one_group_is_the_flash_kernel(kata):
    import torch
    B, H, T, d, g, dv = 2, 3, 700, 64, 4, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=310, dtype="bf16")
    assert np.array_equal(_run_mg(kata, q, k, v, g, "bhtd"), _run_mg(kata, q, k, v, g, "bthd"))
    q1, k1, v1 = workloads.normal_qkv(B, H, T, 16, dv, seed=311, dtype="bf16")
    qd, kd, vd = to_dev(q1, "bf16"), to_dev(k1, "bf16"), to_dev(v1, "bf16")
    a = kata.kata_fwd_quadratic(qd, kd, vd)
    b = kata.kata_fwd_mg_quadratic(qd, kd, vd, 1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_mg_edge_cases(kata):
    # a single token, a tile plus one, and rows whose query is zero (zero
    # denominator: the output row is 0 on both sides)
    for (T, g) in [(1, 4), (129, 2)]:
        q, k, v = workloads.normal_qkv(1, 2, T, 64, 64, seed=320 + T, dtype="bf16")
        q[:, :, T // 2] = 0.0
        ref = oracle.direct_mg(q, k, v, g)
        for layout in ("bhtd", "bthd"):
            got = _run_mg(kata, q, k, v, g, layout)
            assert np.all(got[:, :, T // 2] == 0.0)
            assert row_rel_err(got, ref, v) <= TOL["bf16"]


@pytest.mark.parametrize("name", sorted(workloads.MG_CONFIGS))
def test_mg_full_size_sampled_rows(kata, name):
    """The benchmark's Mg workloads at full size, in the launch configuration
    bench.py times, compared on sampled rows the oracle computes one by one."""
    cfg = workloads.MG_CONFIGS[name]
    B, H, T, d, g, dv = cfg["B"], cfg["H"], cfg["T"], cfg["d"], cfg["groups"], cfg["dv"]
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=cfg["seed"], dtype=cfg["dtype"])
    got = _run_mg(kata, q, k, v, g, cfg["layout"])
    rng = np.random.default_rng(cfg["seed"])
    bh = rng.integers(0, B * H, size=96)
    t = np.concatenate([rng.integers(0, T, size=80), [0, 1, 127, 128, 129, T - 2, T - 1, T // 2] * 2])[:96]
    ref = oracle.direct_mg_rows(q, k, v, g, bh, t)
    vmax = np.abs(v.reshape(B * H, -1)).max(axis=1)[bh]
    rows = got.reshape(B * H, T, dv)[bh, t]
    assert rows_rel_err(rows, ref, vmax) <= TOL["bf16"]


@pytest.mark.parametrize("dtype,d,g,B,H", [
    (dt, d, g, 5, 3) for dt in ("f32", "bf16") for d, g in ((64, 4), (64, 2), (32, 2))
] + [("bf16", 64, 4, 64, 16), ("bf16", 64, 2, 64, 16)])  # and the benchmark's serving shape, B64 H16
def test_mg_decode_step(kata, dtype, d, g, B, H):
    import torch
    dv = 64
    q, k, v, S, z = workloads.decode_inputs_mg(B, H, d, g, dv, seed=d + g, dtype=dtype)
    o_ref, S_ref, z_ref = oracle.decode_step_mg(q, k, v, S, z, g)
    Sd = torch.from_numpy(S).cuda()
    zd = torch.from_numpy(z).cuda()
    o = kata.kata_decode_step_mg(to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype), Sd, zd, g)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    np.testing.assert_allclose(Sd.cpu().numpy(), S_ref, rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(zd.cpu().numpy(), z_ref, rtol=1e-6, atol=1e-5)
    err = row_rel_err(to_np(o)[:, :, None], o_ref[:, :, None], v[:, :, None])
    assert err <= TOL[dtype], err


def test_mg_decode_continues_the_forward(kata):
    """Decode steps from the oracle's Mg state after T tokens reproduce the
    flash Mg forward's outputs for the next tokens."""
    import torch
    B, H, T, d, g, dv = 2, 2, 200, 64, 4, 64
    q, k, v = workloads.normal_qkv(B, H, T + 3, d, dv, seed=330, dtype="bf16")
    o_fwd = _run_mg(kata, q, k, v, g, "bhtd")
    _, S, z = oracle.recurrent_mg(q[:, :, :T], k[:, :, :T], v[:, :, :T], g, return_state=True)
    Sd = torch.from_numpy(S.astype(np.float32)).cuda()
    zd = torch.from_numpy(z.astype(np.float32)).cuda()
    outs = []
    for t in range(T, T + 3):
        outs.append(to_np(kata.kata_decode_step_mg(to_dev(q[:, :, t], "bf16"), to_dev(k[:, :, t], "bf16"),
                                                   to_dev(v[:, :, t], "bf16"), Sd, zd, g)))
    torch.cuda.synchronize()
    assert row_rel_err(np.stack(outs, axis=2), o_fwd[:, :, T:], v) <= TOL["bf16"]


def test_mg_pages_call_shape(kata):
    """parallel_kata_attn: [B,T,H,D] in and out, num_groups factors per head."""
    import torch
    B, T, H, D = 2, 300, 4, 64
    q, k, v = workloads.normal_qkv(B, H, T, D, D, seed=340, dtype="bf16")
    o = kata.parallel_kata_attn(to_dev(_bthd(q), "bf16"), to_dev(_bthd(k), "bf16"), to_dev(_bthd(v), "bf16"),
                                num_groups=2)
    torch.cuda.synchronize()
    assert tuple(o.shape) == (B, T, H, D)
    assert row_rel_err(_bthd(to_np(o)), oracle.direct_mg(q, k, v, 2), v) <= TOL["bf16"]


@pytest.mark.parametrize("g", [2, 4])
def test_mg_many_items_ragged(kata, g):
    """More query-tile items than SMs with a ragged last tile (T = 1000):
    every persistent CTA walks several items; sampled rows against the oracle."""
    B, H, T, d, dv = 4, 16, 1000, 64, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=470 + g, dtype="bf16")
    got = _run_mg(kata, q, k, v, g, "bthd")
    rng = np.random.default_rng(471)
    bh = rng.integers(0, B * H, size=64)
    t = np.concatenate([rng.integers(0, T, size=56), [0, 127, 128, 895, 896, 998, 999, 500]])
    ref = oracle.direct_mg_rows(q, k, v, g, bh, t)
    vmax = np.abs(v.reshape(B * H, -1)).max(axis=1)[bh]
    assert rows_rel_err(got.reshape(B * H, T, dv)[bh, t], ref, vmax) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# KATA-Sigma-g (summed factors) through the same kernel
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["bhtd", "bthd"])
@pytest.mark.parametrize("shape", [(2, 2, 600, 64, 2), (1, 2, 385, 64, 4), (1, 3, 300, 32, 2)])
def test_sg_flash_matches_oracle(kata, shape, layout):
    import torch
    from oracle import sigma_g as osg
    B, H, T, d, g, dv = shape + (64,)
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=520 + T + g, dtype="bf16")
    ref = osg.direct_sg(q, k, v, g)
    if layout == "bthd":
        o = kata.kata_fwd_sg_quadratic(to_dev(_bthd(q), "bf16"), to_dev(_bthd(k), "bf16"), to_dev(_bthd(v), "bf16"),
                                       g, layout="bthd")
        got = _bthd(to_np(o))
    else:
        got = to_np(kata.kata_fwd_sg_quadratic(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), g))
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    assert row_rel_err(got, ref, v) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# KATA-Mg on the exact O(T) chunked path (cluster kernels: each group's
# packed state in its own CTAs, each group's intra-chunk squared scores in
# the first of them)
# ---------------------------------------------------------------------------

def _run_mg_chunked(K, q, k, v, groups, layout, C=64, S0=None, z0=None, return_state=False):
    import torch
    dq, dk, dv_ = ((to_dev(_bthd(x), "bf16") if layout == "bthd" else to_dev(x, "bf16")) for x in (q, k, v))
    res = K.kata_fwd_mg_chunked(dq, dk, dv_, groups, C=C, layout=layout, S0=S0, z0=z0, return_state=return_state)
    torch.cuda.synchronize()
    assert K.kata_get_status() == 0
    o = res[0] if return_state else res
    out = _bthd(to_np(o)) if layout == "bthd" else to_np(o)
    return (out, res[1], res[2]) if return_state else out


MG_CHUNKED_SHAPES = [
    # B, H, T, d, groups -- dv = 64; T ragged, one or several chunks
    (2, 2, 1000, 64, 4),
    (1, 3, 777, 64, 2),
    (1, 2, 129, 64, 4),
    (2, 1, 385, 64, 2),
    (1, 2, 600, 32, 1),   # the single factor p = 32 through the cluster kernel ([B,T,H,*] too)
]


@pytest.mark.parametrize("layout", ["bhtd", "bthd"])
@pytest.mark.parametrize("shape", MG_CHUNKED_SHAPES, ids=lambda s: "B%dH%dT%dd%dg%d" % s)
def test_mg_chunked_matches_oracle(kata, shape, layout):
    B, H, T, d, g = shape
    q, k, v = workloads.normal_qkv(B, H, T, d, 64, seed=400 + T + g, dtype="bf16")
    ref = oracle.direct_mg(q, k, v, g)
    err = row_rel_err(_run_mg_chunked(kata, q, k, v, g, layout), ref, v)
    assert err <= TOL["bf16"], (shape, layout, err)


@pytest.mark.parametrize("g", [4, 2])
@pytest.mark.parametrize("B,H,T,t0", [(4, 16, 700, 300), (1, 2, 20000, 7000)])
def test_mg_chunked_state_in_and_out(kata, g, B, H, T, t0):
    """Final state against the oracle's (elementwise bound from the
    arithmetic, as for the single factor), split-and-resume through the
    device state, and resume from the oracle's state.  With two heads and
    T = 20000 each sequence spans many super-chunks (state build, scan and
    prefix records); with 64 heads and T = 700 each is one super-chunk."""
    import torch
    d, dv = 64, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=17 + g, dtype="bf16")
    o_ref, S_ref, z_ref = oracle.recurrent_mg(q, k, v, g, return_state=True)
    _, S1, z1 = oracle.recurrent_mg(q[:, :, :t0], k[:, :, :t0], v[:, :, :t0], g, return_state=True)
    _, S_abs, z_abs = oracle.recurrent_mg(np.abs(q), np.abs(k), np.abs(v), g, return_state=True)
    eps = 2.0 ** -8 + (T + 4) * 2.0 ** -24

    def state_ok(S_dev, z_dev):
        return (np.all(np.abs(S_dev.cpu().numpy() - S_ref) <= eps * S_abs + 1e-6)
                and np.all(np.abs(z_dev.cpu().numpy() - z_ref) <= eps * z_abs + 1e-6))

    o, S, z = _run_mg_chunked(kata, q, k, v, g, "bhtd", return_state=True)
    assert row_rel_err(o, o_ref, v) <= TOL["bf16"]
    assert state_ok(S, z)
    oa, Sa, za = _run_mg_chunked(kata, q[:, :, :t0], k[:, :, :t0], v[:, :, :t0], g, "bhtd", return_state=True)
    ob, Sb, zb = _run_mg_chunked(kata, q[:, :, t0:], k[:, :, t0:], v[:, :, t0:], g, "bhtd", S0=Sa, z0=za,
                                 return_state=True)
    assert row_rel_err(np.concatenate([oa, ob], axis=2), o_ref, v) <= TOL["bf16"]
    assert state_ok(Sb, zb)
    o2 = _run_mg_chunked(kata, q[:, :, t0:], k[:, :, t0:], v[:, :, t0:], g, "bthd",
                         S0=torch.from_numpy(S1.astype(np.float32)).cuda(),
                         z0=torch.from_numpy(z1.astype(np.float32)).cuda())
    assert row_rel_err(o2, o_ref[:, :, t0:], v) <= TOL["bf16"]


@pytest.mark.parametrize("name", sorted(workloads.MG_CONFIGS))
def test_mg_chunked_full_size_sampled_rows(kata, name):
    """The benchmark's Mg workloads at full size through the chunked path, on
    sampled rows the oracle computes one by one; and the same bits in both
    layouts."""
    cfg = workloads.MG_CONFIGS[name]
    B, H, T, d, g, dv = cfg["B"], cfg["H"], cfg["T"], cfg["d"], cfg["groups"], cfg["dv"]
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=cfg["seed"], dtype=cfg["dtype"])
    got = _run_mg_chunked(kata, q, k, v, g, cfg["layout"])
    assert np.array_equal(got, _run_mg_chunked(kata, q, k, v, g, "bhtd" if cfg["layout"] == "bthd" else "bthd"))
    rng = np.random.default_rng(cfg["seed"])
    bh = rng.integers(0, B * H, size=96)
    t = np.concatenate([rng.integers(0, T, size=80), [0, 1, 127, 128, 129, T - 2, T - 1, T // 2] * 2])[:96]
    ref = oracle.direct_mg_rows(q, k, v, g, bh, t)
    vmax = np.abs(v.reshape(B * H, -1)).max(axis=1)[bh]
    assert rows_rel_err(got.reshape(B * H, T, dv)[bh, t], ref, vmax) <= TOL["bf16"]


def test_mg_chunked_agrees_with_flash(kata):
    B, H, T, d, g, dv = 2, 4, 1500, 64, 4, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=333, dtype="bf16")
    a = _run_mg_chunked(kata, q, k, v, g, "bhtd")
    b = _run_mg(kata, q, k, v, g, "bhtd")
    assert row_rel_err(a, b.astype(np.float64), v) <= 2 * TOL["bf16"]


# ---------------------------------------------------------------------------
# KATA-Sigma-g decode: one step on the summed-feature state [p*p, dv]
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d,g,B,H", [
    (dt, d, g, 5, 3) for dt in ("f32", "bf16") for d, g in ((64, 4), (64, 2), (32, 2))
] + [("bf16", 64, 4, 64, 16)])  # and the serving shape, B64 H16
def test_sg_decode_step(kata, dtype, d, g, B, H):
    """Against the fp64 Sigma-g step: the state element by element, the
    output with the per-row metric.  The starting state is random with the
    structure of a real one (symmetric S, positive-definite z, so the
    denominator is positive: <psi_S(q), z> with both PSD)."""
    import torch
    from oracle import sigma_g as osg
    p, dv = d // g, 64
    q, k, v = (x[:, :, 0] for x in workloads.normal_qkv(B, H, 1, d, dv, seed=400 + d + g, dtype=dtype))
    _, _, _, S, z = workloads.decode_inputs(B, H, p, dv, seed=410 + d + g, dtype=dtype)
    o_ref, S_ref, z_ref = osg.decode_step_sg(q, k, v, S, z, g)
    Sd, zd = torch.from_numpy(S).cuda(), torch.from_numpy(z).cuda()
    o = kata.kata_decode_step_sg(to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype), Sd, zd, g)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    np.testing.assert_allclose(Sd.cpu().numpy(), S_ref, rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(zd.cpu().numpy(), z_ref, rtol=1e-6, atol=1e-5)
    err = row_rel_err(to_np(o)[:, :, None], o_ref[:, :, None], v[:, :, None])
    assert err <= TOL[dtype], err


def test_sg_decode_continues_the_forward(kata):
    """Decode steps from the Sigma-g oracle's state after T tokens reproduce
    the flash Sigma-g forward's outputs for the next tokens."""
    import torch
    from oracle import sigma_g as osg
    B, H, T, d, g, dv = 2, 2, 150, 64, 4, 64
    q, k, v = workloads.normal_qkv(B, H, T + 3, d, dv, seed=420, dtype="bf16")
    o_fwd = to_np(kata.kata_fwd_sg_quadratic(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), g))
    fk = osg.features_sg(k[:, :, :T], g)
    Sd = torch.from_numpy(np.einsum("bhtp,bhte->bhpe", fk, v[:, :, :T].astype(np.float64)).astype(np.float32)).cuda()
    zd = torch.from_numpy(fk.sum(axis=2).astype(np.float32)).cuda()
    outs = []
    for t in range(T, T + 3):
        outs.append(to_np(kata.kata_decode_step_sg(to_dev(q[:, :, t], "bf16"), to_dev(k[:, :, t], "bf16"),
                                                   to_dev(v[:, :, t], "bf16"), Sd, zd, g)))
    torch.cuda.synchronize()
    assert row_rel_err(np.stack(outs, axis=2), o_fwd[:, :, T:], v) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# KATA-Sigma-g on the chunked path (groups of 16 on the p = 16 state)
# ---------------------------------------------------------------------------

def _sg_state(k, v, g):
    from oracle import sigma_g as osg
    fk = osg.features_sg(k, g)
    return (np.einsum("bhtp,bhte->bhpe", fk, np.asarray(v, np.float64)), fk.sum(axis=2))


# one super-chunk per (b,h) (B4 H4 T700), several (B2 H4 T3000) and many
# (B1 H2 T9000: the scan over dozens of records), plus ragged short cases
@pytest.mark.parametrize("B,H,T", [(2, 3, 77), (1, 2, 129), (4, 4, 700), (2, 4, 3000), (1, 2, 9000)])
@pytest.mark.parametrize("g", [2, 4])
def test_sg_chunked_matches_oracle(kata, B, H, T, g):
    import torch
    from oracle import sigma_g as osg
    d, dv = 16 * g, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=430 + T + g, dtype="bf16")
    o_ref = osg.recurrent_sg(q, k, v, g)
    o, S, z = kata.kata_fwd_sg_chunked(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), g,
                                       return_state=True)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    assert row_rel_err(to_np(o), o_ref, v) <= TOL["bf16"]
    # the final state: every packed entry sum_j k^j_a k^j_b is rounded to bf16
    # once (2^-9 relative), the T terms summed in fp32
    S_ref, z_ref = _sg_state(k, v, g)
    S_abs, z_abs = _sg_state(np.abs(k), np.abs(v), g)
    eps = 2.0 ** -8 + (T + 4) * 2.0 ** -24
    assert np.all(np.abs(S.cpu().numpy() - S_ref) <= eps * S_abs + 1e-6)
    assert np.all(np.abs(z.cpu().numpy() - z_ref) <= eps * z_abs + 1e-6)


@pytest.mark.parametrize("g", [2, 4])
def test_sg_chunked_state_in_and_out_and_agrees_with_flash(kata, g):
    import torch
    from oracle import sigma_g as osg
    B, H, T, t0, d, dv = 2, 4, 3000, 1100, 16 * g, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=440 + g, dtype="bf16")
    o_ref = osg.recurrent_sg(q, k, v, g)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    oa, Sa, za = kata.kata_fwd_sg_chunked(qd[:, :, :t0].contiguous(), kd[:, :, :t0].contiguous(),
                                          vd[:, :, :t0].contiguous(), g, return_state=True)
    ob = kata.kata_fwd_sg_chunked(qd[:, :, t0:].contiguous(), kd[:, :, t0:].contiguous(),
                                  vd[:, :, t0:].contiguous(), g, S0=Sa, z0=za)
    o_flash = kata.kata_fwd_sg_quadratic(qd, kd, vd, g)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    o_split = np.concatenate([to_np(oa), to_np(ob)], axis=2)
    assert row_rel_err(o_split, o_ref, v) <= TOL["bf16"]
    assert row_rel_err(o_split, to_np(o_flash), v) <= TOL["bf16"]
    # resume from the oracle's state after t0 tokens
    S1, z1 = _sg_state(k[:, :, :t0], v[:, :, :t0], g)
    o2 = kata.kata_fwd_sg_chunked(qd[:, :, t0:].contiguous(), kd[:, :, t0:].contiguous(), vd[:, :, t0:].contiguous(),
                                  g, S0=torch.from_numpy(S1.astype(np.float32)).cuda(),
                                  z0=torch.from_numpy(z1.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    assert row_rel_err(to_np(o2), o_ref[:, :, t0:], v) <= TOL["bf16"]


def test_sg_chunked_full_size_sampled_rows(kata):
    """B1 H16 T131072, d = 64 in 4 groups: sampled rows from the definition."""
    import torch
    B, H, T, d, g, dv = 1, 16, 131072, 64, 4, 64
    q, k, v = workloads.normal_qkv(B, H, T, d, dv, seed=450, dtype="bf16")
    got = to_np(kata.kata_fwd_sg_chunked(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), g))
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    rng = np.random.default_rng(451)
    rows = np.array(sorted(set([0, 1, 127, 128, 129, T // 2, T - 2, T - 1] + rng.integers(0, T, 16).tolist())))
    for h in (0, 9):
        qg = q[0, h].astype(np.float64).reshape(T, g, 16)
        kg = k[0, h].astype(np.float64).reshape(T, g, 16)
        ref = np.empty((len(rows), dv))
        for i, t in enumerate(rows):
            dots = np.einsum("jp,slp->sjl", qg[t], kg[:t + 1])
            w = (dots * dots).sum(axis=(1, 2))
            ref[i] = (w @ v[0, h, :t + 1].astype(np.float64)) / w.sum()
        vmax = np.full(len(rows), np.abs(v[0, h]).max())
        assert rows_rel_err(got[0, h, rows], ref, vmax) <= TOL["bf16"]

"""GPU parity: every C-ABI path against the fp64 oracle on the same seeded
inputs.  Small cases are compared element by element on every row; the full
benchmark shapes are compared on sampled rows the oracle computes one by one.

Gate (per-row relative error, tests/helpers.py): 1e-4 for fp32 inputs,
2e-2 for bf16 inputs with fp32 accumulation.
"""
import numpy as np
import pytest

import oracle
import workloads
from helpers import TOL, row_rel_err, rows_rel_err, sample_rows, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kata():
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return K


def _run(K, path, q, k, v, dtype, C=64):
    import torch
    qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    if path == "quadratic":
        o = K.kata_fwd_quadratic(qd, kd, vd)
    else:
        o = K.kata_fwd_chunked(qd, kd, vd, C=C)
    torch.cuda.synchronize()
    assert K.kata_get_status() == 0
    return to_np(o)


# ---------------------------------------------------------------------------
# full element-by-element parity at sizes the oracle finishes in seconds
# ---------------------------------------------------------------------------

def test_tiny_config_fp32_all_paths(kata):
    cfg = workloads.CONFIGS["tiny"]
    q, k, v = workloads.make_inputs(cfg)
    ref = oracle.direct(q, k, v)
    np.testing.assert_allclose(oracle.recurrent(q, k, v), ref, rtol=1e-10, atol=1e-12)
    for path, C in [("quadratic", 64), ("chunked", 64), ("chunked", 128)]:
        err = row_rel_err(_run(kata, path, q, k, v, "f32", C), ref, v)
        assert err <= TOL["f32"], (path, C, err)


SHAPES = [
    # B, H, T, p, dv -- T spans several 128-row tiles and ends ragged
    (2, 2, 1000, 16, 64),
    (1, 3, 777, 16, 16),
    (1, 2, 600, 32, 64),
    (2, 1, 385, 32, 16),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("path,C", [("quadratic", 64), ("chunked", 64), ("chunked", 128)])
def test_ragged_shapes(kata, dtype, shape, path, C):
    B, H, T, p, dv = shape
    q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=100 + T, dtype=dtype)
    ref = oracle.direct(q, k, v)
    err = row_rel_err(_run(kata, path, q, k, v, dtype, C), ref, v)
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_short_sequences(kata, T, dtype):
    q, k, v = workloads.normal_qkv(1, 2, T, 16, 64, seed=T, dtype=dtype)
    ref = oracle.direct(q, k, v)
    for path in ("quadratic", "chunked"):
        err = row_rel_err(_run(kata, path, q, k, v, dtype), ref, v)
        assert err <= TOL[dtype], (path, err)
    # o_1 = v_1 whenever q_1.k_1 != 0
    o = _run(kata, "chunked", q, k, v, dtype)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=TOL[dtype], atol=TOL[dtype])


def test_recall_shaped_inputs(kata):
    cfg = dict(workloads.CONFIGS["recall_p32"])
    q, k, v = workloads.recall_qkv(1, 2, 1100, 32, 64, seed=cfg["seed"], dtype="bf16")
    ref = oracle.direct(q, k, v)
    for path in ("quadratic", "chunked"):
        err = row_rel_err(_run(kata, path, q, k, v, "bf16"), ref, v)
        assert err <= TOL["bf16"], (path, err)


def test_zero_denominator_rows_give_zero(kata):
    # q_t orthogonal to every key so far: D_t = 0, o_t = 0 (stated reading)
    T, p, dv = 200, 16, 64
    rng = np.random.default_rng(0)
    k = np.zeros((1, 1, T, p), np.float32)
    k[..., 0] = 1.0                      # every key along e_0
    q = rng.standard_normal((1, 1, T, p)).astype(np.float32)
    q[0, 0, ::3, 0] = 0.0                # every third query orthogonal to all keys
    v = rng.standard_normal((1, 1, T, dv)).astype(np.float32)
    ref = oracle.direct(q, k, v)
    for dtype in ("f32", "bf16"):
        qq, kk, vv = (workloads.round_bf16(x) if dtype == "bf16" else x for x in (q, k, v))
        ref = oracle.direct(qq, kk, vv)
        for path in ("quadratic", "chunked"):
            o = _run(kata, path, qq, kk, vv, dtype)
            assert np.all(o[0, 0, ::3] == 0.0)
            assert row_rel_err(o, ref, vv) <= TOL[dtype]


def test_empty_sequence_is_a_noop(kata):
    import torch
    q = torch.zeros((1, 1, 0, 16), device="cuda", dtype=torch.bfloat16)
    v = torch.zeros((1, 1, 0, 64), device="cuda", dtype=torch.bfloat16)
    assert kata.kata_fwd_quadratic(q, q, v).shape == (1, 1, 0, 64)
    o, S, z = kata.kata_fwd_chunked(q, q, v, return_state=True)
    torch.cuda.synchronize()
    assert float(S.abs().max()) == 0.0 and float(z.abs().max()) == 0.0


# ---------------------------------------------------------------------------
# state: initial / final state, split-and-resume, decode
# ---------------------------------------------------------------------------

# With 128 (b,h) pairs and T = 700 every pair is one super-chunk (no
# workspace: the readout starts from S0 and writes the final state); with 2
# pairs and T = 20000 each spans many, with the state build, the scan and
# the prefix records in between; with 16 pairs and T = 3000 (and the 1900
# tokens resumed from S0 after 1100) each spans a handful (8 super-chunks of
# the bf16 p = 16 plan), the regime of the long-context benchmark.
# p = 32 in bf16 runs the four-block cluster kernels (the state split over
# four coordinate blocks, one CTA each), with the same regimes.
@pytest.mark.parametrize("B,H,T,t0", [(8, 16, 700, 300), (1, 2, 20000, 7000), (2, 8, 3000, 1100)])
@pytest.mark.parametrize("dtype,p", [("f32", 16), ("bf16", 16), ("bf16", 32)])
def test_chunked_state_in_and_out(kata, dtype, p, B, H, T, t0):
    import torch
    dv = 64
    q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=7, dtype=dtype)
    o_ref, S_ref, z_ref = oracle.recurrent(q, k, v, return_state=True)
    _, S1, z1 = oracle.recurrent(q[:, :, :t0], k[:, :, :t0], v[:, :, :t0], return_state=True)
    qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    # elementwise bound on the final state from the arithmetic: every term
    # psi(k_t)_r v_t is rounded once to the operand type (bf16: 2^-9 relative
    # for the psi entry, then exact products into fp32) and T terms are summed
    # in fp32; the bound is  eps * sum_t |psi(k_t)_r| |v_t|  with
    # eps = 2^-8 + (T + 4) 2^-24 for bf16 and (T + 4) 2^-24 for fp32.
    _, S_abs, z_abs = oracle.recurrent(np.abs(q), np.abs(k), np.abs(v), return_state=True, need_output=False)
    eps = (2.0 ** -8 if dtype == "bf16" else 0.0) + (T + 4) * 2.0 ** -24

    def state_ok(S_dev, z_dev):
        return (np.all(np.abs(S_dev.cpu().numpy() - S_ref) <= eps * S_abs + 1e-6)
                and np.all(np.abs(z_dev.cpu().numpy() - z_ref) <= eps * z_abs + 1e-6))

    # whole sequence with final state
    o, S, z = kata.kata_fwd_chunked(qd, kd, vd, return_state=True)
    torch.cuda.synchronize()
    assert row_rel_err(to_np(o), o_ref, v) <= TOL[dtype]
    assert state_ok(S, z)
    # split: first part on the device, resume from the device state
    oa, Sa, za = kata.kata_fwd_chunked(qd[:, :, :t0].contiguous(), kd[:, :, :t0].contiguous(),
                                       vd[:, :, :t0].contiguous(), return_state=True)
    ob, Sb, zb = kata.kata_fwd_chunked(qd[:, :, t0:].contiguous(), kd[:, :, t0:].contiguous(),
                                       vd[:, :, t0:].contiguous(), S0=Sa, z0=za, return_state=True)
    torch.cuda.synchronize()
    o_split = np.concatenate([to_np(oa), to_np(ob)], axis=2)
    assert row_rel_err(o_split, o_ref, v) <= TOL[dtype]
    assert state_ok(Sb, zb)
    # resume from the oracle's state
    o2 = kata.kata_fwd_chunked(qd[:, :, t0:].contiguous(), kd[:, :, t0:].contiguous(), vd[:, :, t0:].contiguous(),
                               S0=torch.from_numpy(S1.astype(np.float32)).cuda(),
                               z0=torch.from_numpy(z1.astype(np.float32)).cuda())
    assert row_rel_err(to_np(o2), o_ref[:, :, t0:], v) <= TOL[dtype]


# the sequential inter-chunk baseline: one CTA walks each sequence's chunks
@pytest.mark.parametrize("B,H,T", [(1, 2, 1000), (2, 3, 2500)])
def test_sequential_baseline_matches_oracle(kata, B, H, T):
    import torch
    p, dv = 16, 64
    q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=31, dtype="bf16")
    o_ref, S_ref, z_ref = oracle.recurrent(q, k, v, return_state=True)
    _, S_abs, z_abs = oracle.recurrent(np.abs(q), np.abs(k), np.abs(v), return_state=True, need_output=False)
    eps = 2.0 ** -8 + (T + 4) * 2.0 ** -24  # as in test_chunked_state_in_and_out
    o, S, z = kata.kata_fwd_chunked_sequential(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"),
                                               return_state=True)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    assert row_rel_err(to_np(o), o_ref, v) <= TOL["bf16"]
    assert np.all(np.abs(S.cpu().numpy() - S_ref) <= eps * S_abs + 1e-6)
    assert np.all(np.abs(z.cpu().numpy() - z_ref) <= eps * z_abs + 1e-6)


def _check_decode(kata, B, H, p, dv, dtype, seed):
    """One decode step against the oracle: the updated state element by
    element, and the output with the per-row metric of the other parity tests
    (one row per (b,h) stream, floored at 1e-3 of that stream's |v|_inf)."""
    import torch
    q, k, v, S, z = workloads.decode_inputs(B, H, p, dv, seed=seed, dtype=dtype)
    o_ref, S_ref, z_ref = oracle.decode_step(q, k, v, S, z)
    Sd = torch.from_numpy(S).cuda()
    zd = torch.from_numpy(z).cuda()
    o = kata.kata_decode_step(to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype), Sd, zd)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    np.testing.assert_allclose(Sd.cpu().numpy(), S_ref, rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(zd.cpu().numpy(), z_ref, rtol=1e-6, atol=1e-5)
    err = row_rel_err(to_np(o)[:, :, None], o_ref[:, :, None], v[:, :, None])
    assert err <= TOL[dtype], err


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p,dv", [(16, 64), (16, 16), (32, 64), (32, 16)])
def test_decode_step(kata, dtype, p, dv):
    _check_decode(kata, 5, 3, p, dv, dtype, seed=p + dv)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_step_serving_shape(kata, dtype):
    """The decode step at the batched-serving size the benchmark times
    (B=64, H=16, state [256 x 64] fp32 per stream: 1024 streams)."""
    c = workloads.DECODE
    _check_decode(kata, c["B"], c["H"], c["p"], c["dv"], dtype, seed=c["seed"])


def test_decode_continues_chunked(kata):
    """T-step decode from the chunked final state equals the forward output."""
    import torch
    B, H, T, p, dv = 2, 2, 300, 16, 64
    q, k, v = workloads.normal_qkv(B, H, T + 4, p, dv, seed=9, dtype="bf16")
    ref = oracle.direct(q, k, v)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    _, S, z = kata.kata_fwd_chunked(qd[:, :, :T].contiguous(), kd[:, :, :T].contiguous(), vd[:, :, :T].contiguous(),
                                    return_state=True)
    outs = []
    for t in range(T, T + 4):
        outs.append(to_np(kata.kata_decode_step(qd[:, :, t].contiguous(), kd[:, :, t].contiguous(),
                                                vd[:, :, t].contiguous(), S, z)))
    torch.cuda.synchronize()
    o = np.stack(outs, axis=2)
    assert row_rel_err(o, ref[:, :, T:], v) <= TOL["bf16"]


# ---------------------------------------------------------------------------
# cross-path agreement and determinism
# ---------------------------------------------------------------------------

def test_paths_agree_and_are_deterministic(kata):
    import torch
    B, H, T, p, dv = 2, 4, 1500, 16, 64
    q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=5, dtype="bf16")
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    oq1 = kata.kata_fwd_quadratic(qd, kd, vd)
    oq2 = kata.kata_fwd_quadratic(qd, kd, vd)
    oc1 = kata.kata_fwd_chunked(qd, kd, vd, C=64)
    oc2 = kata.kata_fwd_chunked(qd, kd, vd, C=64)
    oc3 = kata.kata_fwd_chunked(qd, kd, vd, C=128)
    torch.cuda.synchronize()
    assert torch.equal(oq1, oq2) and torch.equal(oc1, oc2)
    assert row_rel_err(to_np(oc1), to_np(oq1).astype(np.float64), v) <= 2 * TOL["bf16"]
    assert row_rel_err(to_np(oc3), to_np(oc1).astype(np.float64), v) <= 2 * TOL["bf16"]


# ---------------------------------------------------------------------------
# full benchmark shapes, sampled rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["layer340m_ctx2k", "long_ctx131k", "recall_p32"])
@pytest.mark.parametrize("path", ["chunked", "quadratic"])
def test_full_size_sampled_rows(kata, name, path):
    import torch
    cfg = workloads.CONFIGS[name]
    q, k, v = workloads.make_inputs(cfg)
    B, H, T = cfg["B"], cfg["H"], cfg["T"]
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    if path == "quadratic":
        o = kata.kata_fwd_quadratic(qd, kd, vd)
    else:
        o = kata.kata_fwd_chunked(qd, kd, vd, C=cfg["C"])
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    o = o.float().cpu().numpy().reshape(B * H, T, -1)
    rng = np.random.default_rng(123)
    n_rand = 24 if T > 10000 else 64
    bh_list, t_list = [], []
    for bh in rng.choice(B * H, size=min(B * H, 6), replace=False):
        ts = sample_rows(T, cfg["C"], n_rand, rng)
        bh_list += [bh] * len(ts)
        t_list += ts.tolist()
    bh_idx, t_idx = np.array(bh_list), np.array(t_list)
    ref = oracle.direct_rows(q, k, v, bh_idx, t_idx)
    vmax = np.abs(v.reshape(B * H, -1)).max(axis=1)[bh_idx]
    err = rows_rel_err(o[bh_idx, t_idx], ref, vmax)
    assert err <= TOL["bf16"], err


# ---------------------------------------------------------------------------
# CUDA graph capture: the calls only enqueue work on the caller's stream (the
# chunked call with several super-chunks launches state build, scan and
# readout, the last two as programmatic dependents), so a captured step
# replays to the same bits as the eager calls
# ---------------------------------------------------------------------------

def test_graph_replay_matches_eager(kata):
    import torch
    B, H, T, p, dv = 1, 2, 20000, 16, 64  # several super-chunks per head
    q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=11, dtype="bf16")
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    ws = torch.empty(max(256, kata.kata_fwd_chunked_workspace_size(B, H, T, p, dv, 64)), dtype=torch.uint8,
                     device="cuda")
    oq, oc = torch.empty_like(vd), torch.empty_like(vd)
    S = torch.empty((B, H, p * p, dv), dtype=torch.float32, device="cuda")
    z = torch.empty((B, H, p * p), dtype=torch.float32, device="cuda")
    qt, kt, vt = qd[:, :, :1].contiguous(), kd[:, :, :1].contiguous(), vd[:, :, :1].contiguous()
    od = torch.empty((B, H, dv), dtype=torch.bfloat16, device="cuda")

    def step():
        kata.kata_fwd_quadratic(qd, kd, vd, o=oq)
        kata.kata_fwd_chunked(qd, kd, vd, C=64, o=oc, workspace=ws, S_out=S, z_out=z, return_state=True)
        kata.kata_decode_step(qt[:, :, 0], kt[:, :, 0], vt[:, :, 0], S, z, o=od)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    ref = [t.clone() for t in (oq, oc, S, z, od)]
    for t in (oq, oc, S, z, od):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    for got, want in zip((oq, oc, S, z, od), ref):
        assert torch.equal(got, want)
    del g

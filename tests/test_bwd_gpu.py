"""GPU parity of the training entry points against the fp64 gradient oracle
(oracle/backward.py, pinned by finite differences): the forward that saves
the denominators, and the backward pass.

Gate for the gradients (bf16 inputs, fp32 accumulation): per (b,h) and per
tensor, ||g - g_ref||_F / ||g_ref||_F <= 2e-2.  The bf16 operands of the
backward MMAs (q, k, v, dO/D, the squares and dS) each carry one rounding of
relative size 2^-9; summed over a row with mixed signs, the resulting error
stays a small multiple of that, and a norm-relative gate (rather than an
elementwise one) is used because dq and dk are sums whose terms cancel
(sum_s w_ts dw_ts = 0 for every t), so single entries can be small.
"""
import numpy as np
import pytest

import oracle
import workloads
from helpers import TOL, to_dev, to_np
from oracle import backward as obw

pytestmark = pytest.mark.gpu
GRAD_TOL = 2e-2


@pytest.fixture(scope="module")
def kata():
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return K


def _grad_err(got, ref):
    got = np.asarray(got, np.float64).reshape(ref.shape[0] * ref.shape[1], -1)
    ref = np.asarray(ref, np.float64).reshape(got.shape)
    num = np.linalg.norm(got - ref, axis=1)
    den = np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    return float((num / den).max())


def _dO(shape, seed):
    return workloads.round_bf16(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))


def _run(K, q, k, v, dO):
    import torch
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    o, D = K.kata_fwd_quadratic_train(qd, kd, vd)
    dq, dk, dv = K.kata_bwd_quadratic(qd, kd, vd, o, D, to_dev(dO, "bf16"))
    torch.cuda.synchronize()
    assert K.kata_get_status() == 0
    return to_np(o), D.cpu().numpy(), to_np(dq), to_np(dk), to_np(dv)


SHAPES = [
    # B, H, T, p -- several 128-row tiles with a ragged tail, a single tile,
    # an exact tile, and p = 32
    (2, 2, 1000, 16),
    (1, 1, 129, 16),
    (1, 2, 128, 16),
    (1, 3, 777, 32),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_backward_matches_oracle(kata, shape):
    B, H, T, p = shape
    q, k, v = workloads.normal_qkv(B, H, T, p, 64, seed=400 + T + p, dtype="bf16")
    dO = _dO(v.shape, 401 + T)
    o, D, dq, dk, dv = _run(kata, q, k, v, dO)
    o_ref, D_ref = obw.forward_with_d(q, k, v)
    np.testing.assert_allclose(D, D_ref, rtol=1e-2, atol=1e-30)
    gq, gk, gv = obw.backward(q, k, v, dO)
    errs = {n: _grad_err(g, r) for n, g, r in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv))}
    assert max(errs.values()) <= GRAD_TOL, errs


def test_train_forward_is_the_flash_forward(kata):
    import torch
    q, k, v = workloads.normal_qkv(2, 3, 600, 16, 64, seed=410, dtype="bf16")
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    o1 = kata.kata_fwd_quadratic(qd, kd, vd)
    o2, _ = kata.kata_fwd_quadratic_train(qd, kd, vd)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_zero_denominator_rows_pass_no_gradient(kata):
    q, k, v = workloads.normal_qkv(1, 2, 300, 16, 64, seed=420, dtype="bf16")
    q[:, :, [0, 150, 299]] = 0.0
    dO = _dO(v.shape, 421)
    o, D, dq, dk, dv = _run(kata, q, k, v, dO)
    assert np.all(D[:, :, [0, 150, 299]] == 0.0)
    assert np.all(dq[:, :, [0, 150, 299]] == 0.0)
    gq, gk, gv = obw.backward(q, k, v, dO)
    assert max(_grad_err(dq, gq), _grad_err(dk, gk), _grad_err(dv, gv)) <= GRAD_TOL


def test_autograd_wrapper(kata):
    import torch
    q, k, v = workloads.normal_qkv(1, 2, 256, 16, 64, seed=430, dtype="bf16")
    dO = _dO(v.shape, 431)
    qd, kd, vd = (to_dev(x, "bf16").requires_grad_(True) for x in (q, k, v))
    o = kata.kata_attention(qd, kd, vd)
    o.backward(to_dev(dO, "bf16"))
    torch.cuda.synchronize()
    _, _, dq, dk, dv = _run(kata, q, k, v, dO)
    assert np.array_equal(to_np(qd.grad), dq) and np.array_equal(to_np(kd.grad), dk)
    assert np.array_equal(to_np(vd.grad), dv)


def test_backward_full_size_sampled_heads(kata):
    """The training workload at full size (B8 H16 T2048 p16 dv64); the
    oracle's T x T gradient is computed for a few heads and compared whole."""
    cfg = workloads.CONFIGS["layer340m_ctx2k"]
    q, k, v = workloads.make_inputs(cfg)
    dO = _dO(v.shape, 440)
    _, _, dq, dk, dv = _run(kata, q, k, v, dO)
    for (b, h) in [(0, 0), (3, 7), (7, 15)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        gq, gk, gv = obw.backward(q[sl], k[sl], v[sl], dO[sl])
        errs = (_grad_err(dq[sl], gq), _grad_err(dk[sl], gk), _grad_err(dv[sl], gv))
        assert max(errs) <= GRAD_TOL, (b, h, errs)


def test_backward_with_tiny_denominators(kata):
    """Rows whose query is nearly orthogonal to every key seen so far have a
    tiny D_t; their gradient terms scale with 1/D_t and cancel (o_t is almost
    a single value vector).  Query 0 of each head is made nearly orthogonal
    to key 0 (D_0 ~ 1e-6), and query 5 nearly orthogonal to keys 0..5."""
    B, H, T, p = 1, 2, 300, 16
    q, k, v = workloads.normal_qkv(B, H, T, p, 64, seed=0, dtype="bf16")
    rng = np.random.default_rng(450)
    for h in range(H):
        for t in (0, 5):
            K0 = k[0, h, :t + 1].astype(np.float64)
            x = rng.standard_normal(p)
            x -= K0.T @ np.linalg.lstsq(K0.T, x, rcond=None)[0]   # orthogonal to keys 0..t
            x = x / np.linalg.norm(x) + 1e-3 * K0[0] / np.linalg.norm(K0[0])
            q[0, h, t] = workloads.round_bf16((x / np.linalg.norm(x)).astype(np.float32))
    dO = _dO(v.shape, 451)
    _, D, dq, dk, dv = _run(kata, q, k, v, dO)
    assert D[0, :, 0].max() < 1e-4
    gq, gk, gv = obw.backward(q, k, v, dO)
    errs = (_grad_err(dq, gq), _grad_err(dk, gk), _grad_err(dv, gv))
    assert max(errs) <= GRAD_TOL, errs


def test_backward_many_items_ragged(kata):
    """More (tile, head) items than SMs, so every persistent CTA walks several
    items, with a ragged last tile (T = 1000); whole heads compared."""
    B, H, T, p = 4, 16, 1000, 16
    q, k, v = workloads.normal_qkv(B, H, T, p, 64, seed=460, dtype="bf16")
    dO = _dO(v.shape, 461)
    _, _, dq, dk, dv = _run(kata, q, k, v, dO)
    for (b, h) in [(0, 0), (1, 9), (3, 15)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        gq, gk, gv = obw.backward(q[sl], k[sl], v[sl], dO[sl])
        errs = (_grad_err(dq[sl], gq), _grad_err(dk[sl], gk), _grad_err(dv[sl], gv))
        assert max(errs) <= GRAD_TOL, (b, h, errs)


@pytest.mark.parametrize("shape", [(2, 2, 700, 64, 2), (1, 3, 385, 64, 4), (1, 2, 256, 32, 2)])
def test_mg_backward_matches_oracle(kata, shape):
    """KATA-Mg gradients against the fp64 Mg gradient oracle; the autograd
    wrapper gives the same bits."""
    import torch
    B, H, T, d, g = shape
    q, k, v = workloads.normal_qkv(B, H, T, d, 64, seed=490 + T + g, dtype="bf16")
    dO = _dO(v.shape, 491 + T)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    o, D = kata.kata_fwd_mg_quadratic_train(qd, kd, vd, g)
    assert torch.equal(o, kata.kata_fwd_mg_quadratic(qd, kd, vd, g))
    dq, dk, dv = kata.kata_bwd_mg_quadratic(qd, kd, vd, o, D, to_dev(dO, "bf16"), g)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    gq, gk, gv = obw.backward_mg(q, k, v, dO, g)
    errs = (_grad_err(to_np(dq), gq), _grad_err(to_np(dk), gk), _grad_err(to_np(dv), gv))
    assert max(errs) <= GRAD_TOL, errs
    qa, ka, va = (x.clone().requires_grad_(True) for x in (qd, kd, vd))
    kata.kata_attention_mg(qa, ka, va, g).backward(to_dev(dO, "bf16"))
    torch.cuda.synchronize()
    assert torch.equal(qa.grad, dq) and torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)


@pytest.mark.parametrize("B,H,T", [(4, 8, 1000), (1, 2, 5000)])
def test_chunked_backward_is_deterministic(kata, B, H, T):
    """Repeated calls give bitwise the same gradients: no role of the walk
    kernels reads TMEM or shared memory that another role is still writing
    (one super-chunk of 8 chunks per walk at B4 H8, several at B1 H2)."""
    import torch
    q, k, v = workloads.normal_qkv(B, H, T, 16, 64, seed=77 + T, dtype="bf16")
    dO = np.random.default_rng(T).standard_normal((B, H, T, 64)).astype(np.float32)
    qd, kd, vd, dOd = (to_dev(x, "bf16") for x in (q, k, v, dO))
    o, D = kata.kata_fwd_chunked_train(qd, kd, vd)
    first = [x.clone() for x in kata.kata_bwd_chunked(qd, kd, vd, o, D, dOd)]
    for _ in range(4):
        again = kata.kata_bwd_chunked(qd, kd, vd, o, D, dOd)
        torch.cuda.synchronize()
        assert all(torch.equal(a, b) for a, b in zip(first, again))
    assert kata.kata_get_status() == 0


@pytest.mark.parametrize("shape", [(2, 2, 700, 64, 4), (1, 3, 385, 32, 2), (1, 2, 256, 64, 2)])
def test_sg_backward_matches_oracle(kata, shape):
    """KATA-Sigma-g gradients (one single-factor pass per query group x key
    group, accumulated) against the fp64 Sigma-g gradient oracle; the training
    forward equals the plain Sigma-g forward, and the autograd wrapper gives
    the same bits."""
    import torch
    B, H, T, d, g = shape
    q, k, v = workloads.normal_qkv(B, H, T, d, 64, seed=495 + T + g, dtype="bf16")
    dO = _dO(v.shape, 496 + T)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    o, D = kata.kata_fwd_sg_quadratic_train(qd, kd, vd, g)
    assert torch.equal(o, kata.kata_fwd_sg_quadratic(qd, kd, vd, g))
    dq, dk, dv = kata.kata_bwd_sg_quadratic(qd, kd, vd, o, D, to_dev(dO, "bf16"), g)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    gq, gk, gv = obw.backward_sg(q, k, v, dO, g)
    errs = (_grad_err(to_np(dq), gq), _grad_err(to_np(dk), gk), _grad_err(to_np(dv), gv))
    assert max(errs) <= GRAD_TOL, errs
    qa, ka, va = (x.clone().requires_grad_(True) for x in (qd, kd, vd))
    kata.kata_attention_sg(qa, ka, va, g).backward(to_dev(dO, "bf16"))
    torch.cuda.synchronize()
    assert torch.equal(qa.grad, dq) and torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)


# ---------------------------------------------------------------------------
# the O(T) chunked path: forward with D, backward through the chunk states
# ---------------------------------------------------------------------------

# one chunk (no pair crosses a chunk boundary), a ragged second chunk, several
# chunks, and enough (b,h) x chunks for many CTA waves.  The plan walks
# T = 777 as 7 super-chunks and T = 4096 as 16 (summed and scanned first), the
# other shapes as one super-chunk per sequence (each walk starts from zero)
@pytest.mark.parametrize("B,H,T", [(1, 2, 100), (1, 2, 200), (2, 3, 777), (4, 8, 1000), (1, 1, 4096),
                                   (8, 16, 520)])
def test_chunked_backward_matches_oracle(kata, B, H, T):
    """Gradients of the chunked training path against the fp64 gradient
    oracle, with the gate of the flash-path backward; the training forward's
    o equals kata_fwd_chunked's and its D agrees with the flash forward's."""
    import torch
    p = 16
    q, k, v = workloads.normal_qkv(B, H, T, p, 64, seed=520 + T, dtype="bf16")
    dO = _dO(v.shape, 521 + T)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    o, D = kata.kata_fwd_chunked_train(qd, kd, vd)
    assert torch.equal(o, kata.kata_fwd_chunked(qd, kd, vd))
    _, D_flash = kata.kata_fwd_quadratic_train(qd, kd, vd)
    torch.cuda.synchronize()
    np.testing.assert_allclose(D.cpu().numpy(), D_flash.cpu().numpy(), rtol=2e-2, atol=1e-6)
    dq, dk, dv = kata.kata_bwd_chunked(qd, kd, vd, o, D, to_dev(dO, "bf16"))
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    gq, gk, gv = obw.backward(q, k, v, dO)
    errs = (_grad_err(to_np(dq), gq), _grad_err(to_np(dk), gk), _grad_err(to_np(dv), gv))
    assert max(errs) <= GRAD_TOL, errs
    qa, ka, va = (x.clone().requires_grad_(True) for x in (qd, kd, vd))
    kata.kata_attention_chunked(qa, ka, va).backward(to_dev(dO, "bf16"))
    torch.cuda.synchronize()
    assert torch.equal(qa.grad, dq) and torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)

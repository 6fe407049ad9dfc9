"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each test ties the oracle to something other than itself: values worked by
hand from the defining rule (tests/golden/), closed forms, special cases, the
convex-gate identity, and invariances that follow from the definition.  The
tests are chosen so that a plausible slip in the oracle (a dropped term, an
unsquared or transposed score, an exclusive instead of inclusive causal sum, a
missing normalisation, a wrong psi index) fails at least one of them; the
mutation tests at the end plant such slips in copies of the oracle's C source
and check that the pins catch them.
"""
import os
import subprocess
import ctypes
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([Fraction(x) for x in line.split()])
    a = np.array([[float(x) for x in r] for r in rows])
    q, k, v, o = a[:, 0:2], a[:, 2:4], a[:, 4:6], a[:, 6:8]
    return (x[None, None] for x in (q, k, v, o))


# ---------------------------------------------------------------------------
# worked examples (tests/golden)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fn", ["direct", "recurrent"])
def test_worked_example_p2(fn):
    q, k, v, o_expected = _read_golden("worked_example_p2.txt")
    o = getattr(oracle, fn)(q, k, v)
    np.testing.assert_allclose(o, o_expected, rtol=0, atol=1e-14)


@pytest.mark.parametrize("fn", ["direct", "recurrent"])
def test_zero_denominator_reading(fn):
    q, k, v, o_expected = _read_golden("zero_denominator.txt")
    o = getattr(oracle, fn)(q, k, v)
    np.testing.assert_array_equal(o, o_expected)


# ---------------------------------------------------------------------------
# four identities that follow from the definition: direct = recurrent, o_1 = v_1,
# the convex-gate bounds, identical keys give the running mean
# ---------------------------------------------------------------------------

def _rand(B=2, H=2, T=40, p=5, dv=3, seed=11):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, T, p)), rng.standard_normal((B, H, T, p)),
            rng.standard_normal((B, H, T, dv)))


@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (2, 3, 37, 4, 5), (1, 2, 64, 16, 16), (1, 1, 9, 32, 2)])
def test_direct_equals_recurrent(shape):
    B, H, T, p, dv = shape
    q, k, v = _rand(B, H, T, p, dv, seed=T + p)
    np.testing.assert_allclose(oracle.direct(q, k, v), oracle.recurrent(q, k, v), rtol=1e-11, atol=1e-12)


def test_first_output_is_first_value():
    q, k, v = _rand()
    o = oracle.direct(q, k, v)
    np.testing.assert_allclose(o[:, :, 0, :], v[:, :, 0, :], rtol=1e-14, atol=0)


@pytest.mark.parametrize("fn", ["direct", "recurrent"])
def test_convex_gate_bounds(fn):
    """Nonnegative weights: each output coordinate lies in the range of the past values."""
    q, k, v = _rand(T=80, seed=3)
    o = getattr(oracle, fn)(q, k, v)
    lo = np.minimum.accumulate(v, axis=2)
    hi = np.maximum.accumulate(v, axis=2)
    eps = 1e-12
    assert np.all(o >= lo - eps) and np.all(o <= hi + eps)
    # the bound is tight somewhere only through nonnegativity: also check a
    # query anti-aligned with keys still gives weights >= 0 (signs cancel)
    o_neg = getattr(oracle, fn)(-q, k, v)
    np.testing.assert_allclose(o_neg, o, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("fn", ["direct", "recurrent"])
def test_identical_keys_running_mean(fn):
    rng = np.random.default_rng(5)
    B, H, T, p, dv = 1, 2, 33, 6, 4
    kvec = rng.standard_normal(p)
    k = np.broadcast_to(kvec, (B, H, T, p)).copy()
    q = rng.standard_normal((B, H, T, p))
    v = rng.standard_normal((B, H, T, dv))
    o = getattr(oracle, fn)(q, k, v)
    mean = np.cumsum(v, axis=2) / np.arange(1, T + 1)[None, None, :, None]
    np.testing.assert_allclose(o, mean, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# the convex output gate, gate form (ai.info summary, Main Findings:
# o_t = alpha_t r_{t-1} + beta_t v_t with alpha_t = D_{t-1}/D_t,
# beta_t = c_t/D_t, alpha_t + beta_t = 1)
# ---------------------------------------------------------------------------

def test_gate_form_identity():
    q, k, v = _rand(B=1, H=1, T=30, p=4, dv=3, seed=21)
    T = q.shape[2]
    o = oracle.direct(q, k, v)
    for t in range(1, T):
        # previous readout read with the current query: replace q_{t-1} by q_t
        # in the length-t prefix and take its last output
        qq = q[:, :, : t].copy()
        qq[:, :, t - 1] = q[:, :, t]
        r_prev, d_prev = oracle.direct_rows(qq, k[:, :, :t], v[:, :, :t], [0], [t - 1], return_d=True)
        _, d_t = oracle.direct_rows(q, k, v, [0], [t], return_d=True)
        c_t = float(np.dot(q[0, 0, t], k[0, 0, t]) ** 2)
        alpha, beta = d_prev[0] / d_t[0], c_t / d_t[0]
        assert abs(alpha + beta - 1.0) < 1e-12
        np.testing.assert_allclose(o[0, 0, t], alpha * r_prev[0] + beta * v[0, 0, t], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# closed forms and special cases
# ---------------------------------------------------------------------------

def test_orthonormal_keys_exact_retrieval():
    """Keys from an orthonormal basis, query = basis vector j: o_t is the mean
    of the values stored under e_j so far (0 if none yet)."""
    rng = np.random.default_rng(7)
    p, dv, T = 8, 3, 50
    # signed standard basis: exactly orthonormal in floating point
    R = np.eye(p) * rng.choice([-1.0, 1.0], size=p)
    key_ids = rng.integers(0, p, size=T)
    qry_ids = rng.integers(0, p, size=T)
    k = R[:, key_ids].T[None, None]
    q = R[:, qry_ids].T[None, None]
    v = rng.standard_normal((1, 1, T, dv))
    o = oracle.direct(q, k, v)
    for t in range(T):
        match = [s for s in range(t + 1) if key_ids[s] == qry_ids[t]]
        want = v[0, 0, match].mean(axis=0) if match else np.zeros(dv)
        np.testing.assert_allclose(o[0, 0, t], want, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("fn", ["direct", "recurrent"])
def test_p1_closed_form(fn):
    rng = np.random.default_rng(8)
    T, dv = 25, 4
    q = rng.standard_normal((1, 1, T, 1)) + 2.0
    k = rng.standard_normal((1, 1, T, 1))
    v = rng.standard_normal((1, 1, T, dv))
    o = getattr(oracle, fn)(q, k, v)
    k2 = k[0, 0, :, 0] ** 2
    want = np.cumsum(k2[:, None] * v[0, 0], axis=0) / np.cumsum(k2)[:, None]
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# invariances that follow from the definition
# ---------------------------------------------------------------------------

def test_invariances():
    q, k, v = _rand(B=1, H=2, T=35, p=6, dv=4, seed=9)
    rng = np.random.default_rng(10)
    o = oracle.direct(q, k, v)
    T = q.shape[2]
    # sign flips of individual queries and keys
    sq = rng.choice([-1.0, 1.0], size=(1, 2, T, 1))
    sk = rng.choice([-1.0, 1.0], size=(1, 2, T, 1))
    np.testing.assert_allclose(oracle.direct(q * sq, k * sk, v), o, rtol=1e-11, atol=1e-12)
    # per-query scaling and a global key scale
    cq = rng.uniform(0.1, 10.0, size=(1, 2, T, 1))
    np.testing.assert_allclose(oracle.direct(q * cq, k * 3.7, v), o, rtol=1e-10, atol=1e-11)
    # joint rotation of queries and keys
    Rm, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    np.testing.assert_allclose(oracle.direct(q @ Rm.T, k @ Rm.T, v), o, rtol=1e-10, atol=1e-11)
    # affine equivariance in v
    A = rng.standard_normal((4, 4))
    b = rng.standard_normal(4)
    np.testing.assert_allclose(oracle.direct(q, k, v @ A + b), o @ A + b, rtol=1e-10, atol=1e-10)


def test_not_invariant_to_per_key_scaling():
    """Scaling one key changes its weight by c^2: the result must move (guards
    against an implementation that normalises k internally)."""
    q, k, v = _rand(B=1, H=1, T=10, p=3, dv=2, seed=12)
    k2 = k.copy()
    k2[0, 0, 3] *= 5.0
    assert np.abs(oracle.direct(q, k2, v) - oracle.direct(q, k, v))[0, 0, 3:].max() > 1e-3


# ---------------------------------------------------------------------------
# state semantics of the recurrence (checkpoint / resume, decode)
# ---------------------------------------------------------------------------

def test_split_and_resume_and_final_state():
    q, k, v = _rand(B=2, H=1, T=31, p=4, dv=3, seed=13)
    o_full, S_full, z_full = oracle.recurrent(q, k, v, return_state=True)
    t0 = 12
    o1, S1, z1 = oracle.recurrent(q[:, :, :t0], k[:, :, :t0], v[:, :, :t0], return_state=True)
    o2, S2, z2 = oracle.recurrent(q[:, :, t0:], k[:, :, t0:], v[:, :, t0:], S1, z1, return_state=True)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), o_full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S_full, rtol=1e-12, atol=1e-12)
    # the final state is the sum of outer products psi(k_s) v_s^T; check one
    # entry by brute force with explicit indices (i, j, e)
    i, j, e = 2, 1, 0
    want = sum(k[0, 0, s, i] * k[0, 0, s, j] * v[0, 0, s, e] for s in range(31))
    assert abs(S_full[0, 0, i * 4 + j, e] - want) < 1e-12
    assert abs(z_full[0, 0, i * 4 + j] - sum(k[0, 0, s, i] * k[0, 0, s, j] for s in range(31))) < 1e-12
    # decode step continues the sequence
    o_dec, S3, z3 = oracle.decode_step(q[:, :, -1], k[:, :, -1], v[:, :, -1], S_full, z_full)
    qe = np.concatenate([q, q[:, :, -1:]], axis=2)
    ke = np.concatenate([k, k[:, :, -1:]], axis=2)
    ve = np.concatenate([v, v[:, :, -1:]], axis=2)
    np.testing.assert_allclose(o_dec, oracle.direct(qe, ke, ve)[:, :, -1], rtol=1e-11, atol=1e-12)


def test_direct_rows_matches_full_and_threads_do_not_matter():
    q, k, v = _rand(B=2, H=3, T=45, p=4, dv=3, seed=14)
    o = oracle.direct(q, k, v, nthreads=1)
    o4 = oracle.direct(q, k, v, nthreads=4)
    np.testing.assert_array_equal(o, o4)
    bh = np.array([0, 5, 3, 2])
    t = np.array([0, 44, 17, 30])
    rows = oracle.direct_rows(q, k, v, bh, t)
    np.testing.assert_array_equal(rows, o.reshape(6, 45, 3)[bh, t])
    np.testing.assert_array_equal(oracle.recurrent(q, k, v, nthreads=1), oracle.recurrent(q, k, v, nthreads=3))


def test_workload_inputs_shapes_and_bf16_rounding():
    cfg = workloads.CONFIGS["tiny"]
    q, k, v = workloads.make_inputs(cfg)
    assert q.shape == (1, 1, 256, 16) and v.shape == (1, 1, 256, 16)
    np.testing.assert_allclose(np.linalg.norm(q, axis=-1), 1.0, rtol=1e-6)
    qb, kb, vb = workloads.normal_qkv(1, 2, 64, 16, 64, seed=1, dtype="bf16")
    bits = qb.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)  # representable in bfloat16
    # round-to-nearest-even on a few hand-picked cases
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5], np.float32)
    np.testing.assert_array_equal(workloads.round_bf16(x), np.array([1.0, 1.0, 1.0 + 2 ** -7, -2.5], np.float32))
    qr, kr, vr = workloads.recall_qkv(1, 1, 2048, 32, 8, seed=3, dtype="f32")
    # each codeword appears exactly twice per block of 1024 tokens
    blk = kr[0, 0, :1024]
    _, counts = np.unique(blk.round(6), axis=0, return_counts=True)
    assert counts.min() == 2 and counts.max() == 2 and len(counts) == 512


# ---------------------------------------------------------------------------
# mutation check: slips planted in copies of the oracle's C source must fail
# the pins above (the planted copy is compiled to a temporary library; the
# committed oracle is never modified)
# ---------------------------------------------------------------------------

MUTATIONS = {
    "exclusive causal sum": ("for (int64_t s = 0; s <= t; ++s) {\n    const double *k_s", "for (int64_t s = 0; s < t; ++s) {\n    const double *k_s"),
    "unsquared score": ("double w = dot * dot;", "double w = dot;"),
    "missing normalisation": ("o_t[e] = (D > 0.0) ? N[e] / D : 0.0;", "o_t[e] = N[e];"),
    "transposed operands": ("dot += q_t[i] * k_s[i];", "dot += q_t[i] * (k_s[i] + (i == 0 ? k_s[1] - k_s[0] : 0.0));"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kata_oracle.c")).read()
    assert old in src, name
    path = tmp_path / ("mut_%d.c" % abs(hash(name)))
    path.write_text(src.replace(old, new, 1))
    so = str(path) + ".so"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
                           "-o", so, str(path), "-lpthread"])
    lib = ctypes.CDLL(so)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kata_oracle_direct.argtypes = [dp, dp, dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int]
    return lib


def _mutant_direct(lib, q, k, v):
    q, k, v = (np.ascontiguousarray(x, np.float64) for x in (q, k, v))
    B, H, T, p = q.shape
    dv = v.shape[3]
    o = np.empty((B, H, T, dv))
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kata_oracle_direct(q.ctypes.data_as(dp), k.ctypes.data_as(dp), v.ctypes.data_as(dp),
                           o.ctypes.data_as(dp), B, H, T, p, dv, 1)
    return o


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistakes(tmp_path, name):
    old, new = MUTATIONS[name]
    lib = _build_mutant(tmp_path, name, old, new)
    q, k, v, o_expected = _read_golden("worked_example_p2.txt")
    caught = not np.allclose(_mutant_direct(lib, q, k, v), o_expected, atol=1e-12)
    qr, kr, vr = _rand(B=1, H=1, T=20, p=4, dv=3, seed=30)
    o = _mutant_direct(lib, qr, kr, vr)
    caught = caught or not np.allclose(o[:, :, 0], vr[:, :, 0], atol=1e-12)
    lo, hi = np.minimum.accumulate(vr, axis=2), np.maximum.accumulate(vr, axis=2)
    caught = caught or not (np.all(o >= lo - 1e-12) and np.all(o <= hi + 1e-12))
    assert caught, "pin set failed to catch: " + name


# ---------------------------------------------------------------------------
# KATA-Mg (g PSD factors over a head of width d): pins of the grouped oracle
# ---------------------------------------------------------------------------

def _rand_mg(B=1, H=2, T=30, d=8, dv=3, seed=40):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, T, d)), rng.standard_normal((B, H, T, d)),
            rng.standard_normal((B, H, T, dv)))


def test_mg_one_group_is_the_full_map():
    """g = 1 is the full rank-one map (ai.info, Main Findings: both reduced
    families recover the full map at g = 1)."""
    q, k, v = _rand_mg(d=6, seed=41)
    np.testing.assert_allclose(oracle.direct_mg(q, k, v, 1), oracle.direct(q, k, v), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("d,g", [(8, 2), (8, 4), (12, 3), (6, 6)])
def test_mg_direct_equals_recurrent(d, g):
    q, k, v = _rand_mg(d=d, seed=42 + d + g)
    np.testing.assert_allclose(oracle.recurrent_mg(q, k, v, g), oracle.direct_mg(q, k, v, g),
                               rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("j0", [0, 2])
def test_mg_single_active_group_reduces_to_one_factor(j0):
    """With every query group but j0 zero, only (q^j0 . k^j0)^2 is left: the
    single-factor oracle on the j0 slices, whatever the other key groups hold."""
    d, g = 12, 3
    p = d // g
    q, k, v = _rand_mg(d=d, seed=50 + j0)
    qz = np.zeros_like(q)
    qz[..., j0 * p:(j0 + 1) * p] = q[..., j0 * p:(j0 + 1) * p]
    want = oracle.direct(qz[..., j0 * p:(j0 + 1) * p], k[..., j0 * p:(j0 + 1) * p], v)
    np.testing.assert_allclose(oracle.direct_mg(qz, k, v, g), want, rtol=1e-11, atol=1e-12)


def test_mg_width_one_groups_closed_form():
    """g = d (groups of width 1): w_ts = sum_i q_i^2 k_i^2, i.e. first-order
    linear attention with the feature u -> u*u, evaluated by cumulative sums."""
    rng = np.random.default_rng(60)
    T, d, dv = 30, 5, 3
    q = rng.standard_normal((1, 1, T, d))
    k = rng.standard_normal((1, 1, T, d))
    v = rng.standard_normal((1, 1, T, dv))
    fq, fk = q[0, 0] ** 2, k[0, 0] ** 2
    S = np.cumsum(fk[:, :, None] * v[0, 0][:, None, :], axis=0)  # [T, d, dv]
    z = np.cumsum(fk, axis=0)
    want = np.einsum("ti,tie->te", fq, S) / np.einsum("ti,ti->t", fq, z)[:, None]
    np.testing.assert_allclose(oracle.direct_mg(q, k, v, d)[0, 0], want, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(oracle.recurrent_mg(q, k, v, d)[0, 0], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("d,g", [(8, 1), (8, 2), (8, 4), (12, 3)])
def test_mg_feature_dimension_matches_state_size_formula(d, g):
    """The psi_Mg features of random vectors span exactly d(d/g+1)/2
    dimensions, the packed KATA-Mg state width per value column (ai.info,
    Main Findings).  A cross-group product or a dropped group changes it."""
    rng = np.random.default_rng(70 + d + g)
    p = d // g
    P = g * p * p
    n = 3 * P
    u = rng.standard_normal((1, n, d))
    # from the zero state one step leaves z = psi_Mg(k)
    _, _, z = oracle.decode_step_mg(u, u, np.ones((1, n, 1)), np.zeros((1, n, P, 1)), np.zeros((1, n, P)), g)
    assert np.linalg.matrix_rank(z[0]) == d * (d // g + 1) // 2


def test_mg_gate_properties_and_group_permutation():
    d, g = 8, 4
    p = d // g
    q, k, v = _rand_mg(T=25, d=d, seed=80)
    o = oracle.direct_mg(q, k, v, g)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=1e-12, atol=1e-12)   # o_1 = v_1
    lo, hi = np.minimum.accumulate(v, axis=2), np.maximum.accumulate(v, axis=2)
    assert np.all(o >= lo - 1e-12) and np.all(o <= hi + 1e-12)                  # convex gate
    kk = np.broadcast_to(k[:, :, :1], k.shape)                                    # identical keys
    want = np.cumsum(v, axis=2) / np.arange(1, v.shape[2] + 1)[None, None, :, None]
    np.testing.assert_allclose(oracle.direct_mg(q, kk, v, g), want, rtol=1e-11, atol=1e-12)
    perm = np.concatenate([np.arange(j * p, (j + 1) * p) for j in (2, 0, 3, 1)])
    np.testing.assert_allclose(oracle.direct_mg(q[..., perm], k[..., perm], v, g), o, rtol=1e-11, atol=1e-12)


MUTATIONS_MG = {
    "cross-group products": ("dot += q_t[j * p + i] * k_s[j * p + i];",
                             "dot += q_t[j * p + i] * k_s[((j + 1) % g) * p + i];"),
    "last group dropped": ("for (int j = 0; j < g; ++j) {\n    double dot", "for (int j = 0; j < g - 1; ++j) {\n    double dot"),
    "squared sum instead of sum of squares": ("    w += dot * dot;\n  }\n  return w;", "    w += dot;\n  }\n  return w * w;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS_MG))
def test_mg_pins_catch_planted_mistakes(tmp_path, name):
    old, new = MUTATIONS_MG[name]
    lib = _build_mutant(tmp_path, name, old, new)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kata_oracle_direct_mg.argtypes = [dp, dp, dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]

    def mutant(q, k, v, g):
        q, k, v = (np.ascontiguousarray(x, np.float64) for x in (q, k, v))
        B, H, T, d = q.shape
        o = np.empty((B, H, T, v.shape[3]))
        lib.kata_oracle_direct_mg(q.ctypes.data_as(dp), k.ctypes.data_as(dp), v.ctypes.data_as(dp),
                                  o.ctypes.data_as(dp), B, H, T, d, g, v.shape[3], 1)
        return o

    d, g, p = 12, 3, 4
    q, k, v = _rand_mg(d=d, seed=90)
    caught = False
    # the single-active-group reduction, for the first and the last group
    for j0 in (0, g - 1):
        qz = np.zeros_like(q)
        qz[..., j0 * p:(j0 + 1) * p] = q[..., j0 * p:(j0 + 1) * p]
        want = oracle.direct(qz[..., j0 * p:(j0 + 1) * p], k[..., j0 * p:(j0 + 1) * p], v)
        caught = caught or not np.allclose(mutant(qz, k, v, g), want, atol=1e-10)
    # the width-one closed form
    q1, k1, v1 = _rand_mg(B=1, H=1, T=20, d=5, seed=91)
    fq, fk = q1[0, 0] ** 2, k1[0, 0] ** 2
    S = np.cumsum(fk[:, :, None] * v1[0, 0][:, None, :], axis=0)
    want = np.einsum("ti,tie->te", fq, S) / np.einsum("ti,ti->t", fq, np.cumsum(fk, axis=0))[:, None]
    caught = caught or not np.allclose(mutant(q1, k1, v1, 5)[0, 0], want, atol=1e-10)
    assert caught, "Mg pin set failed to catch: " + name


# ---------------------------------------------------------------------------
# backward pass: pins of the fp64 gradient oracle
# ---------------------------------------------------------------------------

from oracle import backward as obw  # noqa: E402


def _loss(q, k, v, dO):
    return float((oracle.direct(q, k, v) * dO).sum())


def test_backward_forward_matches_direct():
    q, k, v = _rand(B=1, H=2, T=30, p=5, dv=3, seed=101)
    o, D = obw.forward_with_d(q, k, v)
    np.testing.assert_allclose(o, oracle.direct(q, k, v), rtol=1e-11, atol=1e-12)
    _, d_rows = oracle.direct_rows(q, k, v, np.zeros(30, np.int64), np.arange(30), return_d=True)
    np.testing.assert_allclose(D[0, 0], d_rows, rtol=1e-12)


def test_backward_matches_finite_differences():
    """Central differences of the (independently pinned) C direct-sum oracle."""
    rng = np.random.default_rng(102)
    q, k, v = _rand(B=1, H=1, T=7, p=3, dv=2, seed=103)
    dO = rng.standard_normal(v.shape)
    dq, dk, dv = obw.backward(q, k, v, dO)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], dO)
                        - _loss(args_m["q"], args_m["k"], args_m["v"], dO)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_identities():
    """o_t is invariant to scaling q_t, to scaling all keys, and shifts with
    v: so q_t . dq_t = 0, sum_s k_s . dk_s = 0 and sum_s dv_s = sum_t dO_t."""
    rng = np.random.default_rng(104)
    q, k, v = _rand(B=2, H=2, T=40, p=6, dv=4, seed=105)
    dO = rng.standard_normal(v.shape)
    dq, dk, dv = obw.backward(q, k, v, dO)
    np.testing.assert_allclose(np.einsum("bhtp,bhtp->bht", q, dq), 0.0, atol=1e-9)
    np.testing.assert_allclose(np.einsum("bhsp,bhsp->bh", k, dk), 0.0, atol=1e-9)
    np.testing.assert_allclose(dv.sum(axis=2), dO.sum(axis=2), rtol=1e-10, atol=1e-10)
    # a row whose query is zero has D_t = 0: its output is the constant 0
    q0 = q.copy()
    q0[:, :, 7] = 0.0
    dq0, _, _ = obw.backward(q0, k, v, dO)
    assert np.all(dq0[:, :, 7] == 0.0)


def test_backward_mg_pins():
    """KATA-Mg gradients: g = 1 equals the single-factor gradients, the Mg
    forward equals the C Mg oracle, and central differences of the C Mg
    oracle match; scaling a whole query row leaves its output unchanged, so
    q_t . dq_t = 0 row by row."""
    q, k, v = _rand_mg(B=1, H=1, T=6, d=4, dv=2, seed=480)
    rng = np.random.default_rng(481)
    dO = rng.standard_normal(v.shape)
    for a, b in zip(obw.backward_mg(q, k, v, dO, 1), obw.backward(q, k, v, dO)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    o, _ = obw.forward_mg_with_d(q, k, v, 2)
    np.testing.assert_allclose(o, oracle.direct_mg(q, k, v, 2), rtol=1e-11, atol=1e-12)
    dq, dk, dv = obw.backward_mg(q, k, v, dO, 2)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            ap = {"q": q, "k": k, "v": v}
            am = dict(ap)
            ap[name], am[name] = xp, xm
            num[idx] = ((oracle.direct_mg(ap["q"], ap["k"], ap["v"], 2) * dO).sum()
                        - (oracle.direct_mg(am["q"], am["k"], am["v"], 2) * dO).sum()) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=name)
    q2, k2, v2 = _rand_mg(B=1, H=2, T=30, d=8, dv=3, seed=482)
    dq2, _, _ = obw.backward_mg(q2, k2, v2, rng.standard_normal(v2.shape), 2)
    np.testing.assert_allclose(np.einsum("bhtd,bhtd->bht", q2, dq2), 0.0, atol=1e-9)


# ---------------------------------------------------------------------------
# KATA-Sigma-g (summed factors): pins of the numpy oracle
# ---------------------------------------------------------------------------

from oracle import sigma_g as osg  # noqa: E402


def test_sigma_g_pins():
    q, k, v = _rand_mg(B=1, H=2, T=20, d=8, dv=3, seed=500)
    # g = 1 is the full rank-one map
    np.testing.assert_allclose(osg.direct_sg(q, k, v, 1), oracle.direct(q, k, v), rtol=1e-11, atol=1e-12)
    # the two forms agree
    for g in (2, 4):
        np.testing.assert_allclose(osg.recurrent_sg(q, k, v, g), osg.direct_sg(q, k, v, g), rtol=1e-10, atol=1e-12)
    # the weight pairs every query group with every key group: permuting the
    # query's groups alone changes nothing (it would for KATA-Mg)
    perm = np.concatenate([np.arange(4, 8), np.arange(0, 4)])
    np.testing.assert_allclose(osg.direct_sg(q[..., perm], k, v, 2), osg.direct_sg(q, k, v, 2), rtol=1e-11, atol=1e-12)
    assert np.abs(oracle.direct_mg(q[..., perm], k, v, 2) - oracle.direct_mg(q, k, v, 2)).max() > 1e-3
    # width-one groups: w = |q|^2 |k|^2, so o_t is the |k|^2-weighted running
    # mean of v whatever q_t (!= 0) is
    q1, k1, v1 = _rand_mg(B=1, H=1, T=15, d=3, dv=2, seed=501)
    kk = (k1[0, 0] ** 2).sum(-1)
    want = np.cumsum(kk[:, None] * v1[0, 0], axis=0) / np.cumsum(kk)[:, None]
    np.testing.assert_allclose(osg.direct_sg(q1, k1, v1, 3)[0, 0], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("d,g", [(8, 2), (8, 4), (12, 3)])
def test_sigma_g_feature_dimension_matches_state_size_formula(d, g):
    """The summed features span (d/g)(d/g+1)/2 dimensions: the KATA-Sigma-g
    state width per value column (ai.info, Main Findings)."""
    rng = np.random.default_rng(510 + d + g)
    p = d // g
    f = osg.features_sg(rng.standard_normal((3 * p * p, d)), g)
    assert np.linalg.matrix_rank(f) == p * (p + 1) // 2


# ---------------------------------------------------------------------------
# first-order (psi(u) = u) attention: pins of the numpy oracle
# ---------------------------------------------------------------------------

from oracle import first_order as ofo  # noqa: E402

# Worked example, by hand (d = 1, dv = 1): q = (1, 1, 2), k = (1, 2, -1),
# v = (3, 5, 7).
#   t = 0: w = (1)            -> 3 / 1                  = 3
#   t = 1: w = (1, 2)         -> (3 + 10) / 3           = 13/3
#   t = 2: w = (2, 4, -2)     -> (6 + 20 - 14) / 4      = 3
FO_Q, FO_K, FO_V = [1.0, 1.0, 2.0], [1.0, 2.0, -1.0], [3.0, 5.0, 7.0]
FO_WANT = [3.0, 13.0 / 3.0, 3.0]


def _fo_pins_hold(mod) -> bool:
    """The pin set of the first-order oracle, as one predicate (used on the
    oracle itself and on copies with planted mistakes)."""
    ok = True
    q = np.array(FO_Q).reshape(1, 1, 3, 1)
    k = np.array(FO_K).reshape(1, 1, 3, 1)
    v = np.array(FO_V).reshape(1, 1, 3, 1)
    for fn in (mod.direct_linear, mod.recurrent_linear):
        ok = ok and np.allclose(fn(q, k, v)[0, 0, :, 0], FO_WANT, rtol=0, atol=1e-13)
        # zero denominator: q = (1, 1), k = (1, -1) -> D_1 = 0 -> o_1 = 0
        o = fn(np.ones((1, 1, 2, 1)), np.array([1.0, -1.0]).reshape(1, 1, 2, 1), np.array([2.0, 4.0]).reshape(1, 1, 2, 1))
        ok = ok and np.allclose(o[0, 0, :, 0], [2.0, 0.0], rtol=0, atol=1e-13)
        # the first output is the first value whenever q_0 . k_0 != 0, also
        # when it is negative: q_0 . k_0 = 1*(-3) + 2*1 = -1
        o = fn(np.array([1.0, 2.0]).reshape(1, 1, 1, 2), np.array([-3.0, 1.0]).reshape(1, 1, 1, 2),
               np.array([3.0, -4.0]).reshape(1, 1, 1, 2))
        ok = ok and np.allclose(o[0, 0, 0], [3.0, -4.0], rtol=0, atol=1e-13)
    # the KATA weight is the first-order weight of the features vec(u u^T):
    # first-order attention on psi(q), psi(k) is the (independently pinned)
    # C oracle's KATA attention on q, k
    q, k, v = _rand(B=1, H=2, T=23, p=3, dv=2, seed=600)
    psi = lambda u: np.einsum("bhti,bhtj->bhtij", u, u).reshape(u.shape[:3] + (u.shape[3] ** 2,))  # noqa: E731
    for fn in (mod.direct_linear, mod.recurrent_linear):
        ok = ok and np.allclose(fn(psi(q), psi(k), v), oracle.direct(q, k, v), rtol=1e-10, atol=1e-12)
    return bool(ok)


def test_first_order_pins():
    assert _fo_pins_hold(ofo)


@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (2, 3, 37, 4, 5), (1, 2, 64, 16, 8)])
def test_first_order_direct_equals_recurrent(shape):
    B, H, T, d, dv = shape
    q, k, v = _rand(B, H, T, d, dv, seed=610 + T)
    np.testing.assert_allclose(ofo.recurrent_linear(q, k, v), ofo.direct_linear(q, k, v), rtol=1e-9, atol=1e-11)


def test_first_order_state_split_and_invariances():
    q, k, v = _rand(B=2, H=2, T=30, p=4, dv=3, seed=620)
    o, S, z = ofo.recurrent_linear(q, k, v, return_state=True)
    # final state closed form: S_T = sum_t k_t v_t^T, z_T = sum_t k_t
    np.testing.assert_allclose(S, np.einsum("bhtd,bhte->bhde", k, v), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, k.sum(axis=2), rtol=1e-12, atol=1e-12)
    # split and resume from the state after 11 tokens
    _, S1, z1 = ofo.recurrent_linear(q[:, :, :11], k[:, :, :11], v[:, :, :11], return_state=True)
    o2 = ofo.recurrent_linear(q[:, :, 11:], k[:, :, 11:], v[:, :, 11:], S0=S1, z0=z1)
    np.testing.assert_allclose(o2, o[:, :, 11:], rtol=1e-10, atol=1e-12)
    # o is unchanged by scaling a query, or all keys, by any c != 0 (the
    # numerator and the denominator scale together), but not by scaling one key
    for c in (3.0, -0.5):
        np.testing.assert_allclose(ofo.direct_linear(c * q, k, v), o, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(ofo.direct_linear(q, c * k, v), o, rtol=1e-9, atol=1e-11)
    k2 = k.copy()
    k2[:, :, 5] *= 4.0
    assert np.abs(ofo.direct_linear(q, k2, v) - o)[:, :, 5:].max() > 1e-3


MUTATIONS_FO = {
    "exclusive causal sum": [("np.tril(np.ones((T, T), dtype=bool))", "np.tril(np.ones((T, T), dtype=bool), k=-1)"),
                             ("    for t in range(T):\n        S += k[:, :, t, :, None] * v[:, :, t, None, :]\n"
                              "        z += k[:, :, t]\n        N = np.einsum(\"bhd,bhde->bhe\", q[:, :, t], S)\n"
                              "        D = np.einsum(\"bhd,bhd->bh\", q[:, :, t], z)\n",
                              "    for t in range(T):\n        N = np.einsum(\"bhd,bhde->bhe\", q[:, :, t], S)\n"
                              "        D = np.einsum(\"bhd,bhd->bh\", q[:, :, t], z)\n"
                              "        S += k[:, :, t, :, None] * v[:, :, t, None, :]\n        z += k[:, :, t]\n")],
    "squared weights": [("W = np.where(np.tril(np.ones((T, T), dtype=bool)), W, 0.0)",
                         "W = np.where(np.tril(np.ones((T, T), dtype=bool)), W * W, 0.0)"),
                        ("        z += k[:, :, t]\n", "        z += k[:, :, t] * k[:, :, t]\n")],
    "no normalisation": [("    return _div(N, W.sum(axis=-1))", "    return N"),
                         ("        o[:, :, t] = _div(N, D)", "        o[:, :, t] = N")],
    "query and key swapped": [("\"bhtd,bhsd->bhts\", q, k", "\"bhtd,bhsd->bhts\", k, q"),
                              ("np.einsum(\"bhd,bhde->bhe\", q[:, :, t], S)", "np.einsum(\"bhd,bhde->bhe\", k[:, :, t], S)")],
    "negative denominators zeroed": [("    nz = D != 0", "    nz = D > 0")],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS_FO))
def test_first_order_pins_catch_planted_mistakes(name):
    import inspect
    import types
    src = inspect.getsource(ofo)
    for old, new in MUTATIONS_FO[name]:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    mutant = types.ModuleType("first_order_mutant")
    exec(compile(src, "first_order_mutant", "exec"), mutant.__dict__)
    assert not _fo_pins_hold(mutant), "first-order pin set failed to catch: " + name


def test_sigma_g_decode_step_pins():
    """One decode step from the state after tokens 0..t-1 gives the
    recurrence's output at token t and its state after t; g = 1 is the C
    oracle's single-factor step."""
    q, k, v = _rand_mg(B=2, H=2, T=9, d=8, dv=3, seed=520)
    for g in (2, 4):
        p = 8 // g
        fk = osg.features_sg(k, g)
        S = np.einsum("bhtp,bhte->bhpe", fk[:, :, :8], v[:, :, :8])
        z = fk[:, :, :8].sum(axis=2)
        o, S2, z2 = osg.decode_step_sg(q[:, :, 8], k[:, :, 8], v[:, :, 8], S, z, g)
        np.testing.assert_allclose(o, osg.recurrent_sg(q, k, v, g)[:, :, 8], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(S2, np.einsum("bhtp,bhte->bhpe", fk, v), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(z2, fk.sum(axis=2), rtol=1e-12, atol=1e-12)
        assert S2.shape == (2, 2, p * p, 3)
    rng = np.random.default_rng(521)
    S = rng.standard_normal((2, 2, 64, 3))
    z = np.abs(rng.standard_normal((2, 2, 64))) + 1.0
    o1, S1, z1 = osg.decode_step_sg(q[:, :, 0], k[:, :, 0], v[:, :, 0], S, z, 1)
    o2, S2, z2 = oracle.decode_step(q[:, :, 0], k[:, :, 0], v[:, :, 0], S, z)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-12)


def test_backward_sg_pins():
    """KATA-Sigma-g gradients: g = 1 equals the single-factor gradients, the
    forward equals the Sigma-g oracle, central differences of that oracle
    match, and scaling a whole query row leaves its output unchanged, so
    q_t . dq_t = 0 row by row (likewise for a key row only through the
    normalisation, which is not a pin)."""
    q, k, v = _rand_mg(B=1, H=1, T=6, d=4, dv=2, seed=490)
    rng = np.random.default_rng(491)
    dO = rng.standard_normal(v.shape)
    for a, b in zip(obw.backward_sg(q, k, v, dO, 1), obw.backward(q, k, v, dO)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    o, _ = obw.forward_sg_with_d(q, k, v, 2)
    np.testing.assert_allclose(o, osg.direct_sg(q, k, v, 2), rtol=1e-11, atol=1e-12)
    dq, dk, dv = obw.backward_sg(q, k, v, dO, 2)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            ap = {"q": q, "k": k, "v": v}
            am = dict(ap)
            ap[name], am[name] = xp, xm
            num[idx] = ((osg.direct_sg(ap["q"], ap["k"], ap["v"], 2) * dO).sum()
                        - (osg.direct_sg(am["q"], am["k"], am["v"], 2) * dO).sum()) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7, err_msg=name)
    q2, k2, v2 = _rand_mg(B=1, H=2, T=30, d=8, dv=3, seed=492)
    dq2, _, _ = obw.backward_sg(q2, k2, v2, rng.standard_normal(v2.shape), 2)
    np.testing.assert_allclose(np.einsum("bhtd,bhtd->bht", q2, dq2), 0.0, atol=1e-9)

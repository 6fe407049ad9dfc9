"""fp64 CPU oracle for the KATA forward pass (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
and never calls it; the product path does not import it.

The arithmetic lives in ``kata_oracle.c`` (plain C, fp64, pthreads over
(batch, head) pairs).  This module compiles it with gcc on first use and
marshals numpy arrays through ctypes.  Functions:

* :func:`direct` -- the defining double sum
  o_t = sum_{s<=t} (q_t.k_s)^2 v_s / sum_{s<=t} (q_t.k_s)^2
  (gist.science technical summary, sec. 2.1 "Output Gating" and sec. 2.2
  "PSD Kegel (Rank-One)"; ai.info summary, Main Findings).
* :func:`direct_rows` -- the same sum on selected (bh, t) rows.
* :func:`recurrent` -- the explicit psi(u)=vec(uu^T) state recurrence
  S_t = S_{t-1} + psi(k_t) v_t^T, z_t = z_{t-1} + psi(k_t),
  o_t = psi(q_t)^T S_t / psi(q_t)^T z_t, with optional initial and final
  state (ai.info summary, Methodology in Plain English).
* :func:`decode_step` -- one step of that recurrence from a given state.
* :func:`direct_mg`, :func:`direct_mg_rows`, :func:`recurrent_mg`,
  :func:`decode_step_mg` -- the same for KATA-Mg: the head's d coordinates
  split into g groups of width d/g, weight sum_j (q_t^j . k_s^j)^2, one
  shared value vector and denominator, state [g*(d/g)^2, dv] (arXiv
  abstract; gist.science sec. 2.3 "Varianten"; ai.info Main Findings, the
  KATA-Mg state size d(d/g+1)/2 * dv).

Readings (the pages leave these open): inclusive causal sum (s <= t);
D_t = 0 gives o_t = 0; no score scaling; q, k used as given.

Every pin of these functions lives in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kata_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkata_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile kata_oracle.c into libkata_oracle.so beside it (gcc -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.kata_oracle_direct.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                               ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            lib.kata_oracle_direct_rows.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                                    ctypes.c_int, ctypes.c_int, _ip, _ip, ctypes.c_int64,
                                                    _dp, _dp]
            lib.kata_oracle_recurrent.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                                  ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                                  _dp, _dp, _dp, _dp, ctypes.c_int]
            lib.kata_oracle_direct_mg.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                                  ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int]
            lib.kata_oracle_direct_mg_rows.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip, _ip,
                                                       ctypes.c_int64, _dp, _dp]
            lib.kata_oracle_recurrent_mg.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                                     ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     _dp, _dp, _dp, _dp, ctypes.c_int]
            lib.kata_oracle_default_threads.argtypes = []
            for f in (lib.kata_oracle_direct, lib.kata_oracle_direct_rows, lib.kata_oracle_recurrent,
                      lib.kata_oracle_direct_mg, lib.kata_oracle_direct_mg_rows, lib.kata_oracle_recurrent_mg,
                      lib.kata_oracle_default_threads):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def default_threads() -> int:
    """Threads the oracle uses when ``nthreads`` is 0 (one per online CPU)."""
    return int(_load().kata_oracle_default_threads())


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _check(rc):
    if rc != 0:
        raise ValueError("oracle returned error %d" % rc)


def _shape(q, k, v):
    if q.ndim != 4 or k.shape != q.shape or v.ndim != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("expected q,k [B,H,T,p] and v [B,H,T,dv]")
    B, H, T, p = q.shape
    return B, H, T, p, v.shape[3]


def direct(q, k, v, nthreads: int = 0) -> np.ndarray:
    """o [B,H,T,dv] from the defining double sum (fp64)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, p, dv = _shape(q, k, v)
    o = np.empty((B, H, T, dv), np.float64)
    _check(_load().kata_oracle_direct(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, T, p, dv, nthreads))
    return o


def direct_rows(q, k, v, bh_idx, t_idx, return_d: bool = False):
    """Direct sum on rows (bh_idx[r], t_idx[r]); bh = b*H + h.  Returns o_rows [R,dv] (and D [R])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, p, dv = _shape(q, k, v)
    bh_idx = np.ascontiguousarray(bh_idx, dtype=np.int64)
    t_idx = np.ascontiguousarray(t_idx, dtype=np.int64)
    if bh_idx.shape != t_idx.shape or bh_idx.ndim != 1:
        raise ValueError("bh_idx and t_idx must be 1-D of equal length")
    R = bh_idx.shape[0]
    o = np.empty((R, dv), np.float64)
    d = np.empty((R,), np.float64) if return_d else None
    _check(_load().kata_oracle_direct_rows(_ptr(q), _ptr(k), _ptr(v), B * H, T, p, dv,
                                           bh_idx.ctypes.data_as(_ip), t_idx.ctypes.data_as(_ip), R,
                                           _ptr(o), _ptr(d)))
    return (o, d) if return_d else o


def recurrent(q, k, v, S0=None, z0=None, return_state: bool = False, need_output: bool = True,
              nthreads: int = 0):
    """Explicit psi recurrence (fp64).

    S0 [B,H,p*p,dv] and z0 [B,H,p*p] are the state before the first token
    (both or neither).  Returns o [B,H,T,dv] (None if need_output is False),
    and (S_T, z_T) when return_state is True.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, p, dv = _shape(q, k, v)
    P = p * p
    if (S0 is None) != (z0 is None):
        raise ValueError("give both S0 and z0 or neither")
    if S0 is not None:
        S0 = _f64(S0).reshape(B, H, P, dv)
        z0 = _f64(z0).reshape(B, H, P)
    o = np.empty((B, H, T, dv), np.float64) if need_output else None
    S_out = np.empty((B, H, P, dv), np.float64) if return_state else None
    z_out = np.empty((B, H, P), np.float64) if return_state else None
    _check(_load().kata_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, T, p, dv,
                                         _ptr(S0), _ptr(z0), _ptr(S_out), _ptr(z_out), nthreads))
    if return_state:
        return o, S_out, z_out
    return o


def decode_step(q, k, v, S, z, nthreads: int = 0):
    """One recurrent step: q,k [B,H,p], v [B,H,dv], S [B,H,p*p,dv], z [B,H,p*p].

    The state is updated with (k, v) first, then read with q (inclusive, as in
    the causal sum).  Returns (o [B,H,dv], S_new, z_new).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    o, S1, z1 = recurrent(q[:, :, None, :], k[:, :, None, :], v[:, :, None, :], S, z,
                          return_state=True, nthreads=nthreads)
    return o[:, :, 0, :], S1, z1


# ---------------------------------------------------------------------------
# KATA-Mg: g PSD factors over a head of width d
# ---------------------------------------------------------------------------

def _shape_mg(q, k, v, groups):
    B, H, T, d, dv = _shape(q, k, v)
    if groups < 1 or d % groups != 0:
        raise ValueError("groups must divide the head width d")
    return B, H, T, d, dv


def direct_mg(q, k, v, groups: int, nthreads: int = 0) -> np.ndarray:
    """o [B,H,T,dv] from the defining sum with w_ts = sum_j (q_t^j . k_s^j)^2 (fp64).

    q, k are [B,H,T,d]; group j is coordinates j*d/g .. (j+1)*d/g - 1.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d, dv = _shape_mg(q, k, v, groups)
    o = np.empty((B, H, T, dv), np.float64)
    _check(_load().kata_oracle_direct_mg(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, T, d, groups, dv, nthreads))
    return o


def direct_mg_rows(q, k, v, groups: int, bh_idx, t_idx, return_d: bool = False):
    """:func:`direct_mg` on rows (bh_idx[r], t_idx[r]).  Returns o_rows [R,dv] (and D [R])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d, dv = _shape_mg(q, k, v, groups)
    bh_idx = np.ascontiguousarray(bh_idx, dtype=np.int64)
    t_idx = np.ascontiguousarray(t_idx, dtype=np.int64)
    if bh_idx.shape != t_idx.shape or bh_idx.ndim != 1:
        raise ValueError("bh_idx and t_idx must be 1-D of equal length")
    R = bh_idx.shape[0]
    o = np.empty((R, dv), np.float64)
    dd = np.empty((R,), np.float64) if return_d else None
    _check(_load().kata_oracle_direct_mg_rows(_ptr(q), _ptr(k), _ptr(v), B * H, T, d, groups, dv,
                                              bh_idx.ctypes.data_as(_ip), t_idx.ctypes.data_as(_ip), R,
                                              _ptr(o), _ptr(dd)))
    return (o, dd) if return_d else o


def recurrent_mg(q, k, v, groups: int, S0=None, z0=None, return_state: bool = False, nthreads: int = 0):
    """Explicit psi_Mg recurrence (fp64) on the state [B,H,g*p*p,dv], p = d/g.

    Row r = j*p*p + a*p + b of the state belongs to group j and holds the
    products of its coordinates a and b.  Returns o, or (o, S_T, z_T).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d, dv = _shape_mg(q, k, v, groups)
    p = d // groups
    P = groups * p * p
    if (S0 is None) != (z0 is None):
        raise ValueError("give both S0 and z0 or neither")
    if S0 is not None:
        S0 = _f64(S0).reshape(B, H, P, dv)
        z0 = _f64(z0).reshape(B, H, P)
    o = np.empty((B, H, T, dv), np.float64)
    S_out = np.empty((B, H, P, dv), np.float64) if return_state else None
    z_out = np.empty((B, H, P), np.float64) if return_state else None
    _check(_load().kata_oracle_recurrent_mg(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, T, d, groups, dv,
                                            _ptr(S0), _ptr(z0), _ptr(S_out), _ptr(z_out), nthreads))
    if return_state:
        return o, S_out, z_out
    return o


def decode_step_mg(q, k, v, S, z, groups: int, nthreads: int = 0):
    """One Mg recurrent step: q,k [B,H,d], v [B,H,dv], S [B,H,g*p*p,dv], z [B,H,g*p*p].

    Update with (k, v) first, then read with q.  Returns (o [B,H,dv], S_new, z_new).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    o, S1, z1 = recurrent_mg(q[:, :, None, :], k[:, :, None, :], v[:, :, None, :], groups, S, z,
                             return_state=True, nthreads=nthreads)
    return o[:, :, 0, :], S1, z1

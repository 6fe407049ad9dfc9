"""kata_fwd_chunked_noalloc: the chunked forward for callers that cannot
allocate device memory -- a C host program with no allocator of its own, or
a loop that must not call cudaMalloc because it can block and synchronise
the device.  Its scratch space is a fixed array owned by the library
(KATA_NOALLOC_SCRATCH_BYTES, 16 MiB), shared by every call.

Both calls run the same plan and the same kernels as the allocating entry
point kata_fwd_chunked, so their results must agree bit for bit; one of them
is also checked against the fp64 oracle with the per-row metric of the other
parity tests.  The cases cover two calls in a row, an initial state, and a
shape whose workspace fills the array to within a few percent.  The file's
name makes pytest collect it last.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import workloads
from helpers import TOL, row_rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_scratch_bytes():
    """KATA_NOALLOC_SCRATCH_BYTES as include/kata.h states it."""
    text = open(os.path.join(ROOT, "include", "kata.h")).read()
    m = re.search(r"#define KATA_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m, "KATA_NOALLOC_SCRATCH_BYTES not found in kata.h"
    return int(m.group(1)) << int(m.group(2))


@pytest.fixture(scope="module")
def kata():
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return K


def _both(kata, qd, kd, vd, S0=None, z0=None):
    import torch
    o_ref, S_ref, z_ref = kata.kata_fwd_chunked(qd, kd, vd, C=64, S0=S0, z0=z0, return_state=True)
    o, S, z = kata.kata_fwd_chunked_noalloc(qd, kd, vd, C=64, S0=S0, z0=z0, return_state=True)
    torch.cuda.synchronize()
    assert kata.kata_get_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref) and torch.equal(z, z_ref)
    return o, S, z


@pytest.mark.parametrize("dtype,shape", [("bf16", (1, 2, 20000, 16, 64)), ("bf16", (2, 4, 1500, 16, 64)),
                                         ("f32", (1, 2, 700, 16, 16))])
def test_noalloc_matches_allocating_call_twice(kata, dtype, shape):
    B, H, T, p, dv = shape
    for seed in (21, 22):  # two calls in a row share the scratch array
        q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=seed, dtype=dtype)
        o, S, z = _both(kata, to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype))
        if seed == 21:
            o_ref = oracle.recurrent(q, k, v)
            assert row_rel_err(to_np(o), o_ref, v) <= TOL[dtype]


def test_noalloc_with_initial_state(kata):
    import torch
    B, H, T, p, dv = 1, 2, 20000, 16, 64  # several super-chunks: records in the scratch array
    q, k, v = workloads.normal_qkv(B, H, T + 300, p, dv, seed=23, dtype="bf16")
    _, S1, z1 = oracle.recurrent(q[:, :, :300], k[:, :, :300], v[:, :, :300], return_state=True)
    S0 = torch.from_numpy(S1.astype(np.float32)).cuda()
    z0 = torch.from_numpy(z1.astype(np.float32)).cuda()
    qd, kd, vd = (to_dev(x[:, :, 300:], "bf16") for x in (q, k, v))
    o, _, _ = _both(kata, qd, kd, vd, S0=S0, z0=z0)
    ref = oracle.recurrent(q, k, v)[:, :, 300:]
    assert row_rel_err(to_np(o), ref, v) <= TOL["bf16"]


def test_noalloc_shape_that_fills_the_array(kata):
    """fp32, p = 32: a record is 1024 x 68 floats; the largest H with T = 256
    whose workspace fits the array uses it to within a few percent, so the
    top of the array is written and read back."""
    from kernelized_feature_map_b200 import _abi
    cap = header_scratch_bytes()
    assert _abi.NOALLOC_SCRATCH_BYTES == cap
    T, p, dv = 256, 32, 64
    fits = [H for H in range(1, 64)
            if 0 < _abi.kata_fwd_chunked_workspace_size(1, H, T, p, dv, 64, dtype=_torch_f32()) <= cap]
    H = max(fits)
    need = _abi.kata_fwd_chunked_workspace_size(1, H, T, p, dv, 64, dtype=_torch_f32())
    assert need >= 0.95 * cap, (H, need)
    assert _abi.kata_fwd_chunked_workspace_size(1, H + 1, T, p, dv, 64, dtype=_torch_f32()) > cap
    q, k, v = workloads.normal_qkv(1, H, T, p, dv, seed=24, dtype="f32")
    o, _, _ = _both(kata, to_dev(q, "f32"), to_dev(k, "f32"), to_dev(v, "f32"))
    assert row_rel_err(to_np(o), oracle.recurrent(q, k, v), v) <= TOL["f32"]


def _torch_f32():
    import torch
    return torch.float32


def test_noalloc_rejects_sizes_beyond_the_array(kata):
    from kernelized_feature_map_b200 import _abi
    L = _abi.lib()
    need = _abi.kata_fwd_chunked_workspace_size(1, 512, 131072, 16, 64, 64)
    assert need > header_scratch_bytes()
    fake = ctypes.c_void_p(0x100000)
    rc = L.kata_fwd_chunked_noalloc(fake, fake, fake, fake, 1, 512, 131072, 16, 64, 64, _abi.KATA_BF16,
                                    None, None, None, None, ctypes.c_void_p(0))
    assert rc == _abi.KATA_ERR_WORKSPACE
    # argument errors come first, as for kata_fwd_chunked
    rc = L.kata_fwd_chunked_noalloc(None, fake, fake, fake, 1, 512, 131072, 16, 64, 64, _abi.KATA_BF16,
                                    None, None, None, None, ctypes.c_void_p(0))
    assert rc == _abi.KATA_ERR_INVALID_ARG

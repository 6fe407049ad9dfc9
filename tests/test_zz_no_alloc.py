"""kata_fwd_chunked_noalloc: the chunked forward for callers that cannot
allocate device memory (no allocator of their own, or a loop that must not
call cudaMalloc).  Its scratch space is a fixed 16 MiB array owned by the
library, shared by every call.

The test calls it through the C ABI twice in a row, with different inputs,
and checks each result against the allocating entry point kata_fwd_chunked
on the same inputs, within the tolerances of the other parity tests.  The
file's name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest

import workloads
from helpers import TOL, row_rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kata():
    import torch
    import kernelized_feature_map_b200 as K
    from kernelized_feature_map_b200 import build
    build.build()
    assert torch.cuda.is_available()
    return K


@pytest.mark.parametrize("dtype,shape", [("bf16", (2, 4, 1500, 16, 64)), ("f32", (1, 2, 700, 16, 16))])
def test_noalloc_matches_allocating_call_twice(kata, dtype, shape):
    import torch
    B, H, T, p, dv = shape
    for seed in (21, 22):  # two calls in a row share the scratch array
        q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=seed, dtype=dtype)
        qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
        o_ref, S_ref, z_ref = kata.kata_fwd_chunked(qd, kd, vd, C=64, return_state=True)
        o, S, z = kata.kata_fwd_chunked_noalloc(qd, kd, vd, C=64, return_state=True)
        torch.cuda.synchronize()
        assert kata.kata_get_status() == 0
        assert row_rel_err(to_np(o), to_np(o_ref).astype(np.float64), v) <= TOL[dtype]
        np.testing.assert_allclose(S.cpu().numpy(), S_ref.cpu().numpy(), rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(z.cpu().numpy(), z_ref.cpu().numpy(), rtol=1e-5, atol=1e-5)


def test_noalloc_rejects_sizes_beyond_the_array(kata):
    from kernelized_feature_map_b200 import _abi
    L = _abi.lib()
    need = _abi.kata_fwd_chunked_workspace_size(1, 512, 131072, 16, 64, 64)
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x100000)
    rc = L.kata_fwd_chunked_noalloc(fake, fake, fake, fake, 1, 512, 131072, 16, 64, 64, _abi.KATA_BF16,
                                    None, None, None, None, ctypes.c_void_p(0))
    assert rc == _abi.KATA_ERR_WORKSPACE

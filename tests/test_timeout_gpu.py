"""Failure detection without a GPU fault: every wait inside the tcgen05
kernels is bounded, and a wait that runs out records KATA_ERR_TIMEOUT in the
library's device status word, lets the copies and MMAs its CTA issued land,
frees its Tensor Memory and returns.

With the wait limit set to 0 cycles, any wait that is not already satisfied
gives up at once, so a call on a small case is certain to hit the path.  The
test checks that the call returns, that kata_get_status() reports the
timeout (and clears it), and that the next call with the default limit runs
normally and passes parity against the fp64 oracle.
"""
import numpy as np
import pytest

import oracle
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


# T = 1000 runs the chunked path as one super-chunk per head (a single
# readout launch); T = 20000 with two heads runs the state build, the scan
# and the readout
@pytest.mark.parametrize("path,T", [("quadratic", 1000), ("chunked", 1000), ("chunked", 20000)])
def test_short_wait_limit_reports_timeout_then_recovers(kata, path, T):
    import torch
    from kernelized_feature_map_b200 import _abi
    B, H, p, dv = 1, 2, 16, 64
    q, k, v = workloads.normal_qkv(B, H, T, p, dv, seed=41, dtype="bf16")
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")

    def call():
        if path == "quadratic":
            return kata.kata_fwd_quadratic(qd, kd, vd)
        return kata.kata_fwd_chunked(qd, kd, vd, C=64)

    torch.cuda.synchronize()
    assert kata.kata_get_status() == _abi.KATA_OK
    try:
        kata.kata_set_wait_limit(0)
        call()  # enqueues and returns: the launch itself succeeds
        status = kata.kata_get_status()
        assert status == _abi.KATA_ERR_TIMEOUT, _abi.status_string(status)
        assert kata.kata_get_status() == _abi.KATA_OK  # reading the status clears it
    finally:
        kata.kata_set_wait_limit(-1)
    o = call()
    torch.cuda.synchronize()
    assert kata.kata_get_status() == _abi.KATA_OK
    assert row_rel_err(to_np(o), oracle.direct(q, k, v), v) <= TOL["bf16"]

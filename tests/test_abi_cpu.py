"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/kata.h declares, and rejects bad arguments before
anything is launched."""
import ctypes
import os
import re

import pytest

from kernelized_feature_map_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(kata_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    build.build()
    return _abi.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert len(declared) >= 8
    for name in declared:
        assert hasattr(L, name), name
        assert name in _abi.SIGNATURES, "binding lacks " + name


def test_only_abi_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(_declared_functions())


def test_status_strings_and_version(L):
    assert _abi.kata_abi_version() == 10400
    for code, name in [(0, "KATA_OK"), (2, "KATA_ERR_UNSUPPORTED"), (6, "KATA_ERR_TIMEOUT")]:
        assert _abi.status_string(code) == name
    assert _abi.status_string(99) == "KATA_ERR_UNKNOWN"


def test_workspace_size_query(L):
    ws = _abi.kata_fwd_chunked_workspace_size
    # zero for T == 0 and for unsupported shapes
    assert ws(1, 1, 0, 16, 64, 64) == 0
    assert ws(1, 1, 100, 8, 64, 64) == 0
    assert ws(1, 1, 100, 16, 64, 96) == 0
    # CUDA-core layout: one fp32 record of P x (dv + 4) per (b,h) per super-chunk
    n = ws(1, 1, 256, 16, 16, 64, dtype=None)
    assert n > 0 and n % (256 * 20 * 4) == 0
    # tensor-core layout (bf16, p = 16, dv = 64): 65 rows x 144 packed
    # coordinates per (b,h) per super-chunk, and none at all when the whole
    # sequence is one super-chunk (the readout starts from S0 and writes the
    # final state itself)
    assert ws(8, 16, 2048, 16, 64, 64) == 0
    n = ws(1, 16, 131072, 16, 64, 64)
    assert n > 0 and n % (16 * 65 * 144 * 4) == 0
    # grows with T (more super-chunks) and never shrinks
    sizes = [ws(1, 16, t, 16, 64, 64) for t in (1024, 4096, 16384, 65536, 131072)]
    assert sizes == sorted(sizes)


def _round256(n):
    return (n + 255) // 256 * 256


def test_chunked_backward_workspace_size(L):
    """kata_bwd_chunked's workspace: 8 bytes per row (rounded up to 256) and,
    when the plan splits a sequence into G > 1 super-chunks, two 65 x 144 fp32
    records (forward and gradient state sums) per super-chunk of every (b,h).
    The plan keeps one super-chunk when the (b,h) walks alone fill the SMs
    (B8 H16 T2048: 256 walks of 16 chunks) and splits long sequences so that
    both walks of every super-chunk run in about two waves (B1 H16 T131072:
    9 super-chunks, 288 walks of 114 chunks)."""
    f = L.kata_bwd_chunked_workspace_size
    rec = 2 * 65 * 144 * 4
    assert f(8, 16, 2048, 16, 64, 1) == _round256(8 * 16 * 2048 * 8)
    assert f(1, 16, 131072, 16, 64, 1) == _round256(16 * 131072 * 8) + 16 * 9 * rec
    # B1 H1 T4096: 32 chunks, walks of 2 chunks in 16 super-chunks (one wave)
    assert f(1, 1, 4096, 16, 64, 1) == _round256(4096 * 8) + 16 * rec
    # a single chunk has no pair across chunks, but the row constants remain
    assert f(1, 2, 100, 16, 64, 1) == _round256(2 * 100 * 8)
    # other shapes and fp32 are not served
    assert f(1, 1, 1000, 32, 64, 1) == 0 and f(1, 1, 1000, 16, 16, 1) == 0 and f(1, 1, 1000, 16, 64, 0) == 0


VP = ctypes.c_void_p


def _fake(addr):
    return VP(addr)


def test_argument_errors_before_launch(L):
    a, b, c, d = _fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000)
    st = VP(0)
    f = L.kata_fwd_quadratic
    assert f(a, b, c, d, 1, 1, 16, 8, 64, 1, st) == _abi.KATA_ERR_UNSUPPORTED      # p
    assert f(a, b, c, d, 1, 1, 16, 16, 32, 1, st) == _abi.KATA_ERR_UNSUPPORTED     # dv
    assert f(a, b, c, d, 0, 1, 16, 16, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG     # B
    assert f(a, b, c, d, 1, 1, -1, 16, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG     # T
    assert f(a, b, c, d, 1, 1, 16, 16, 64, 7, st) == _abi.KATA_ERR_INVALID_ARG     # dtype
    assert f(None, b, c, d, 1, 1, 16, 16, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG  # null
    assert f(_fake(0x10008), b, c, d, 1, 1, 16, 16, 64, 1, st) == _abi.KATA_ERR_MISALIGNED
    assert f(a, b, c, d, 1, 1, 0, 16, 64, 1, st) == _abi.KATA_OK                   # T = 0: no-op
    g = L.kata_fwd_chunked
    ws = _fake(0x50000)
    assert g(a, b, c, d, 1, 1, 16, 16, 64, 96, 1, None, None, None, None, ws, 1 << 20, st) == _abi.KATA_ERR_UNSUPPORTED
    assert g(a, b, c, d, 1, 1, 16, 16, 64, 64, 1, _fake(0x60000), None, None, None, ws, 1 << 20, st) == _abi.KATA_ERR_INVALID_ARG
    assert g(a, b, c, d, 1, 1, 16, 16, 64, 64, 1, None, None, None, _fake(0x60000), ws, 1 << 20, st) == _abi.KATA_ERR_INVALID_ARG
    # a sequence of several super-chunks needs a workspace (one super-chunk needs none)
    assert g(a, b, c, d, 1, 16, 131072, 16, 64, 64, 1, None, None, None, None, ws, 16, st) == _abi.KATA_ERR_WORKSPACE
    assert g(a, b, c, d, 1, 16, 131072, 16, 64, 64, 1, None, None, None, None, None, 1 << 20,
             st) == _abi.KATA_ERR_WORKSPACE
    assert g(a, b, c, d, 1, 16, 131072, 16, 64, 64, 1, None, None, None, None, _fake(0x50010), 1 << 30,
             st) == _abi.KATA_ERR_MISALIGNED
    assert g(a, b, c, d, 1, 1, 0, 16, 64, 64, 1, None, None, None, None, None, 0, st) == _abi.KATA_OK
    sq = L.kata_fwd_chunked_sequential
    assert sq(a, b, c, d, 1, 1, 16, 16, 64, 64, 0, None, None, None, None, st) == _abi.KATA_ERR_UNSUPPORTED  # fp32
    assert sq(a, b, c, d, 1, 1, 16, 32, 64, 64, 1, None, None, None, None, st) == _abi.KATA_ERR_UNSUPPORTED  # p=32
    assert sq(a, b, c, d, 1, 1, 16, 16, 64, 96, 1, None, None, None, None, st) == _abi.KATA_ERR_UNSUPPORTED  # C
    assert sq(a, b, c, d, 1, 1, 16, 16, 64, 64, 1, _fake(0x60000), None, None, None, st) == _abi.KATA_ERR_INVALID_ARG
    h = L.kata_decode_step
    assert h(a, b, c, d, _fake(0x70000), None, 1, 1, 16, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG
    assert h(a, b, c, d, _fake(0x70000), _fake(0x80000), 1, 1, 24, 64, 1, st) == _abi.KATA_ERR_UNSUPPORTED
    assert h(a, b, c, d, _fake(0x70004), _fake(0x80000), 1, 1, 16, 64, 1, st) == _abi.KATA_ERR_MISALIGNED


def test_binding_requires_cuda_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 16)
    with pytest.raises(TypeError):
        _abi.kata_fwd_quadratic(q, q, torch.zeros(1, 1, 4, 64))


def test_mg_argument_errors_before_launch(L):
    a, b, c, d = _fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000)
    S, z = _fake(0x70000), _fake(0x80000)
    st = VP(0)
    m = L.kata_fwd_mg_quadratic  # q k v o B H T d groups dv layout dtype stream
    BHTD, BTHD = _abi.KATA_LAYOUT_BHTD, _abi.KATA_LAYOUT_BTHD
    assert m(a, b, c, d, 1, 1, 16, 64, 3, 64, BHTD, 1, st) == _abi.KATA_ERR_INVALID_ARG   # d % groups
    assert m(a, b, c, d, 1, 1, 16, 64, 0, 64, BHTD, 1, st) == _abi.KATA_ERR_INVALID_ARG   # groups
    assert m(a, b, c, d, 1, 1, 16, 64, 8, 64, BHTD, 1, st) == _abi.KATA_ERR_UNSUPPORTED   # p = 8
    assert m(a, b, c, d, 1, 1, 16, 64, 4, 16, BHTD, 1, st) == _abi.KATA_ERR_UNSUPPORTED   # dv 16 with groups
    assert m(a, b, c, d, 1, 1, 16, 128, 4, 64, BHTD, 1, st) == _abi.KATA_ERR_UNSUPPORTED  # p 32 x 4 groups
    assert m(a, b, c, d, 1, 1, 16, 64, 4, 64, 2, 1, st) == _abi.KATA_ERR_INVALID_ARG      # layout
    assert m(a, b, c, d, 1, 1, 16, 64, 4, 64, BHTD, 0, st) == _abi.KATA_ERR_UNSUPPORTED   # fp32
    assert m(None, b, c, d, 1, 1, 16, 64, 4, 64, BTHD, 1, st) == _abi.KATA_ERR_INVALID_ARG
    assert m(_fake(0x10008), b, c, d, 1, 1, 16, 64, 4, 64, BTHD, 1, st) == _abi.KATA_ERR_MISALIGNED
    assert m(a, b, c, d, 1, 1, 0, 64, 4, 64, BTHD, 1, st) == _abi.KATA_OK                 # T = 0: no-op
    md = L.kata_decode_step_mg  # q k v o S z B H d groups dv dtype stream
    assert md(a, b, c, d, S, None, 1, 1, 64, 4, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG
    assert md(a, b, c, d, S, z, 1, 1, 64, 4, 16, 1, st) == _abi.KATA_ERR_UNSUPPORTED
    assert md(a, b, c, d, S, z, 1, 1, 48, 4, 64, 1, st) == _abi.KATA_ERR_UNSUPPORTED      # p = 12
    assert md(a, b, c, d, S, z, 1, 1, 64, 5, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG
    assert md(a, b, c, d, _fake(0x70004), z, 1, 1, 64, 2, 64, 1, st) == _abi.KATA_ERR_MISALIGNED


def test_training_entry_points_reject_bad_arguments(L):
    a, b, c, d = _fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000)
    D, dO, gq, gk, gv, ws = (_fake(0x50000 + 0x10000 * i) for i in range(6))
    st = VP(0)
    f = L.kata_fwd_quadratic_train  # q k v o D B H T p dv dtype stream
    assert f(a, b, c, d, D, 1, 1, 16, 16, 64, 0, st) == _abi.KATA_ERR_UNSUPPORTED   # fp32
    assert f(a, b, c, d, D, 1, 1, 16, 16, 16, 1, st) == _abi.KATA_ERR_UNSUPPORTED   # dv 16
    assert f(a, b, c, d, None, 1, 1, 16, 16, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG
    assert f(a, b, c, d, _fake(0x50004), 1, 1, 16, 16, 64, 1, st) == _abi.KATA_ERR_MISALIGNED
    assert f(a, b, c, d, D, 1, 1, 0, 16, 64, 1, st) == _abi.KATA_OK
    ws_size = _abi.lib().kata_bwd_quadratic_workspace_size
    assert ws_size(2, 3, 100, 16, 64, 1) == 2 * 3 * 100 * 8
    assert ws_size(2, 3, 100, 16, 64, 0) == 0 and ws_size(1, 1, 0, 16, 64, 1) == 0
    g = L.kata_bwd_quadratic  # q k v o D dO dq dk dv B H T p dv dtype ws bytes stream
    n = 1 * 1 * 16 * 8
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 16, 24, 64, 1, ws, n, st) == _abi.KATA_ERR_UNSUPPORTED
    assert g(a, b, c, d, D, None, gq, gk, gv, 1, 1, 16, 16, 64, 1, ws, n, st) == _abi.KATA_ERR_INVALID_ARG
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 16, 16, 64, 1, ws, n - 1, st) == _abi.KATA_ERR_WORKSPACE
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 16, 16, 64, 1, None, n, st) == _abi.KATA_ERR_WORKSPACE
    assert g(a, b, c, d, D, dO, gq, gk, _fake(0x90008), 1, 1, 16, 16, 64, 1, ws, n, st) == _abi.KATA_ERR_MISALIGNED
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 0, 16, 64, 1, None, 0, st) == _abi.KATA_OK


def test_mg_training_entry_points_reject_bad_arguments(L):
    a, b, c, d = _fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000)
    D, dO, gq, gk, gv, ws = (_fake(0x50000 + 0x10000 * i) for i in range(6))
    st = VP(0)
    f = L.kata_fwd_mg_quadratic_train  # q k v o D B H T d groups dv dtype stream
    assert f(a, b, c, d, D, 1, 1, 16, 64, 1, 64, 1, st) == _abi.KATA_ERR_UNSUPPORTED   # one group: single-factor call
    assert f(a, b, c, d, D, 1, 1, 16, 64, 2, 64, 0, st) == _abi.KATA_ERR_UNSUPPORTED   # fp32
    assert f(a, b, c, d, None, 1, 1, 16, 64, 2, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG
    assert f(a, b, c, d, D, 1, 1, 16, 64, 3, 64, 1, st) == _abi.KATA_ERR_INVALID_ARG   # 64 % 3
    assert f(a, b, c, d, D, 1, 1, 0, 64, 2, 64, 1, st) == _abi.KATA_OK
    g = L.kata_bwd_mg_quadratic  # q k v o D dO dq dk dv B H T d groups dv dtype ws bytes stream
    n = 16 * 8
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 16, 64, 2, 16, 1, ws, n, st) == _abi.KATA_ERR_UNSUPPORTED
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 16, 64, 2, 64, 1, ws, n - 1, st) == _abi.KATA_ERR_WORKSPACE
    assert g(a, b, c, d, D, None, gq, gk, gv, 1, 1, 16, 64, 2, 64, 1, ws, n, st) == _abi.KATA_ERR_INVALID_ARG
    assert g(a, b, c, d, D, dO, gq, gk, gv, 1, 1, 0, 64, 4, 64, 1, None, 0, st) == _abi.KATA_OK


def test_sg_argument_errors_before_launch(L):
    a, b, c, d = _fake(0x10000), _fake(0x20000), _fake(0x30000), _fake(0x40000)
    st = VP(0)
    f = L.kata_fwd_sg_quadratic  # q k v o B H T d groups dv layout dtype stream
    assert f(a, b, c, d, 1, 1, 16, 64, 1, 64, 0, 1, st) == _abi.KATA_ERR_UNSUPPORTED   # one group
    assert f(a, b, c, d, 1, 1, 16, 64, 3, 64, 0, 1, st) == _abi.KATA_ERR_INVALID_ARG   # 64 % 3
    assert f(a, b, c, d, 1, 1, 16, 64, 2, 64, 5, 1, st) == _abi.KATA_ERR_INVALID_ARG   # layout
    assert f(a, b, c, d, 1, 1, 16, 64, 2, 64, 0, 0, st) == _abi.KATA_ERR_UNSUPPORTED   # fp32
    assert f(a, b, c, d, 1, 1, 0, 64, 2, 64, 1, 1, st) == _abi.KATA_OK


def test_noalloc_scratch_size_matches_header():
    """The binding's copy of the no-allocation scratch size is the header's
    KATA_NOALLOC_SCRATCH_BYTES (the library asserts the same at build time)."""
    text = open(os.path.join(ROOT, "include", "kata.h")).read()
    m = re.search(r"#define KATA_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m
    assert _abi.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))

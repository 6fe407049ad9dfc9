"""Thin ctypes binding of libkata's C ABI (include/kata.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  Functions carry the C names and take torch tensors
(device memory and the current CUDA stream are PyTorch's; nothing else is).
If the library is missing, every call raises: there is no other path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkata.so")

KATA_OK, KATA_ERR_INVALID_ARG, KATA_ERR_UNSUPPORTED, KATA_ERR_MISALIGNED = 0, 1, 2, 3
KATA_ERR_WORKSPACE, KATA_ERR_CUDA, KATA_ERR_TIMEOUT = 4, 5, 6
KATA_F32, KATA_BF16 = 0, 1
KATA_LAYOUT_BHTD, KATA_LAYOUT_BTHD = 0, 1

# name -> (restype, argtypes), mirroring include/kata.h
_c_int, _c_size, _vp, _fp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
SIGNATURES = {
    "kata_fwd_quadratic": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "kata_fwd_chunked_workspace_size": (_c_size, [_c_int] * 7),
    "kata_fwd_chunked": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                  _fp, _fp, _fp, _fp, _vp, _c_size, _vp]),
    "kata_fwd_chunked_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                          _c_int, _fp, _fp, _fp, _fp, _vp]),
    "kata_fwd_chunked_sequential": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                             _c_int, _fp, _fp, _fp, _fp, _vp]),
    "kata_fwd_linear_chunked_workspace_size": (_c_size, [_c_int] * 6),
    "kata_fwd_linear_chunked": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 7 + [_fp, _fp, _fp, _fp, _vp, _c_size, _vp]),
    "kata_fwd_linear_chunked_sequential": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 7 + [_fp, _fp, _fp, _fp, _vp]),
    "kata_decode_step": (_c_int, [_vp, _vp, _vp, _vp, _fp, _fp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "kata_fwd_quadratic_train": (_c_int, [_vp, _vp, _vp, _vp, _fp] + [_c_int] * 6 + [_vp]),
    "kata_bwd_quadratic_workspace_size": (_c_size, [_c_int] * 6),
    "kata_bwd_quadratic": (_c_int, [_vp] * 9 + [_c_int] * 6 + [_vp, _c_size, _vp]),
    "kata_fwd_mg_quadratic": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 8 + [_vp]),
    "kata_fwd_chunked_train": (_c_int, [_vp, _vp, _vp, _vp, _fp] + [_c_int] * 7 + [_vp, _c_size, _vp]),
    "kata_bwd_chunked_workspace_size": (_c_size, [_c_int] * 6),
    "kata_bwd_chunked": (_c_int, [_vp] * 9 + [_c_int] * 6 + [_vp, _c_size, _vp]),
    "kata_fwd_mg_quadratic_train": (_c_int, [_vp, _vp, _vp, _vp, _fp] + [_c_int] * 7 + [_vp]),
    "kata_fwd_sg_quadratic": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 8 + [_vp]),
    "kata_fwd_mg_chunked_workspace_size": (_c_size, [_c_int] * 8),
    "kata_fwd_mg_chunked": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 9 + [_fp, _fp, _fp, _fp, _vp, _c_size, _vp]),
    "kata_bwd_mg_quadratic": (_c_int, [_vp] * 9 + [_c_int] * 7 + [_vp, _c_size, _vp]),
    "kata_decode_step_mg": (_c_int, [_vp, _vp, _vp, _vp, _fp, _fp] + [_c_int] * 6 + [_vp]),
    "kata_decode_step_sg": (_c_int, [_vp, _vp, _vp, _vp, _fp, _fp] + [_c_int] * 6 + [_vp]),
    "kata_fwd_sg_chunked_workspace_size": (_c_size, [_c_int] * 7),
    "kata_fwd_sg_quadratic_train": (_c_int, [_vp, _vp, _vp, _vp, _fp] + [_c_int] * 7 + [_vp]),
    "kata_bwd_sg_quadratic": (_c_int, [_vp] * 9 + [_c_int] * 7 + [_vp, _c_size, _vp]),
    "kata_fwd_sg_chunked": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 8 + [_fp, _fp, _fp, _fp, _vp, _c_size, _vp]),
    "kata_get_status": (_c_int, [_vp]),
    "kata_status_string": (ctypes.c_char_p, [_c_int]),
    "kata_set_wait_limit": (None, [ctypes.c_longlong]),
    "kata_abi_version": (_c_int, []),
}

_lib = None


class KataError(RuntimeError):
    """A libkata call returned a status other than KATA_OK."""

    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, status_string(status), status))


def lib():
    """The loaded libkata (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libkata.so is not built (run: python -m kernelized_feature_map_b200.build); "
                               "there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kata_status_string(int(status)).decode()


def _check(fn, status):
    if status != KATA_OK:
        raise KataError(fn, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KATA_BF16
    if t.dtype == torch.float32:
        return KATA_F32
    raise TypeError("q, k, v must be torch.bfloat16 or torch.float32, got %s" % t.dtype)


def _stream_ptr(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


def _opt(t, name):
    return None if t is None else _dev(t, name)


def kata_fwd_quadratic(q, k, v, o=None, stream=None):
    """Flash-style O(T^2) forward.  q,k [B,H,T,p], v [B,H,T,dv] -> o [B,H,T,dv]."""
    B, H, T, p = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    _check("kata_fwd_quadratic", lib().kata_fwd_quadratic(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, p, dv, _dtype_code(q), _stream_ptr(stream)))
    return o


def kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, dtype=torch.bfloat16) -> int:
    code = KATA_BF16 if dtype == torch.bfloat16 else KATA_F32
    return int(lib().kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, code))


def kata_fwd_chunked(q, k, v, C=64, S0=None, z0=None, return_state=False, o=None, workspace=None,
                     S_out=None, z_out=None, stream=None):
    """Exact O(T) chunked-state forward.

    Returns o, or (o, S_T, z_T) when return_state is True.  S0/z0 give an
    initial state ([B,H,p*p,dv], [B,H,p*p] fp32).  ``workspace`` may be a
    preallocated uint8 CUDA tensor of at least the queried size.
    """
    B, H, T, p = q.shape
    dv = v.shape[-1]
    dev = q.device
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, p * p, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, p * p), dtype=torch.float32, device=dev)
    need = kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kata_fwd_chunked", lib().kata_fwd_chunked(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, p, dv, C, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"),
        _opt(workspace, "workspace"), ws_bytes, _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


NOALLOC_SCRATCH_BYTES = 16 << 20  # size of the library-owned scratch array


def kata_fwd_chunked_noalloc(q, k, v, C=64, S0=None, z0=None, return_state=False, o=None, S_out=None, z_out=None,
                             stream=None):
    """kata_fwd_chunked with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory: the state records live in
    a 16 MiB device array owned by the library (sizes that need more raise
    KataError with KATA_ERR_WORKSPACE).  Calls share that array, so calls that
    overlap on the GPU must be serialised by the caller.  The output and
    optional state tensors are still the caller's (allocated here only when
    not passed in).
    """
    B, H, T, p = q.shape
    dv = v.shape[-1]
    dev = q.device
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, p * p, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, p * p), dtype=torch.float32, device=dev)
    _check("kata_fwd_chunked_noalloc", lib().kata_fwd_chunked_noalloc(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, p, dv, C, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"), _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


def kata_fwd_chunked_sequential(q, k, v, C=64, S0=None, z0=None, return_state=False, o=None, S_out=None,
                                z_out=None, stream=None):
    """Sequential inter-chunk baseline: one CTA per (b,h) walks all of its
    chunks in order (no super-chunk sums, no scan).  bf16, p=16, dv=64 only."""
    B, H, T, p = q.shape
    dv = v.shape[-1]
    dev = q.device
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, p * p, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, p * p), dtype=torch.float32, device=dev)
    _check("kata_fwd_chunked_sequential", lib().kata_fwd_chunked_sequential(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, p, dv, C, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"), _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


def kata_fwd_linear_chunked_workspace_size(B, H, T, d, dv, C) -> int:
    return int(lib().kata_fwd_linear_chunked_workspace_size(B, H, T, d, dv, C))


def kata_fwd_linear_chunked(q, k, v, C=64, S0=None, z0=None, return_state=False, o=None, workspace=None,
                            S_out=None, z_out=None, stream=None):
    """First-order (psi(u) = u) chunked forward with the associative scan.

    q,k [B,H,T,d], v [B,H,T,dv] (bf16, d=16, dv=64).  Returns o, or
    (o, S_T, z_T) when return_state is True; S0/z0 ([B,H,d,dv], [B,H,d] fp32)
    give an initial state.
    """
    B, H, T, d = q.shape
    dv = v.shape[-1]
    dev = q.device
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, d, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    need = kata_fwd_linear_chunked_workspace_size(B, H, T, d, dv, C)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kata_fwd_linear_chunked", lib().kata_fwd_linear_chunked(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d, dv, C, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"),
        _opt(workspace, "workspace"), ws_bytes, _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


def kata_fwd_linear_chunked_sequential(q, k, v, C=64, S0=None, z0=None, return_state=False, o=None, S_out=None,
                                       z_out=None, stream=None):
    """The matched sequential baseline of kata_fwd_linear_chunked: one CTA per
    (b,h) walks all of its chunks in order (no super-chunk sums, no scan)."""
    B, H, T, d = q.shape
    dv = v.shape[-1]
    dev = q.device
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, d, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    _check("kata_fwd_linear_chunked_sequential", lib().kata_fwd_linear_chunked_sequential(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d, dv, C, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"), _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


def kata_decode_step(q, k, v, S, z, o=None, stream=None):
    """One decode step; S [B,H,p*p,dv] and z [B,H,p*p] (fp32) are updated in place."""
    B, H, p = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check("kata_decode_step", lib().kata_decode_step(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(S, "S"), _dev(z, "z"), B, H, p, dv,
        _dtype_code(q), _stream_ptr(stream)))
    return o


def kata_fwd_quadratic_train(q, k, v, o=None, D=None, stream=None):
    """Flash-style forward that also returns each row's denominator.

    q,k [B,H,T,p], v [B,H,T,dv] (bf16) -> (o [B,H,T,dv], D [B,H,T] fp32).
    """
    B, H, T, p = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if D is None:
        D = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check("kata_fwd_quadratic_train", lib().kata_fwd_quadratic_train(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), B, H, T, p, dv, _dtype_code(q),
        _stream_ptr(stream)))
    return o, D


def kata_bwd_quadratic(q, k, v, o, D, dO, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of the flash-style forward for the upstream
    gradient dO, from the forward's o and D (kata_fwd_quadratic_train)."""
    B, H, T, p = q.shape
    dvw = v.shape[-1]
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    need = int(lib().kata_bwd_quadratic_workspace_size(B, H, T, p, dvw, _dtype_code(q)))
    if workspace is None:
        workspace = torch.empty(max(256, need), dtype=torch.uint8, device=q.device)
    _check("kata_bwd_quadratic", lib().kata_bwd_quadratic(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), _dev(dO, "dO"), _dev(dq, "dq"),
        _dev(dk, "dk"), _dev(dv, "dv"), B, H, T, p, dvw, _dtype_code(q), _dev(workspace, "workspace"),
        workspace.numel(), _stream_ptr(stream)))
    return dq, dk, dv


class KataAttention(torch.autograd.Function):
    """Autograd wrapper: forward by kata_fwd_quadratic_train, backward by
    kata_bwd_quadratic (argument marshalling only)."""

    @staticmethod
    def forward(ctx, q, k, v):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, D = kata_fwd_quadratic_train(q, k, v)
        ctx.save_for_backward(q, k, v, o, D)
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, D = ctx.saved_tensors
        return kata_bwd_quadratic(q, k, v, o, D, dO.contiguous())


def kata_attention(q, k, v):
    """Differentiable flash-style KATA attention, q,k [B,H,T,p], v [B,H,T,dv]."""
    return KataAttention.apply(q, k, v)


def kata_fwd_sg_quadratic(q, k, v, groups, layout="bhtd", o=None, stream=None):
    """Flash-style KATA-Sigma-g forward: weight sum_{j,l} (q^j . k^l)^2 over
    every pair of a query group and a key group.  Layouts as for
    kata_fwd_mg_quadratic; groups > 1."""
    if layout == "bhtd":
        B, H, T, d = q.shape
        code = KATA_LAYOUT_BHTD
    elif layout == "bthd":
        B, T, H, d = q.shape
        code = KATA_LAYOUT_BTHD
    else:
        raise ValueError("layout must be 'bhtd' or 'bthd'")
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    _check("kata_fwd_sg_quadratic", lib().kata_fwd_sg_quadratic(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d, int(groups), dv, code,
        _dtype_code(q), _stream_ptr(stream)))
    return o


def kata_fwd_chunked_train(q, k, v, C=64, o=None, D=None, workspace=None, stream=None):
    """The chunked forward (bf16, p=16, dv=64) that also returns each row's denominator."""
    B, H, T, p = q.shape
    dv = v.shape[-1]
    dev = q.device
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if D is None:
        D = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    need = kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kata_fwd_chunked_train", lib().kata_fwd_chunked_train(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), B, H, T, p, dv, C, _dtype_code(q),
        _opt(workspace, "workspace"), ws_bytes, _stream_ptr(stream)))
    return o, D


def kata_bwd_chunked(q, k, v, o, D, dO, workspace=None, stream=None):
    """Gradients (dq, dk, dv) by the O(T) chunked backward, from o and D."""
    B, H, T, p = q.shape
    dvw = v.shape[-1]
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    need = int(lib().kata_bwd_chunked_workspace_size(B, H, T, p, dvw, _dtype_code(q)))
    if workspace is None:
        workspace = torch.empty(max(256, need), dtype=torch.uint8, device=q.device)
    _check("kata_bwd_chunked", lib().kata_bwd_chunked(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), _dev(dO, "dO"), _dev(dq, "dq"),
        _dev(dk, "dk"), _dev(dv, "dv"), B, H, T, p, dvw, _dtype_code(q), _dev(workspace, "workspace"),
        workspace.numel(), _stream_ptr(stream)))
    return dq, dk, dv


class KataAttentionChunked(torch.autograd.Function):
    """Autograd wrapper of the chunked forward and backward (marshalling only)."""

    @staticmethod
    def forward(ctx, q, k, v):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, D = kata_fwd_chunked_train(q, k, v)
        ctx.save_for_backward(q, k, v, o, D)
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, D = ctx.saved_tensors
        return kata_bwd_chunked(q, k, v, o, D, dO.contiguous())


def kata_attention_chunked(q, k, v):
    """Differentiable KATA attention on the O(T) chunked path, q,k [B,H,T,16], v [B,H,T,64] (bf16)."""
    return KataAttentionChunked.apply(q, k, v)


def kata_fwd_mg_quadratic_train(q, k, v, groups, o=None, D=None, stream=None):
    """KATA-Mg forward ([B,H,T,d], groups > 1) that also returns each row's denominator."""
    B, H, T, d = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if D is None:
        D = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check("kata_fwd_mg_quadratic_train", lib().kata_fwd_mg_quadratic_train(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), B, H, T, d, int(groups), dv,
        _dtype_code(q), _stream_ptr(stream)))
    return o, D


def kata_bwd_mg_quadratic(q, k, v, o, D, dO, groups, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of the KATA-Mg forward from its o and D."""
    B, H, T, d = q.shape
    dvw = v.shape[-1]
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    need = int(lib().kata_bwd_quadratic_workspace_size(B, H, T, d // int(groups), dvw, _dtype_code(q)))
    if workspace is None:
        workspace = torch.empty(max(256, need), dtype=torch.uint8, device=q.device)
    _check("kata_bwd_mg_quadratic", lib().kata_bwd_mg_quadratic(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), _dev(dO, "dO"), _dev(dq, "dq"),
        _dev(dk, "dk"), _dev(dv, "dv"), B, H, T, d, int(groups), dvw, _dtype_code(q), _dev(workspace, "workspace"),
        workspace.numel(), _stream_ptr(stream)))
    return dq, dk, dv


class KataAttentionMg(torch.autograd.Function):
    """Autograd wrapper of the KATA-Mg forward and backward (marshalling only)."""

    @staticmethod
    def forward(ctx, q, k, v, groups):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, D = kata_fwd_mg_quadratic_train(q, k, v, groups)
        ctx.groups = int(groups)
        ctx.save_for_backward(q, k, v, o, D)
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, D = ctx.saved_tensors
        dq, dk, dv = kata_bwd_mg_quadratic(q, k, v, o, D, dO.contiguous(), ctx.groups)
        return dq, dk, dv, None


def kata_attention_mg(q, k, v, groups):
    """Differentiable KATA-Mg attention, q,k [B,H,T,d], v [B,H,T,dv], groups > 1."""
    return KataAttentionMg.apply(q, k, v, groups)


def kata_fwd_sg_quadratic_train(q, k, v, groups, o=None, D=None, stream=None):
    """KATA-Sigma-g forward ([B,H,T,d], groups > 1) that also returns each row's denominator."""
    B, H, T, d = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if D is None:
        D = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check("kata_fwd_sg_quadratic_train", lib().kata_fwd_sg_quadratic_train(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), B, H, T, d, int(groups), dv,
        _dtype_code(q), _stream_ptr(stream)))
    return o, D


def kata_bwd_sg_quadratic(q, k, v, o, D, dO, groups, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of the KATA-Sigma-g forward from its o and D."""
    B, H, T, d = q.shape
    dvw = v.shape[-1]
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    need = int(lib().kata_bwd_quadratic_workspace_size(B, H, T, d // int(groups), dvw, _dtype_code(q)))
    if workspace is None:
        workspace = torch.empty(max(256, need), dtype=torch.uint8, device=q.device)
    _check("kata_bwd_sg_quadratic", lib().kata_bwd_sg_quadratic(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(D, "D"), _dev(dO, "dO"), _dev(dq, "dq"),
        _dev(dk, "dk"), _dev(dv, "dv"), B, H, T, d, int(groups), dvw, _dtype_code(q), _dev(workspace, "workspace"),
        workspace.numel(), _stream_ptr(stream)))
    return dq, dk, dv


class KataAttentionSg(torch.autograd.Function):
    """Autograd wrapper of the KATA-Sigma-g forward and backward (marshalling only)."""

    @staticmethod
    def forward(ctx, q, k, v, groups):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, D = kata_fwd_sg_quadratic_train(q, k, v, groups)
        ctx.groups = int(groups)
        ctx.save_for_backward(q, k, v, o, D)
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, o, D = ctx.saved_tensors
        dq, dk, dv = kata_bwd_sg_quadratic(q, k, v, o, D, dO.contiguous(), ctx.groups)
        return dq, dk, dv, None


def kata_attention_sg(q, k, v, groups):
    """Differentiable KATA-Sigma-g attention, q,k [B,H,T,d], v [B,H,T,dv], groups > 1."""
    return KataAttentionSg.apply(q, k, v, groups)


def kata_fwd_mg_quadratic(q, k, v, groups, layout="bhtd", o=None, stream=None):
    """Flash-style KATA-Mg forward with `groups` PSD factors per head.

    layout "bhtd": q,k [B,H,T,d], v,o [B,H,T,dv]; layout "bthd": q,k
    [B,T,H,d], v,o [B,T,H,dv].  The score of a pair is the sum over the
    groups (consecutive blocks of d/groups coordinates) of the squared group
    dot products.
    """
    if layout == "bhtd":
        B, H, T, d = q.shape
        code = KATA_LAYOUT_BHTD
    elif layout == "bthd":
        B, T, H, d = q.shape
        code = KATA_LAYOUT_BTHD
    else:
        raise ValueError("layout must be 'bhtd' or 'bthd'")
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    _check("kata_fwd_mg_quadratic", lib().kata_fwd_mg_quadratic(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d, int(groups), dv, code,
        _dtype_code(q), _stream_ptr(stream)))
    return o


def kata_fwd_mg_chunked_workspace_size(B, H, T, d, groups, dv, C, dtype=torch.bfloat16) -> int:
    code = KATA_BF16 if dtype == torch.bfloat16 else KATA_F32
    return int(lib().kata_fwd_mg_chunked_workspace_size(B, H, T, d, int(groups), dv, C, code))


def kata_fwd_mg_chunked(q, k, v, groups, C=64, layout="bhtd", S0=None, z0=None, return_state=False, o=None,
                        workspace=None, S_out=None, z_out=None, stream=None):
    """Exact O(T) chunked-state KATA-Mg forward with `groups` PSD factors per head.

    Layouts as kata_fwd_mg_quadratic.  Returns o, or (o, S_T, z_T) when
    return_state is True; the state is [B,H,groups*p*p,dv] and
    [B,H,groups*p*p] fp32 (p = d / groups), S0/z0 an initial state of the
    same shapes.  ``workspace`` may be a preallocated uint8 CUDA tensor of at
    least the queried size.
    """
    if layout == "bhtd":
        B, H, T, d = q.shape
        code = KATA_LAYOUT_BHTD
    elif layout == "bthd":
        B, T, H, d = q.shape
        code = KATA_LAYOUT_BTHD
    else:
        raise ValueError("layout must be 'bhtd' or 'bthd'")
    dv = v.shape[-1]
    g = int(groups)
    p = d // g
    dev = q.device
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, g * p * p, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, g * p * p), dtype=torch.float32, device=dev)
    need = kata_fwd_mg_chunked_workspace_size(B, H, T, d, g, dv, C, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kata_fwd_mg_chunked", lib().kata_fwd_mg_chunked(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d, g, dv, C, code, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"),
        _opt(workspace, "workspace"), ws_bytes, _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


def parallel_kata_attn(q, k, v, num_groups=2, stream=None):
    """The pages' attention call shape: q,k,v [B,T,H,D] -> o [B,T,H,D], with
    num_groups PSD factors per head (KATA-Mg, forward only)."""
    return kata_fwd_mg_quadratic(q, k, v, num_groups, layout="bthd", stream=stream)


def kata_decode_step_mg(q, k, v, S, z, groups, o=None, stream=None):
    """One KATA-Mg decode step: q,k [B,H,d], v [B,H,dv]; S [B,H,groups*p*p,dv]
    and z [B,H,groups*p*p] (fp32, p = d/groups) are updated in place."""
    B, H, d = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check("kata_decode_step_mg", lib().kata_decode_step_mg(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(S, "S"), _dev(z, "z"), B, H, d, int(groups),
        dv, _dtype_code(q), _stream_ptr(stream)))
    return o


def kata_fwd_sg_chunked_workspace_size(B, H, T, d, groups, dv, C) -> int:
    return int(lib().kata_fwd_sg_chunked_workspace_size(B, H, T, d, int(groups), dv, C))


def kata_fwd_sg_chunked(q, k, v, groups, C=64, S0=None, z0=None, return_state=False, o=None, workspace=None,
                        S_out=None, z_out=None, stream=None):
    """KATA-Sigma-g on the exact O(T) chunked path: q,k [B,H,T,d], v [B,H,T,dv]
    (bf16, d = 16 * groups, groups 2 or 4, dv = 64).  The state ([B,H,p*p,dv],
    [B,H,p*p] fp32, p = d/groups) is that of the summed feature."""
    B, H, T, d = q.shape
    dv = v.shape[-1]
    dev = q.device
    p = d // int(groups)
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if return_state and S_out is None:
        S_out = torch.empty((B, H, p * p, dv), dtype=torch.float32, device=dev)
        z_out = torch.empty((B, H, p * p), dtype=torch.float32, device=dev)
    need = kata_fwd_sg_chunked_workspace_size(B, H, T, d, groups, dv, C)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kata_fwd_sg_chunked", lib().kata_fwd_sg_chunked(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), B, H, T, d, int(groups), dv, C, _dtype_code(q),
        _opt(S0, "S0"), _opt(z0, "z0"), _opt(S_out, "S_out"), _opt(z_out, "z_out"),
        _opt(workspace, "workspace"), ws_bytes, _stream_ptr(stream)))
    if return_state:
        return o, S_out, z_out
    return o


def kata_decode_step_sg(q, k, v, S, z, groups, o=None, stream=None):
    """One KATA-Sigma-g decode step: q,k [B,H,d], v [B,H,dv]; S [B,H,p*p,dv]
    and z [B,H,p*p] (fp32, p = d/groups, the summed feature's state) are
    updated in place."""
    B, H, d = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check("kata_decode_step_sg", lib().kata_decode_step_sg(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(S, "S"), _dev(z, "z"), B, H, d, int(groups),
        dv, _dtype_code(q), _stream_ptr(stream)))
    return o


def kata_get_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib().kata_get_status(_stream_ptr(stream)))


def kata_set_wait_limit(cycles: int) -> None:
    lib().kata_set_wait_limit(int(cycles))


def kata_abi_version() -> int:
    return int(lib().kata_abi_version())

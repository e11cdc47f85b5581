"""Thin ctypes binding of libgdn_b200.so (include/gdn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the library.  torch is used for device memory (outputs and the
workspace when the caller passes none) and for the current stream.  If the
library is missing, importing works but every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn_b200.so")
# GDN_DEBUG_BOUNDS=1 in the environment selects the bounds-checking build of the same library
# (built by `python -m gated_delta_rule_fg_b200.build --debug-bounds`).
BOUNDS_LIB_PATH = os.path.join(_HERE, "libgdn_b200_bounds.so")
if os.environ.get("GDN_DEBUG_BOUNDS", "") not in ("", "0"):
    LIB_PATH = BOUNDS_LIB_PATH

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA = 0, 1, 2, 3
GDN_ERR_TIMEOUT, GDN_ERR_WORKSPACE, GDN_ERR_RANGE, GDN_ERR_BOUNDS = 4, 5, 6, 7
GDN_F32, GDN_BF16 = 0, 1
GDN_ALPHA_SCALAR, GDN_BETA_SCALAR, GDN_SINGLE_STREAM = 1, 2, 4

# Every symbol include/gdn.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
SIGNATURES = {
    "gdn_chunk_fwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_chunk_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                           ctypes.c_uint, _P, _SZ, _P]),
    "gdn_chunk_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                   ctypes.c_uint, _P]),
    "gdn_plus_chunk_fwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_plus_chunk_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                ctypes.c_uint, _P, _SZ, _P]),
    "gdn_plus_chunk_fwd_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_deltaproduct_fwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gdn_deltaproduct_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                  _I, _P, _SZ, _P]),
    "gdn_chunk_fwd_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_chunk_fwd_tensor_cores": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_deltaproduct_fwd_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gdn_recurrent_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                ctypes.c_uint, _P]),
    "gdn_chunk_bwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_chunk_bwd": (_I, [_P] * 16 + [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint, _P, _SZ, _P]),
    "gdn_chunk_bwd_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn2_chunk_fwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn2_chunk_fwd": (_I, [_P] * 9 + [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint, _I, _P, _SZ, _P]),
    "gdn2_chunk_fwd_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint]),
    "gdn_workspace_status": (_I, [_P, _P]),
    "gdn_status_string": (ctypes.c_char_p, [_I]),
    "gdn_version": (_I, []),
}

_lib = None


class GdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} (status {code})")
        self.code = code


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdn_b200.so is not built ({LIB_PATH}); run "
                               "`python -m gated_delta_rule_fg_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().gdn_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _check(t, name, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def chunk_fwd_tensor_cores(B, H, T, dk, dv, chunk, dtype_code, flags=0) -> int:
    """1: gdn_chunk_fwd takes the tensor-core path for these sizes; 0: the float32 CUDA-core
    path; -1: invalid or unsupported sizes."""
    return int(lib().gdn_chunk_fwd_tensor_cores(B, H, T, dk, dv, chunk, dtype_code, flags))


def chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags))


def plus_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn_plus_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags))


def plus_chunk_fwd_launches(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn_plus_chunk_fwd_launches(B, H, T, dk, dv, chunk, dtype_code, flags))


def deltaproduct_fwd_workspace_size(B, H, T, nh, dk, dv, chunk, dtype_code) -> int:
    return int(lib().gdn_deltaproduct_fwd_workspace_size(B, H, T, nh, dk, dv, chunk, dtype_code))


def chunk_fwd_launches(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn_chunk_fwd_launches(B, H, T, dk, dv, chunk, dtype_code, flags))


def deltaproduct_fwd_launches(B, H, T, nh, dk, dv, chunk, dtype_code) -> int:
    return int(lib().gdn_deltaproduct_fwd_launches(B, H, T, nh, dk, dv, chunk, dtype_code))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def chunk_fwd(q, k, v, alpha, beta, S0=None, *, chunk=64, alpha_scalar=False, beta_scalar=False,
              out=None, S_final=None, want_state=True, workspace=None, stream=None, single_stream=False):
    """FG^2-GDN chunkwise forward through gdn_chunk_fwd.

    q, k [B,T,H,dk], v [B,T,H,dv] (bf16 or float32, same dtype); alpha/beta float32
    [B,T,H,dk] or [B,T,H] with alpha_scalar/beta_scalar; S0 float32 [B,H,dk,dv] or None.
    Returns (out [B,T,H,dv] in q's dtype, S_final float32 [B,H,dk,dv] or None).
    """
    code = _dtype_code(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta"), (S0, "S0")):
        _check(t, n, torch.float32)
    flags = ((GDN_ALPHA_SCALAR if alpha_scalar else 0) | (GDN_BETA_SCALAR if beta_scalar else 0)
             | (GDN_SINGLE_STREAM if single_stream else 0))
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(S_final, "S_final", torch.float32)
    need = chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, code, flags)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                             _ptr(out), _ptr(S_final), B, H, T, dk, dv, chunk, code, flags,
                             _ptr(workspace), workspace.numel(), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd")
    return out, S_final


def plus_chunk_fwd(q, k, v, alpha, beta_k, beta_v, S0=None, *, chunk=64, alpha_scalar=False,
                   beta_scalar=False, out=None, S_final=None, want_state=True, workspace=None,
                   stream=None):
    """FG^2-GDN+ chunkwise forward through gdn_plus_chunk_fwd: beta_k scales the keys
    and beta_v ([B,T,H,dv], or [B,T,H] with beta_scalar) the values.  Otherwise as
    chunk_fwd."""
    code = _dtype_code(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype)
    for t, n in ((alpha, "alpha"), (beta_k, "beta_k"), (beta_v, "beta_v"), (S0, "S0")):
        _check(t, n, torch.float32)
    flags = (GDN_ALPHA_SCALAR if alpha_scalar else 0) | (GDN_BETA_SCALAR if beta_scalar else 0)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(S_final, "S_final", torch.float32)
    need = plus_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, code, flags)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().gdn_plus_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k), _ptr(beta_v),
                                  _ptr(S0), _ptr(out), _ptr(S_final), B, H, T, dk, dv, chunk, code,
                                  flags, _ptr(workspace), workspace.numel(), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_plus_chunk_fwd")
    return out, S_final


def chunk_fwd_noalloc(q, k, v, alpha, beta, S0=None, *, chunk=64, alpha_scalar=False,
                      beta_scalar=False, out=None, S_final=None, want_state=True, stream=None):
    """gdn_chunk_fwd_noalloc: as chunk_fwd, with the library's built-in 64 MiB scratch
    instead of a caller workspace (for callers that cannot allocate device memory)."""
    code = _dtype_code(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta"), (S0, "S0")):
        _check(t, n, torch.float32)
    flags = (GDN_ALPHA_SCALAR if alpha_scalar else 0) | (GDN_BETA_SCALAR if beta_scalar else 0)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(S_final, "S_final", torch.float32)
    st = lib().gdn_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                                     _ptr(out), _ptr(S_final), B, H, T, dk, dv, chunk, code, flags,
                                     _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_fwd_noalloc")
    return out, S_final


def deltaproduct_fwd(q, k, v, gamma, beta, S0=None, *, chunk=64, out=None, S_final=None,
                     want_state=True, workspace=None, stream=None):
    """DeltaProduct n_h forward through gdn_deltaproduct_fwd.

    q [B,T,H,dk]; k [B,T,H,n_h,dk]; v [B,T,H,n_h,dv]; gamma [B,T,H]; beta [B,T,H,n_h]
    (float32); S0 float32 [B,H,dk,dv] or None.  Returns (out, S_final).
    """
    code = _dtype_code(q)
    B, T, H, nh, dk = k.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype)
    for t, n in ((gamma, "gamma"), (beta, "beta"), (S0, "S0")):
        _check(t, n, torch.float32)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = deltaproduct_fwd_workspace_size(B, H, T, nh, dk, dv, chunk, code)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().gdn_deltaproduct_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(S0),
                                    _ptr(out), _ptr(S_final), B, H, T, nh, dk, dv, chunk, code,
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_deltaproduct_fwd")
    return out, S_final


def chunk_bwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn_chunk_bwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags))


def chunk_bwd_launches(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn_chunk_bwd_launches(B, H, T, dk, dv, chunk, dtype_code, flags))


def chunk_bwd(q, k, v, alpha, beta, S0, dout, dS_final=None, *, beta_v=None, chunk=32,
              alpha_scalar=False, beta_scalar=False, workspace=None, stream=None):
    """Backward of chunk_fwd / plus_chunk_fwd through gdn_chunk_bwd.

    Same inputs as the forward plus the cotangents dout ([B,T,H,dv], q's dtype) and
    dS_final (float32 [B,H,dk,dv] or None).  Returns a dict of float32 gradients:
    q, k, v, alpha, beta (and beta_v when given), S0.
    """
    code = _dtype_code(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _check(t, n, q.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta"), (beta_v, "beta_v"), (S0, "S0"),
                 (dS_final, "dS_final")):
        _check(t, n, torch.float32)
    flags = (GDN_ALPHA_SCALAR if alpha_scalar else 0) | (GDN_BETA_SCALAR if beta_scalar else 0)
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"q": torch.empty((B, T, H, dk), **f32), "k": torch.empty((B, T, H, dk), **f32),
         "v": torch.empty((B, T, H, dv), **f32), "alpha": torch.empty(alpha.shape, **f32),
         "beta": torch.empty(beta.shape, **f32), "S0": torch.empty((B, H, dk, dv), **f32)}
    if beta_v is not None:
        g["beta_v"] = torch.empty(beta_v.shape, **f32)
    need = chunk_bwd_workspace_size(B, H, T, dk, dv, chunk, code, flags)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().gdn_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(beta_v), _ptr(S0),
                             _ptr(dout), _ptr(dS_final), _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]),
                             _ptr(g["alpha"]), _ptr(g["beta"]), _ptr(g.get("beta_v")), _ptr(g["S0"]),
                             B, H, T, dk, dv, chunk, code, flags, _ptr(workspace), workspace.numel(),
                             _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_chunk_bwd")
    return g


GDN2_NONE, GDN2_CLIP_DECAY, GDN2_SHRINK_J = 0, 1, 2


def gdn2_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags) -> int:
    return int(lib().gdn2_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, dtype_code, flags))


def gdn2_chunk_fwd(q, k, v, alpha, eta, b_gate, S0=None, *, mode=GDN2_NONE, chunk=32,
                   alpha_scalar=False, out=None, S_final=None, want_state=True, workspace=None,
                   stream=None):
    """GDN2 (non-tied erase j' = eta k^ (.) b, write k^) through gdn2_chunk_fwd, with the
    token-wise stability transform `mode` (GDN2_NONE / GDN2_CLIP_DECAY / GDN2_SHRINK_J).
    q, k [B,T,H,dk], v [B,T,H,dv]; alpha float32 [B,T,H,dk] (or [B,T,H]); eta float32
    [B,T,H]; b_gate float32 [B,T,H,dk]; S0 float32 [B,H,dk,dv] or None."""
    code = _dtype_code(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype)
    for t, n in ((alpha, "alpha"), (eta, "eta"), (b_gate, "b_gate"), (S0, "S0")):
        _check(t, n, torch.float32)
    flags = GDN_ALPHA_SCALAR if alpha_scalar else 0
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = gdn2_chunk_fwd_workspace_size(B, H, T, dk, dv, chunk, code, flags)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = lib().gdn2_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(eta), _ptr(b_gate), _ptr(S0),
                              _ptr(out), _ptr(S_final), B, H, T, dk, dv, chunk, code, flags, int(mode),
                              _ptr(workspace), workspace.numel(), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn2_chunk_fwd")
    return out, S_final


def recurrent_step(q, k, v, alpha, beta_k, S_in=None, *, beta_v=None, alpha_scalar=False,
                   beta_scalar=False, out=None, S_out=None, in_place=False, stream=None):
    """One recurrent (decode) step through gdn_recurrent_step.

    q, k [B,H,dk], v [B,H,dv] (bf16 or float32); alpha/beta_k float32 [B,H,dk] or [B,H];
    beta_v float32 [B,H,dv] / [B,H] or None; S_in float32 [B,H,dk,dv] or None.  With
    in_place=True the new state overwrites S_in.  Returns (out [B,H,dv], S_out).
    """
    code = _dtype_code(q)
    B, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype)
    for t, n in ((alpha, "alpha"), (beta_k, "beta_k"), (beta_v, "beta_v"), (S_in, "S_in")):
        _check(t, n, torch.float32)
    flags = (GDN_ALPHA_SCALAR if alpha_scalar else 0) | (GDN_BETA_SCALAR if beta_scalar else 0)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    if S_out is None:
        if in_place:
            if S_in is None:
                raise ValueError("in_place needs S_in")
            S_out = S_in
        else:
            S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype)
    _check(S_out, "S_out", torch.float32)
    st = lib().gdn_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k), _ptr(beta_v),
                                  _ptr(S_in), _ptr(S_out), _ptr(out), B, H, dk, dv, code, flags,
                                  _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_recurrent_step")
    return out, S_out


def workspace_status(workspace, stream=None) -> int:
    """Device-side status recorded in `workspace` (waits for the stream, then clears it)."""
    return int(lib().gdn_workspace_status(_ptr(workspace), _stream(stream)))

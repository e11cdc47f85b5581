"""ctypes wrapper around the fp64 C oracle (gdn_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, the smoke check and the CPU
baseline of bench.py, never by the product path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_lib = None


def host_cpu() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _so_path() -> str:
    """The library is built with -march=native, so its file name carries a hash of the host
    CPU's model and feature flags: a copy built on another machine is never loaded."""
    import hashlib
    ident = host_cpu()
    try:
        with open("/proc/cpuinfo") as f:
            flags = next((l for l in f if l.startswith("flags")), "")
        ident += flags
    except OSError:
        pass
    tag = hashlib.sha256(ident.encode()).hexdigest()[:12]
    return os.path.join(_BUILD, f"libgdn_oracle_{tag}.so")


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into oracle/_build/ (gcc -O3 -march=native, OpenMP)."""
    so = _so_path()
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(_SRC):
        tmp = so + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-march=native", "-fopenmp", "-shared", "-fPIC", "-o", tmp,
                               _SRC, "-lm"])
        os.replace(tmp, so)
    return so


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        f = ctypes.c_void_p
        i = ctypes.c_int
        _lib.oracle_gdn_seq.argtypes = [f, f, f, f, f, f, f, f, f, i, i, i, i, i, i, i,
                                        ctypes.c_double, f, i, i]
        _lib.oracle_gdn_seq.restype = i
        _lib.oracle_deltaproduct_seq.argtypes = [f, f, f, f, f, f, f, f, i, i, i, i, i, i,
                                                 ctypes.c_double, f, i, i]
        _lib.oracle_deltaproduct_seq.restype = i
        _lib.oracle_max_threads.restype = i
    return _lib


def _f32(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _pairs(pairs):
    if pairs is None:
        return None, 0
    arr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    return arr, arr.shape[0]


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def gdn_seq(q, k, v, alpha, beta, S0=None, *, alpha_scalar=False, beta_scalar=False,
            eps=1e-6, pairs=None, nthreads=0, beta_v=None):
    """Token-by-token FG^2-GDN recurrence in fp64.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; alpha, beta: [B,T,H,dk] or [B,T,H] when
    scalar; S0: [B,H,dk,dv] or None (zero state).  beta_v ([B,T,H,dv], or [B,T,H]
    when scalar) selects FG^2-GDN+: beta then scales the keys and beta_v the values.
    Inputs are read as float32
    values (bf16 data must be passed exactly upcast).  Returns (o, S_final) in
    float64, o [B,T,H,dv], S_final [B,H,dk,dv].  With `pairs` (a list of
    (b, h)), only those heads are computed and the other entries stay zero.
    """
    q, k, v, alpha, beta, beta_v, S0 = map(_f32, (q, k, v, alpha, beta, beta_v, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    sf = np.zeros((B, H, dk, dv), dtype=np.float64)
    parr, npairs = _pairs(pairs)
    rc = lib().oracle_gdn_seq(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(beta_v), _ptr(S0),
                              _ptr(o), _ptr(sf), B, H, T, dk, dv, int(alpha_scalar),
                              int(beta_scalar), float(eps), _ptr(parr), npairs, int(nthreads))
    if rc != 0:
        raise ValueError("channel-wise beta needs dk == dv (or a separate beta_v)")
    return o, sf


def deltaproduct_seq(q, k, v, gamma, beta, S0=None, *, eps=1e-6, pairs=None, nthreads=0):
    """DeltaProduct n_h with a scalar forget gate, token by token in fp64.

    q: [B,T,H,dk]; k: [B,T,H,nh,dk]; v: [B,T,H,nh,dv]; gamma: [B,T,H];
    beta: [B,T,H,nh].  Returns (o [B,T,H,dv], S_final [B,H,dk,dv]) in float64.
    """
    q, k, v, gamma, beta, S0 = map(_f32, (q, k, v, gamma, beta, S0))
    B, T, H, nh, dk = k.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    sf = np.zeros((B, H, dk, dv), dtype=np.float64)
    parr, npairs = _pairs(pairs)
    lib().oracle_deltaproduct_seq(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(S0),
                                  _ptr(o), _ptr(sf), B, H, T, nh, dk, dv, float(eps),
                                  _ptr(parr), npairs, int(nthreads))
    return o, sf

"""Helpers shared by the GPU parity tests: device transfer and the tolerance check."""
from __future__ import annotations

import os

import numpy as np

# Tolerances of the method's stated acceptance metric max|x - ref| / RMS(ref):
TOL_F32 = 1e-4      # float32 path
TOL_BF16 = 2e-2     # bf16 inputs, fp32 accumulation


def to_dev(x, dtype=None):
    import torch
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(dtype) if dtype is not None else t


def bf16_half_ulp(x):
    """Half a bf16 ulp at |x|'s binade: 2^(floor(log2|x|) - 8), 0 at 0."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    out = np.zeros_like(ax)
    nz = ax > 0
    out[nz] = np.exp2(np.floor(np.log2(ax[nz])) - 8.0)
    return out


# Every parity() call appends (test id, kind, plain max|err|/RMS, tol): the conftest prints the
# worst plain figures at the end of the run, so a passing run shows how close the bf16 path
# comes to the literal bound as well as to the per-element allowance.
RECORDS = []


def parity(got, ref, tol, out_bf16=False):
    """Element-wise check err_i <= tol * RMS(ref) (+ the bf16 half-ulp of the element when
    the output is stored as bf16).  Returns (max err / RMS, max excess / RMS)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0.0:
        rms = 1.0
    err = np.abs(got - ref)
    allow = tol * rms
    if out_bf16:
        allow = allow + bf16_half_ulp(np.maximum(np.abs(got), np.abs(ref)))
    excess = float(np.max(err - allow)) if err.size else 0.0
    RECORDS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0],
                    "bf16-out" if out_bf16 else ("f32" if tol < 1e-3 else "bf16-path f32"),
                    float(err.max() / rms) if err.size else 0.0, tol))
    assert excess <= 0.0, (f"max|err|/RMS = {err.max() / rms:.4g}, worst excess over the allowance "
                           f"{excess / rms:.4g} RMS (tol {tol})")
    return (float(err.max() / rms) if err.size else 0.0), excess / rms

"""Seeded synthetic inputs for the FG^2-GDN forward (numpy only).

This module is shared by the tests, the benchmark and the oracle-side checks.
It holds none of the method's arithmetic: it draws random numbers, applies the
gate activations that produce alpha / beta / gamma values in their documented
ranges, and rounds to bf16 where a configuration stores bf16.

Recipe (one numpy PCG64 generator per configuration, seeded with the
configuration number; draws in the order q, k, v, alpha-logits, beta-logits,
S0; DeltaProduct: q, k, v, beta, gamma-logits):
  q, k, v  ~ N(0, 1)                        (q, k are normalised inside the op)
  alpha    = exp(-s * softplus(x)), x ~ N(0, 1), s = 0.1 (0.02 for near-1 decay)
  beta     = sigmoid(x), x ~ N(0, std)      (std 1, or 2 for the wide config)
  S0       = 0, or ~ N(0, std 0.01)
  beta_v   = sigmoid(x), x ~ N(0, std)      (FG^2-GDN+ only; drawn last, after S0,
                                             [B,T,H,dv], or [B,T,H] with scalar beta)
GDN2 (make_gdn2_inputs): q, k, v ~ N(0,1); alpha as above; eta = 2 sigmoid(N(0,1)) in
  (0, 2); b = sigmoid(N(0, 2)) in (0, 1); S0 ~ N(0, s0_std); drawn in that order.
  DeltaProduct: beta ~ U[0, 2] per sub-step, gamma = sigmoid(x), x ~ N(2, 1)
bf16 tensors are rounded to nearest-even from the float32 draws; the float32
copy kept alongside holds exactly the rounded values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    r = (u + np.uint32(0x7FFF) + lsb) >> 16
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bf16 (returned as float32)."""
    return bf16_to_f32(bf16_bits(x))


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


@dataclass
class GdnConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str = "bf16"              # storage dtype of q, k, v and o: "bf16" or "f32"
    alpha_scale: float = 0.1         # alpha = exp(-alpha_scale * softplus(N(0,1)))
    alpha_scalar: bool = False
    beta_std: float = 1.0            # beta = sigmoid(N(0, beta_std))
    beta_scalar: bool = False
    s0_std: float = 0.0              # 0 -> S0 is None
    deltaproduct_nh: int = 0         # > 0 -> DeltaProduct with this many sub-steps
    plus: bool = False               # FG^2-GDN+: a separate value rate beta_v
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads the operator is specified on (shapes, dtypes and
# distributions as stated with the method's target); seed = index.
CONFIGS = {
    "fg2_f32_small": GdnConfig("fg2_f32_small", B=1, H=2, T=256, dk=32, dv=32, chunk=16,
                               dtype="f32", seed=1),
    "kda_bf16": GdnConfig("kda_bf16", B=4, H=16, T=4096, dk=128, dv=128, chunk=64,
                          beta_scalar=True, s0_std=0.01, seed=2),
    "fg2_prefill_32k": GdnConfig("fg2_prefill_32k", B=1, H=16, T=32768, dk=128, dv=128,
                                 chunk=64, seed=3),
    "fg2_train_b8": GdnConfig("fg2_train_b8", B=8, H=16, T=4096, dk=128, dv=128, chunk=64,
                              alpha_scale=0.02, beta_std=2.0, s0_std=0.01, seed=4),
    "deltaproduct_nh2": GdnConfig("deltaproduct_nh2", B=2, H=8, T=8192, dk=128, dv=128,
                                  chunk=64, deltaproduct_nh=2, seed=5),
}


def make_inputs(cfg: GdnConfig, *, seed: int | None = None, T: int | None = None,
                B: int | None = None, H: int | None = None) -> dict:
    """Draw one batch of inputs for `cfg` (optionally with smaller B/H/T).

    Returns a dict of float32 numpy arrays holding exactly the stored values
    (q, k, v already rounded to bf16 when cfg.dtype == "bf16"), plus "S0"
    (None when cfg.s0_std == 0).  GDN keys: q k v alpha beta S0.  DeltaProduct
    keys: q k v beta gamma S0 (k, v carry an extra n_h axis).
    """
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    T = cfg.T if T is None else T
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    rb = round_bf16 if cfg.dtype == "bf16" else (lambda a: a)
    f32 = np.float32
    if cfg.deltaproduct_nh > 0:
        nh = cfg.deltaproduct_nh
        q = rb(rng.standard_normal((B, T, H, cfg.dk), dtype=f32))
        k = rb(rng.standard_normal((B, T, H, nh, cfg.dk), dtype=f32))
        v = rb(rng.standard_normal((B, T, H, nh, cfg.dv), dtype=f32))
        beta = rng.uniform(0.0, 2.0, size=(B, T, H, nh)).astype(f32)
        gamma = _sigmoid(rng.normal(2.0, 1.0, size=(B, T, H)).astype(f32)).astype(f32)
        S0 = None
        if cfg.s0_std > 0:
            S0 = (cfg.s0_std * rng.standard_normal((B, H, cfg.dk, cfg.dv), dtype=f32)).astype(f32)
        return dict(q=q, k=k, v=v, beta=beta, gamma=gamma, S0=S0)
    q = rb(rng.standard_normal((B, T, H, cfg.dk), dtype=f32))
    k = rb(rng.standard_normal((B, T, H, cfg.dk), dtype=f32))
    v = rb(rng.standard_normal((B, T, H, cfg.dv), dtype=f32))
    ashape = (B, T, H) if cfg.alpha_scalar else (B, T, H, cfg.dk)
    bshape = (B, T, H) if cfg.beta_scalar else (B, T, H, cfg.dk)
    alpha = np.exp(-cfg.alpha_scale * _softplus(rng.standard_normal(ashape, dtype=f32))).astype(f32)
    beta = _sigmoid(cfg.beta_std * rng.standard_normal(bshape, dtype=f32)).astype(f32)
    S0 = None
    if cfg.s0_std > 0:
        S0 = (cfg.s0_std * rng.standard_normal((B, H, cfg.dk, cfg.dv), dtype=f32)).astype(f32)
    x = dict(q=q, k=k, v=v, alpha=alpha, beta=beta, S0=S0)
    if cfg.plus:
        vshape = (B, T, H) if cfg.beta_scalar else (B, T, H, cfg.dv)
        x["beta_v"] = _sigmoid(cfg.beta_std * rng.standard_normal(vshape, dtype=f32)).astype(f32)
    return x


def make_gdn2_inputs(B: int, T: int, H: int, dk: int, dv: int, *, dtype: str = "f32", seed: int = 0,
                     alpha_scale: float = 0.1, s0_std: float = 0.1) -> dict:
    """Seeded inputs of the GDN2 operator: q k v alpha eta b S0 (float32 numpy arrays
    holding the stored values; q, k, v rounded to bf16 when dtype == "bf16")."""
    rng = np.random.default_rng(seed)
    rb = round_bf16 if dtype == "bf16" else (lambda a: a)
    f32 = np.float32
    q = rb(rng.standard_normal((B, T, H, dk), dtype=f32))
    k = rb(rng.standard_normal((B, T, H, dk), dtype=f32))
    v = rb(rng.standard_normal((B, T, H, dv), dtype=f32))
    alpha = np.exp(-alpha_scale * _softplus(rng.standard_normal((B, T, H, dk), dtype=f32))).astype(f32)
    eta = (2.0 * _sigmoid(rng.standard_normal((B, T, H), dtype=f32))).astype(f32)
    b = _sigmoid(2.0 * rng.standard_normal((B, T, H, dk), dtype=f32)).astype(f32)
    S0 = (s0_std * rng.standard_normal((B, H, dk, dv), dtype=f32)).astype(f32) if s0_std > 0 else None
    return dict(q=q, k=k, v=v, alpha=alpha, eta=eta, b=b, S0=S0)

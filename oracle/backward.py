"""Gradients of the FG^2-GDN forward: fp64 autograd through the token-by-token
recurrence (plain PyTorch CPU ops).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The gradient of a loss L(o, S_final) is, by definition, the derivative of the
forward map; here the forward map is eq. (11) of the FG^2-GDN reading notes
(sec. 2.2; eq. (13) of sec. 2.3 for the split rates of FG^2-GDN+) written out one
token at a time, and torch.autograd (a library primitive) takes the derivative.
Callers give the output cotangents dO and dS_final; the returned gradients are
those of  L = <o, dO> + <S_final, dS_final>.

Pinned (tests/test_oracle_pins.py) by central finite differences on tiny inputs
and by closed forms (the gradient of o_1 for T = 1 and a zero state).
Long sequences use torch.utils.checkpoint over segments of the token loop, a
memory device only: every token is still differentiated in fp64.
"""
from __future__ import annotations

import numpy as np
import torch
from torch.utils.checkpoint import checkpoint


def _normalise(x, eps):
    return x / torch.sqrt((x * x).sum(-1, keepdim=True) + eps)


def _segment(S, q, k, v, alpha, beta, beta_v, eps, alpha_scalar, beta_scalar):
    """Tokens of one segment; q, k [B,n,H,dk], v [B,n,H,dv]; S [B,H,dk,dv]."""
    outs = []
    for t in range(q.shape[1]):
        qn = _normalise(q[:, t], eps)                           # [B,H,dk]
        kn = _normalise(k[:, t], eps)
        a = alpha[:, t][..., None] if alpha_scalar else alpha[:, t]
        bk = beta[:, t][..., None] if beta_scalar else beta[:, t]
        src = beta if beta_v is None else beta_v
        bv = src[:, t][..., None] if beta_scalar else src[:, t]
        kt = torch.sqrt(bk) * kn                                # k~ = sqrt(beta^k) (.) k^
        vt = torch.sqrt(bv) * v[:, t]                           # v~ = sqrt(beta^v) (.) v
        X = a[..., None] * S                                    # Diag(alpha) S
        u = vt - torch.einsum("bhc,bhcj->bhj", kt, X)           # v~ - X^T k~
        S = X + kt[..., None] * u[..., None, :]                 # (I - k~ k~^T) X + k~ v~^T
        outs.append(torch.einsum("bhcj,bhc->bhj", S, qn))       # o = S^T q^
    return S, torch.stack(outs, dim=1)


def gdn_forward_torch(q, k, v, alpha, beta, S0=None, *, beta_v=None, alpha_scalar=False,
                      beta_scalar=False, eps=1e-6, segment=256):
    """Differentiable fp64 forward.  Tensors as in oracle.gdn_seq (float64 torch).
    Returns (o [B,T,H,dv], S_final [B,H,dk,dv])."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = torch.zeros(B, H, dk, dv, dtype=torch.float64) if S0 is None else S0
    outs = []
    for s0 in range(0, T, segment):
        sl = slice(s0, min(T, s0 + segment))
        args = (S, q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], beta[:, sl],
                None if beta_v is None else beta_v[:, sl])
        if T > segment and torch.is_grad_enabled():
            S, o = checkpoint(_segment, *args, eps, alpha_scalar, beta_scalar, use_reentrant=False)
        else:
            S, o = _segment(*args, eps, alpha_scalar, beta_scalar)
        outs.append(o)
    o = torch.cat(outs, dim=1) if outs else torch.zeros(B, 0, H, dv, dtype=torch.float64)
    return o, S


def gdn_grads(q, k, v, alpha, beta, S0, dO, dS_final=None, *, beta_v=None, alpha_scalar=False,
              beta_scalar=False, eps=1e-6, pairs=None):
    """Gradients of <o, dO> + <S_final, dS_final> with respect to every input.

    numpy inputs (read as float32 values, computed in float64).  S0 None means a zero
    initial state (its gradient is still returned).  With `pairs` (list of (b, h)) only
    those heads are differentiated; other entries of the results stay zero.
    Returns a dict of float64 arrays: q k v alpha beta S0 (and beta_v when given), plus
    "o" and "S_final" of the forward.
    """
    f64 = lambda a: None if a is None else torch.from_numpy(np.asarray(a, dtype=np.float32).astype(np.float64))
    B, T, H, dk = np.shape(q)
    dv = np.shape(v)[-1]
    if S0 is None:
        S0 = np.zeros((B, H, dk, dv), dtype=np.float32)
    if dS_final is None:
        dS_final = np.zeros((B, H, dk, dv), dtype=np.float32)
    names = ["q", "k", "v", "alpha", "beta", "S0"] + (["beta_v"] if beta_v is not None else [])
    full = dict(q=q, k=k, v=v, alpha=alpha, beta=beta, S0=S0, beta_v=beta_v)
    res = {n: np.zeros(np.shape(full[n]), dtype=np.float64) for n in names}
    res["o"] = np.zeros((B, T, H, dv))
    res["S_final"] = np.zeros((B, H, dk, dv))
    groups = [(b, h) for b in range(B) for h in range(H)] if pairs is None else list(pairs)
    for b, h in groups:
        def take(a, has_t=True):
            a = np.asarray(a)
            return a[b:b + 1, :, h:h + 1] if has_t else a[b:b + 1, h:h + 1]
        ins = {n: f64(take(full[n], n != "S0")).requires_grad_(True) for n in names}
        o, S = gdn_forward_torch(ins["q"], ins["k"], ins["v"], ins["alpha"], ins["beta"], ins["S0"],
                                 beta_v=ins.get("beta_v"), alpha_scalar=alpha_scalar,
                                 beta_scalar=beta_scalar, eps=eps)
        loss = (o * f64(take(dO))).sum() + (S * f64(take(dS_final, False))).sum()
        grads = torch.autograd.grad(loss, [ins[n] for n in names], allow_unused=True)
        for n, g in zip(names, grads):
            if g is None:
                continue
            if n == "S0":
                res[n][b, h] = g.numpy()[0, 0]
            else:
                res[n][b, :, h] = g.numpy()[0, :, 0]
        res["o"][b, :, h] = o.detach().numpy()[0, :, 0]
        res["S_final"][b, h] = S.detach().numpy()[0, 0]
    return res

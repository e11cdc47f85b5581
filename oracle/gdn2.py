"""GDN2 (non-tied erase / write directions) with its token-wise stability transforms,
fp64 numpy, token by token.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: Su Jianlin's note on GDN2 stability ("Problem Description", eq. (spec) in
"The Spectral Norm", "Simple Strategy", "Modifying Itself").  The note writes the state
as d_v x d_k and the update as S_t = S_{t-1} D_t (I - eta_t j_t k_t^T) + eta_t v_t k_t^T.
This library keeps the state as X = S^T (d_k x d_v), so the same update reads

    X_t = (I - eta_t k_t j_t^T) D_t X_{t-1} + eta_t k_t v_t^T ,   o_t = X_t^T q_t .

Readings (none is fixed by the note):
  - k and q are L2-normalised as everywhere in this library (x / sqrt(sum x^2 + eps));
    the note assumes a normalised k.
  - j is GDN2's own parameterisation j = k^ (.) b with b in [0, 1]^{d_k} (the note's
    closing remark), so j^T k^ >= 0.
  - eta is absorbed into j for the transforms (j' = eta j), as "Modifying Itself" does;
    the write term keeps eta: X_t = D X + k^ (eta v - (D X)^T j')^T.
  - mode "clip": D -> min(D, 1/rho), rho = ||I - j' k^T||_2 from the closed form with
    ||k|| = 1: (||j'|| + sqrt(||j'||^2 - 4 j'^T k + 4)) / 2 ("Simple Strategy").
  - mode "shrink": c = j'^T k, gamma_max = max_i D_ii, tau = (c - 1) gamma_max + 1/gamma_max,
    lambda* = min(1, sqrt((tau^2 - c^2) / (||j'||^2 - c^2))), j* = c k + lambda* (j' - c k)
    ("Modifying Itself"); lambda* = 1 when ||j'||^2 = c^2 (j' already along k), and the
    radicand is clamped at 0.
"""
from __future__ import annotations

import numpy as np

MODES = {"none": 0, "clip": 1, "shrink": 2}


def _unit(x, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def transform(k_hat, b, eta, alpha, mode):
    """Token-wise transforms for arrays [..., d] (k_hat, b, alpha) and [...] (eta).
    Returns (j', D): the erase vector with eta absorbed, and the (possibly clipped) decay."""
    k_hat = np.asarray(k_hat, dtype=np.float64)
    jp = np.asarray(eta, dtype=np.float64)[..., None] * k_hat * np.asarray(b, dtype=np.float64)
    D = np.asarray(alpha, dtype=np.float64).copy()
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    if m == 0:
        return jp, D
    c = np.sum(jp * k_hat, axis=-1)
    nj2 = np.sum(jp * jp, axis=-1)
    if m == 1:
        rho = (np.sqrt(nj2) + np.sqrt(np.maximum(nj2 - 4.0 * c + 4.0, 0.0))) / 2.0
        return jp, np.minimum(D, (1.0 / rho)[..., None])
    gmax = np.max(D, axis=-1)
    tau = (c - 1.0) * gmax + 1.0 / gmax
    den = nj2 - c * c
    lam = np.where(den > 0.0, np.sqrt(np.maximum(tau * tau - c * c, 0.0) / np.where(den > 0.0, den, 1.0)), 1.0)
    lam = np.minimum(1.0, lam)
    ck = c[..., None] * k_hat
    return ck + lam[..., None] * (jp - ck), D


def gdn2_seq(q, k, v, alpha, eta, b, S0=None, *, mode="none", eps=1e-6):
    """Token-by-token GDN2.  q, k, b, alpha: [B,T,H,dk]; v: [B,T,H,dv]; eta: [B,T,H];
    S0: [B,H,dk,dv] or None.  Inputs read as float32 values.  Returns (o, S_final), fp64."""
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float32).astype(np.float64)
    q, k, v, alpha, eta, b, S0 = map(f, (q, k, v, alpha, eta, b, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    qh = _unit(q, eps)
    kh = _unit(k, eps)
    jp, D = transform(kh, b, eta, alpha, mode)
    for bb in range(B):
        for h in range(H):
            X = np.zeros((dk, dv)) if S0 is None else S0[bb, h].copy()
            for t in range(T):
                A = np.eye(dk) - np.outer(kh[bb, t, h], jp[bb, t, h])
                X = A @ (D[bb, t, h][:, None] * X) + eta[bb, t, h] * np.outer(kh[bb, t, h], v[bb, t, h])
                o[bb, t, h] = X.T @ qh[bb, t, h]
            sf[bb, h] = X
    return o, sf


def gdn2_chunked(q, k, v, alpha, eta, b, S0=None, *, chunk, mode="none", eps=1e-6):
    """The same recurrence chunk by chunk in the non-tied WY form: with write vectors
    w = k^, erase vectors e = j', values v~ = eta v and g the in-chunk cumulative log D,
        A_ri = sum_c e_rc w_ic e^{g_rc - g_ic} (i < r),  (I + A) U = V~ - (E e^g) S,
        O = (Q^ e^g) S + P U,  P_ri = sum_c q_rc w_ic e^{g_rc - g_ic} (i <= r),
        S <- Diag(e^{g_C}) S + (W e^{g_C - g})^T U ."""
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float32).astype(np.float64)
    q, k, v, alpha, eta, b, S0 = map(f, (q, k, v, alpha, eta, b, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    qh = _unit(q, eps)
    kh = _unit(k, eps)
    jp, D = transform(kh, b, eta, alpha, mode)
    for bb in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[bb, h].copy()
            w, e, vt = kh[bb, :, h], jp[bb, :, h], eta[bb, :, h][:, None] * v[bb, :, h]
            for c0 in range(0, T, chunk):
                r = slice(c0, min(T, c0 + chunk))
                n = r.stop - r.start
                g = np.cumsum(np.log(D[bb, r, h]), axis=0)
                low = np.tril(np.ones((n, n), dtype=bool))
                Dm = np.exp(np.where(low[:, :, None], g[:, None, :] - g[None, :, :], -np.inf))
                A = np.einsum("rc,ic,ric->ri", e[r], w[r], Dm) * np.tril(np.ones((n, n)), -1)
                P = np.einsum("rc,ic,ric->ri", qh[bb, r, h], w[r], Dm)
                R = vt[r] - (e[r] * np.exp(g)) @ S
                U = np.zeros((n, dv))
                for i in range(n):
                    U[i] = R[i] - A[i, :i] @ U[:i]
                o[bb, r, h] = (qh[bb, r, h] * np.exp(g)) @ S + P @ U
                S = np.exp(g[-1])[:, None] * S + (w[r] * np.exp(g[-1][None, :] - g)).T @ U
            sf[bb, h] = S
    return o, sf

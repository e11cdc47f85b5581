"""Chunked (WY / UT) form of the FG^2-GDN recurrence, fp64 numpy.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

This is the oracle's second, independent evaluation of eq. (11) of the
FG^2-GDN reading notes (sec. 2.2), following the chunkwise scheme named in
sec. 2.4 of the same notes ("split the sequence into chunks of length C,
accumulate the transitions inside a chunk in parallel, pass the state from
chunk to chunk") and the DPLR form of the transition given there,
Diag(alpha_t) + a_t b_t^T with a_t = -k~_t, b_t = k~_t (.) alpha_t.

Derivation used (state S at the start of a chunk, rows r = 1..n of the chunk,
g_r = sum_{s<=r} log alpha_s taken per channel inside the chunk):
    u_r  = v~_r - (Diag(alpha_r) S_{r-1})^T k~_r   (the per-token correction)
    A_ri = sum_c k~_rc k~_ic exp(g_rc - g_ic)      (i < r)
    (I + A) U = V~ - (K~ (.) e^g) S                (solved by forward substitution)
    O    = (Q^ (.) e^g) S + P U,  P_ri = sum_c q^_rc k~_ic exp(g_rc - g_ic)  (i <= r)
    S   <- Diag(e^{g_n}) S + (K~ (.) e^{g_n - g})^T U
The decay factors exp(g_r - g_i) are formed element by element for i <= r
only, so no factor ever exceeds 1 and nothing overflows.  No blocking,
fusion or reordering beyond this is done.
"""
from __future__ import annotations

import numpy as np


def _normalise(x, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def gdn_chunked(q, k, v, alpha, beta, S0=None, *, chunk, alpha_scalar=False,
                beta_scalar=False, eps=1e-6, beta_v=None):
    """Chunkwise evaluation of the recurrence; same arguments and returns as
    oracle.gdn_seq (o [B,T,H,dv], S_final [B,H,dk,dv], both float64).  With beta_v
    (FG^2-GDN+, reading notes sec. 2.3 eq. (13)) the values are scaled by sqrt(beta_v)."""
    q = np.asarray(q, dtype=np.float32).astype(np.float64)
    k = np.asarray(k, dtype=np.float32).astype(np.float64)
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    alpha = np.asarray(alpha, dtype=np.float32).astype(np.float64)
    beta = np.asarray(beta, dtype=np.float32).astype(np.float64)
    if beta_v is not None:
        beta_v = np.asarray(beta_v, dtype=np.float32).astype(np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if not beta_scalar and beta_v is None and dk != dv:
        raise ValueError("channel-wise beta needs dk == dv")
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float32)[b, h].astype(np.float64)
            qh = _normalise(q[b, :, h], eps)
            kh = _normalise(k[b, :, h], eps)
            src_v = beta if beta_v is None else beta_v
            if beta_scalar:
                bk = np.repeat(beta[b, :, h][:, None], dk, axis=1)
                bv = np.repeat(src_v[b, :, h][:, None], dv, axis=1)
            else:
                bk = beta[b, :, h]
                bv = src_v[b, :, h]
            al = np.repeat(alpha[b, :, h][:, None], dk, axis=1) if alpha_scalar else alpha[b, :, h]
            kt = np.sqrt(bk) * kh
            vt = np.sqrt(bv) * v[b, :, h]
            for c0 in range(0, T, chunk):
                r = slice(c0, min(T, c0 + chunk))
                n = r.stop - r.start
                g = np.cumsum(np.log(al[r]), axis=0)                       # (n, dk)
                lower = np.tril(np.ones((n, n), dtype=bool))               # i <= r
                expo = np.where(lower[:, :, None], g[:, None, :] - g[None, :, :], -np.inf)
                D = np.exp(expo)                                           # (n, n, dk): [r, i, c]
                A = np.einsum("rc,ic,ric->ri", kt[r], kt[r], D) * np.tril(np.ones((n, n)), -1)
                P = np.einsum("rc,ic,ric->ri", qh[r], kt[r], D)
                Gam = np.exp(g)
                R = vt[r] - (kt[r] * Gam) @ S
                U = np.zeros((n, dv))
                for i in range(n):                                          # forward substitution
                    U[i] = R[i] - A[i, :i] @ U[:i]
                o[b, r, h] = (qh[r] * Gam) @ S + P @ U
                S = np.exp(g[-1])[:, None] * S + (kt[r] * np.exp(g[-1][None, :] - g)).T @ U
            sf[b, h] = S
    return o, sf

"""Closed forms about the delta-rule transition, fp64 numpy.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

- Spectral norm of I - eta j k^T: Su Jianlin's note on GDN2 stability
  (kexue.fm translation 11945), section "The Spectral Norm", eq. (spec), and
  the unnormalised form in "Modifying Itself".
- The shrink of j toward KDA that keeps j*^T k = c and caps the norm at
  1/gamma_max: same note, "Modifying Itself" (tau and lambda*).
- The secular equation of the diagonal-plus-rank-1 transition
  diag(w) - kappa (a (.) kappa)^T: secularmode README, "An exact secular
  spectrum" and "Retention is safe; instability is only from below".
"""
from __future__ import annotations

import numpy as np


def rank1_spectral_norm(j, k, eta=1.0):
    """||I - eta j k^T||_2 from the closed form.

    With unit j, k the note gives (eta + sqrt(eta^2 - 4 eta j^T k + 4)) / 2.
    For general vectors the norms are absorbed as the note describes: k is
    normalised and its norm, together with eta, moves into j; then the
    unnormalised form (||j|| + sqrt(||j||^2 - 4 j^T k + 4)) / 2 applies.
    """
    j = np.asarray(j, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    nk = np.linalg.norm(k)
    if nk == 0.0 or eta == 0.0:
        return 1.0
    jj = eta * nk * j
    ku = k / nk
    nj = np.linalg.norm(jj)
    c = float(jj @ ku)
    # the radicand is >= (||j|| - 2)^2 >= 0 because c <= ||j||; clamp rounding below zero
    return 0.5 * (nj + np.sqrt(max(nj * nj - 4.0 * c + 4.0, 0.0)))


def gdn2_shrink(j, k, gamma_max):
    """j* = c k + lambda* (j - c k) with c = j^T k (k unit), tau = (c-1) gamma_max + 1/gamma_max,
    lambda* = min(1, sqrt((tau^2 - c^2) / (||j||^2 - c^2))).  Needs tau >= c (c >= 0 suffices)."""
    j = np.asarray(j, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    c = float(j @ k)
    tau = (c - 1.0) * gamma_max + 1.0 / gamma_max
    denom = float(j @ j) - c * c
    lam = 1.0 if denom <= 0.0 else min(1.0, np.sqrt(max(tau * tau - c * c, 0.0) / denom))
    return c * k + lam * (j - c * k), lam


def dplr_matrix(w, kappa, a):
    """diag(w) - kappa (a (.) kappa)^T."""
    w, kappa, a = (np.asarray(x, dtype=np.float64) for x in (w, kappa, a))
    return np.diag(w) - np.outer(kappa, a * kappa)


def secular_f(w, kappa, a, lam):
    """f(lambda) = 1 - sum_i a_i kappa_i^2 / (w_i - lambda)."""
    w, kappa, a = (np.asarray(x, dtype=np.float64) for x in (w, kappa, a))
    return 1.0 - np.sum(a * kappa * kappa / (w - lam))


def secular_det(w, kappa, a, lam):
    """det(A - lambda I) = prod_i (w_i - lambda) * f(lambda)."""
    w = np.asarray(w, dtype=np.float64)
    return float(np.prod(w - lam)) * secular_f(w, kappa, a, lam)


def over_removal_budget(w, kappa, a):
    """sum_i a_i kappa_i^2 / (w_i + 1); -1 is an eigenvalue exactly when this equals 1."""
    w, kappa, a = (np.asarray(x, dtype=np.float64) for x in (w, kappa, a))
    return float(np.sum(a * kappa * kappa / (w + 1.0)))

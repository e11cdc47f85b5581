"""Pins of the GDN2 oracle (oracle.gdn2) to Su Jianlin's GDN2 stability note and to
independent computations: the KDA special case through the C oracle, brute-force SVD
of every token's transition after each transform, and two algorithms (token by token
vs non-tied WY chunks)."""
import numpy as np
import pytest

import oracle
from oracle import gdn2


def _inputs(seed, T=9, H=2, dk=6, dv=5, eta_max=1.5):
    r = np.random.default_rng(seed)
    f = np.float32
    return dict(q=r.standard_normal((1, T, H, dk)).astype(f), k=r.standard_normal((1, T, H, dk)).astype(f),
                v=r.standard_normal((1, T, H, dv)).astype(f),
                alpha=r.uniform(0.5, 1.0, (1, T, H, dk)).astype(f),
                eta=r.uniform(0.1, eta_max, (1, T, H)).astype(f),
                b=r.uniform(0.0, 1.0, (1, T, H, dk)).astype(f),
                S0=r.standard_normal((1, H, dk, dk)).astype(f)[..., :dv].copy())


def test_kda_special_case_through_the_c_oracle():
    """j = k (b = 1): GDN2 is KDA with write rate eta ("Problem Description": KDA is k = j),
    i.e. FG^2-GDN with scalar beta = eta."""
    x = _inputs(1, dv=6)
    b1 = np.ones_like(x["b"])
    o1, s1 = gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], b1, x["S0"])
    o2, s2 = oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], x["S0"], beta_scalar=True)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-12)


def test_clip_bounds_every_transition_by_one():
    """Simple Strategy: with D -> min(D, 1/rho), ||D (I - j' k^T)||_2 <= 1 for every token
    (brute-force SVD), and only entries above 1/rho change."""
    x = _inputs(2, T=40, eta_max=2.5)
    kh = x["k"].astype(np.float64) / np.linalg.norm(x["k"].astype(np.float64), axis=-1, keepdims=True)
    jp, D = gdn2.transform(kh, x["b"], x["eta"], x["alpha"], "clip")
    for idx in np.ndindex(x["eta"].shape):
        A = np.eye(6) - np.outer(jp[idx], kh[idx])
        rho = np.linalg.norm(A, 2)
        assert np.linalg.norm(D[idx][:, None] * A, 2) <= 1.0 + 1e-12
        a = x["alpha"][idx].astype(np.float64)
        np.testing.assert_array_equal(D[idx] == a, a <= 1.0 / rho + 1e-15)


def test_closed_form_rho_matches_svd():
    """eq. (spec) with eta absorbed: ||I - j k^T||_2 = (||j|| + sqrt(||j||^2 - 4 j^T k + 4)) / 2."""
    r = np.random.default_rng(3)
    for _ in range(50):
        k = r.standard_normal(7)
        k /= np.linalg.norm(k)
        j = r.uniform(0, 2) * k * r.uniform(0, 1, 7)
        nj, c = np.linalg.norm(j), j @ k
        closed = (nj + np.sqrt(nj * nj - 4 * c + 4)) / 2
        assert abs(closed - np.linalg.norm(np.eye(7) - np.outer(j, k), 2)) < 1e-12


def test_shrink_keeps_erase_rate_and_bounds_norm():
    """Modifying Itself: j*^T k = j'^T k, ||I - j* k^T||_2 <= 1/gamma_max (equal when the
    shrink is active), and gamma_max = 1 gives j* = c k (KDA)."""
    x = _inputs(4, T=60, eta_max=2.5)
    kh = x["k"].astype(np.float64) / np.linalg.norm(x["k"].astype(np.float64), axis=-1, keepdims=True)
    jp0, _ = gdn2.transform(kh, x["b"], x["eta"], x["alpha"], "none")
    js, D = gdn2.transform(kh, x["b"], x["eta"], x["alpha"], "shrink")
    np.testing.assert_array_equal(D, x["alpha"].astype(np.float64))
    active = 0
    for idx in np.ndindex(x["eta"].shape):
        c0, c1 = jp0[idx] @ kh[idx], js[idx] @ kh[idx]
        assert abs(c0 - c1) < 1e-12
        gmax = x["alpha"][idx].astype(np.float64).max()
        n_star = np.linalg.norm(np.eye(6) - np.outer(js[idx], kh[idx]), 2)
        assert n_star <= 1.0 / gmax + 1e-9
        if np.linalg.norm(js[idx] - jp0[idx]) > 1e-12:
            active += 1
            assert abs(n_star - 1.0 / gmax) < 1e-9
    assert active > 0
    ones = np.ones_like(x["alpha"])
    js1, _ = gdn2.transform(kh, x["b"], x["eta"], ones, "shrink")
    c = np.sum(jp0 * kh, axis=-1, keepdims=True)
    # tau = (c - 1) + 1 recovers c only to rounding, and the square root in lambda* turns
    # a 1e-16 radicand into ~1e-8; without the shrink the difference would be O(1)
    np.testing.assert_allclose(js1, c * kh, rtol=0, atol=1e-7)
    assert np.abs(jp0 - c * kh).max() > 0.1


@pytest.mark.parametrize("mode", ["none", "clip", "shrink"])
@pytest.mark.parametrize("chunk", [1, 5, 16])
def test_sequential_equals_nontied_chunks(mode, chunk):
    x = _inputs(5, T=37, dk=8, dv=4, eta_max=2.0)
    o1, s1 = gdn2.gdn2_seq(**x, mode=mode)
    o2, s2 = gdn2.gdn2_chunked(**x, chunk=chunk, mode=mode)
    assert np.abs(o1 - o2).max() <= 1e-11 * np.sqrt(np.mean(o1 ** 2))
    assert np.abs(s1 - s2).max() <= 1e-11 * np.sqrt(np.mean(s1 ** 2))


def test_clip_is_identity_for_tied_keys_and_small_eta():
    """The "iff": with j = k and eta <= 2, rho = 1, so clipping changes nothing."""
    x = _inputs(6, eta_max=2.0)
    b1 = np.ones_like(x["b"])
    o1, s1 = gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], b1, x["S0"], mode="clip", eps=0.0)
    o2, s2 = gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], b1, x["S0"], mode="none", eps=0.0)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-12)

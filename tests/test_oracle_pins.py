"""Pins of the fp64 oracle against facts the method's pages fix.

None of these tests calls the CUDA library.  Each check ties the oracle to
something other than itself: a closed form, an invariant, a special case that
reduces to a textbook rule, brute-force linear algebra (numpy / torch
autograd) on small inputs, or the oracle's second, independent algorithm.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import spectral

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _gdn_inputs(seed, B=1, T=12, H=2, dk=6, dv=6, alpha_scalar=False, beta_scalar=False,
                s0=True, beta_max=1.0):
    r = _rng(seed)
    q = r.standard_normal((B, T, H, dk)).astype(np.float32)
    k = r.standard_normal((B, T, H, dk)).astype(np.float32)
    v = r.standard_normal((B, T, H, dv)).astype(np.float32)
    ash = (B, T, H) if alpha_scalar else (B, T, H, dk)
    bsh = (B, T, H) if beta_scalar else (B, T, H, dk)
    alpha = r.uniform(0.5, 1.0, ash).astype(np.float32)
    beta = r.uniform(0.0, beta_max, bsh).astype(np.float32)
    S0 = r.standard_normal((B, H, dk, dv)).astype(np.float32) if s0 else None
    return q, k, v, alpha, beta, S0


def _unit(x):
    x = np.asarray(x, dtype=np.float64)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# --------------------------------------------------------------------------- write invariant
def test_write_invariant_unit_key():
    """Delta-rule write (reading notes sec. 2.1, eq. (6); eq. (11)): with ||k~_t|| = 1 the
    updated state satisfies S_t^T k~_t = v~_t exactly."""
    q, k, v, alpha, _, S0 = _gdn_inputs(1, T=10, dk=8, dv=8)
    beta = np.ones_like(alpha)
    # Step one token at a time; the state re-enters through the float32 S0 argument, and
    # the invariant is checked on the fp64 state each single-step call returns.
    S = S0.astype(np.float64)
    for t in range(q.shape[1]):
        sl = slice(t, t + 1)
        _, Sn = oracle.gdn_seq(q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], beta[:, sl],
                               S.astype(np.float32), eps=0.0)
        kt = _unit(k[0, t])                                     # beta = 1 -> k~ = k^
        for h in range(q.shape[2]):
            np.testing.assert_allclose(Sn[0, h].T @ kt[h], v[0, t, h], rtol=0, atol=1e-12)
        S = Sn


def test_write_identity_general_beta():
    """General form of the same identity, derived from eq. (11):
    S_t^T k~ = (1 - ||k~||^2) (Diag(alpha) S_{t-1})^T k~ + ||k~||^2 v~."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(2, T=1, dk=7, dv=7)
    _, S1 = oracle.gdn_seq(q, k, v, alpha, beta, S0, eps=0.0)
    for h in range(q.shape[2]):
        kt = np.sqrt(beta[0, 0, h].astype(np.float64)) * _unit(k[0, 0, h])
        vt = np.sqrt(beta[0, 0, h].astype(np.float64)) * v[0, 0, h]
        X = alpha[0, 0, h][:, None].astype(np.float64) * S0[0, h]
        n2 = kt @ kt
        want = (1 - n2) * (X.T @ kt) + n2 * vt
        np.testing.assert_allclose(S1[0, h].T @ kt, want, rtol=0, atol=1e-12)


def test_update_is_one_gradient_step():
    """The delta rule is one online gradient step on 1/2 ||S^T k - v||^2 (reading notes
    sec. 2.1); with the sqrt(beta) absorption of eq. (11) the step is taken on
    1/2 ||X^T k~ - v~||^2 from X = Diag(alpha) S_{t-1}.  The gradient comes from torch
    autograd, not from the oracle's formula."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(3, T=1, dk=5, dv=5)
    _, S1 = oracle.gdn_seq(q, k, v, alpha, beta, S0, eps=0.0)
    for h in range(q.shape[2]):
        kt = torch.tensor(np.sqrt(beta[0, 0, h].astype(np.float64)) * _unit(k[0, 0, h]))
        vt = torch.tensor(np.sqrt(beta[0, 0, h].astype(np.float64)) * v[0, 0, h].astype(np.float64))
        X = torch.tensor(alpha[0, 0, h][:, None].astype(np.float64) * S0[0, h], requires_grad=True)
        loss = 0.5 * ((X.T @ kt - vt) ** 2).sum()
        (grad,) = torch.autograd.grad(loss, X)
        np.testing.assert_allclose(S1[0, h], (X - grad).detach().numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- special cases
def _textbook(q, k, v, decay, rate, S0):
    """Textbook delta-rule loop with explicit d x d transition matrices:
    S_t = (I - rate_t k^_t k^_t^T) Diag(decay_t) S_{t-1} + rate_t k^_t v_t^T,  o_t = S_t^T q^_t.
    decay_t is a dk-vector, rate_t a scalar (DeltaNet eq. (6) when decay = 1)."""
    T, dk = q.shape
    S = np.zeros((dk, v.shape[1])) if S0 is None else S0.astype(np.float64)
    o = np.zeros((T, v.shape[1]))
    I = np.eye(dk)
    for t in range(T):
        kh = _unit(k[t])
        S = (I - rate[t] * np.outer(kh, kh)) @ np.diag(decay[t]) @ S + rate[t] * np.outer(kh, v[t])
        o[t] = S.T @ _unit(q[t])
    return o, S


@pytest.mark.parametrize("mode", ["deltanet", "gdn", "kda"])
def test_special_cases_reduce_to_textbook(mode):
    """DeltaNet (alpha = 1, scalar beta), GDN (scalar alpha, scalar beta) and KDA
    (channel-wise alpha, scalar beta) are special cases of eq. (11) (reading notes sec. 1
    table; Su Jianlin's note, "Problem Description")."""
    dk = dv = 6
    alpha_scalar = mode == "gdn"
    q, k, v, alpha, beta, S0 = _gdn_inputs(4, T=9, dk=dk, dv=dv, alpha_scalar=alpha_scalar,
                                           beta_scalar=True)
    if mode == "deltanet":
        alpha = np.ones_like(alpha)
    o, sf = oracle.gdn_seq(q, k, v, alpha, beta, S0, alpha_scalar=alpha_scalar, beta_scalar=True,
                           eps=0.0)
    for h in range(q.shape[2]):
        a = alpha[0, :, h]
        decay = np.repeat(a[:, None], dk, axis=1) if alpha_scalar else a
        ot, St = _textbook(q[0, :, h], k[0, :, h], v[0, :, h], decay.astype(np.float64),
                           beta[0, :, h].astype(np.float64), S0[0, h])
        np.testing.assert_allclose(o[0, :, h], ot, rtol=0, atol=1e-12)
        np.testing.assert_allclose(sf[0, h], St, rtol=0, atol=1e-12)


def test_channelwise_beta_with_equal_entries_is_kda():
    """A channel-wise beta whose entries are equal reproduces the scalar-beta (KDA) run."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(5, T=8, beta_scalar=True)
    bvec = np.repeat(beta[..., None], q.shape[-1], axis=-1)
    o1, s1 = oracle.gdn_seq(q, k, v, alpha, beta, S0, beta_scalar=True)
    o2, s2 = oracle.gdn_seq(q, k, v, alpha, bvec, S0)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------- closed forms
def test_beta_zero_closed_form():
    """beta = 0 leaves only the decay: S_T = Diag(prod alpha) S0 and
    o_t = (Diag(prod_{s<=t} alpha_s) S0)^T q^_t (eq. (11))."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(6, T=7)
    beta = np.zeros_like(beta)
    o, sf = oracle.gdn_seq(q, k, v, alpha, beta, S0, eps=0.0)
    for h in range(q.shape[2]):
        cum = np.cumprod(alpha[0, :, h].astype(np.float64), axis=0)
        for t in range(q.shape[1]):
            want = (cum[t][:, None] * S0[0, h]).T @ _unit(q[0, t, h])
            np.testing.assert_allclose(o[0, t, h], want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(sf[0, h], cum[-1][:, None] * S0[0, h], rtol=0, atol=1e-12)


def test_single_token_closed_form():
    """T = 1, S0 = 0: S = k~ v~^T and o = (k~^T q^) v~ (eq. (11), readout of the updated state)."""
    q, k, v, alpha, beta, _ = _gdn_inputs(7, T=1)
    o, sf = oracle.gdn_seq(q, k, v, alpha, beta, None, eps=0.0)
    for h in range(q.shape[2]):
        kt = np.sqrt(beta[0, 0, h].astype(np.float64)) * _unit(k[0, 0, h])
        vt = np.sqrt(beta[0, 0, h].astype(np.float64)) * v[0, 0, h]
        np.testing.assert_allclose(sf[0, h], np.outer(kt, vt), rtol=0, atol=1e-14)
        np.testing.assert_allclose(o[0, 0, h], (kt @ _unit(q[0, 0, h])) * vt, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------- chunked form
@pytest.mark.parametrize("chunk", [1, 3, 16, 64])
@pytest.mark.parametrize("mode", ["fg2", "kda", "gdn"])
def test_sequential_equals_chunked(chunk, mode):
    """The token-by-token recurrence and the chunkwise WY/UT form (reading notes sec. 2.4)
    are two independent algorithms for the same result; T is not a multiple of the chunk."""
    a_s = mode == "gdn"
    b_s = mode in ("kda", "gdn")
    q, k, v, alpha, beta, S0 = _gdn_inputs(8, B=2, T=77, H=2, dk=8, dv=8, alpha_scalar=a_s,
                                           beta_scalar=b_s)
    o1, s1 = oracle.gdn_seq(q, k, v, alpha, beta, S0, alpha_scalar=a_s, beta_scalar=b_s)
    o2, s2 = oracle.gdn_chunked(q, k, v, alpha, beta, S0, chunk=chunk, alpha_scalar=a_s,
                                beta_scalar=b_s)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.sqrt(np.mean(o1 ** 2))
    assert np.abs(s1 - s2).max() <= 1e-12 * np.sqrt(np.mean(s1 ** 2))


def test_chunked_strong_decay_does_not_overflow():
    """Decay factors are formed only for i <= r, so tiny alpha (log-decay span of
    hundreds inside a chunk) stays finite and equals the sequential result."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(9, T=40, dk=4, dv=4)
    alpha = np.full_like(alpha, 1e-8)
    o1, s1 = oracle.gdn_seq(q, k, v, alpha, beta, S0)
    o2, s2 = oracle.gdn_chunked(q, k, v, alpha, beta, S0, chunk=16)
    assert np.all(np.isfinite(o2))
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- invariants
def test_superposition_in_state_and_values():
    """The map (S0, v) -> (o, S_T) is linear for fixed q, k, alpha, beta (eq. (11))."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(10, T=15)
    o, s = oracle.gdn_seq(q, k, v, alpha, beta, S0)
    oa, sa = oracle.gdn_seq(q, k, np.zeros_like(v), alpha, beta, S0)
    ob, sb = oracle.gdn_seq(q, k, v, alpha, beta, None)
    np.testing.assert_allclose(o, oa + ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s, sa + sb, rtol=0, atol=1e-12)


def test_scale_invariance_of_q_and_k():
    """q and k are L2-normalised, so positive rescaling changes nothing (eps = 0)."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(11, T=10)
    o, s = oracle.gdn_seq(q, k, v, alpha, beta, S0, eps=0.0)
    # powers of two keep the float32 inputs exact
    o2, s2 = oracle.gdn_seq(4.0 * q, 0.25 * k, v, alpha, beta, S0, eps=0.0)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s, s2, rtol=0, atol=1e-12)
    # other factors round the float32 inputs once (relative 2^-24)
    o3, s3 = oracle.gdn_seq(3.7 * q, 0.3 * k, v, alpha, beta, S0, eps=0.0)
    np.testing.assert_allclose(o, o3, rtol=0, atol=1e-5)


def test_time_split_resume():
    """Running T1 tokens and feeding S_final as S0 to the next T2 tokens equals one run."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(12, T=20, dk=8, dv=8)
    o, s = oracle.gdn_chunked(q, k, v, alpha, beta, S0, chunk=4)
    a = slice(0, 11)
    b = slice(11, 20)
    o1, s1 = oracle.gdn_chunked(q[:, a], k[:, a], v[:, a], alpha[:, a], beta[:, a], S0, chunk=4)
    o2, s2 = oracle.gdn_chunked(q[:, b], k[:, b], v[:, b], alpha[:, b], beta[:, b], s1, chunk=4)
    # S0 passes through float32 in the second call; compare against that rounding.
    assert np.abs(np.concatenate([o1, o2], axis=1) - o).max() < 1e-6
    assert np.abs(s2 - s).max() < 1e-6


def test_nonexpansive_transition():
    """Two runs that differ only in S0 contract step by step:
    ||S_t - S'_t||_2 <= max_i alpha_{t,i} ||S_{t-1} - S'_{t-1}||_2 because
    ||(I - k~ k~^T) Diag(alpha)||_2 <= max alpha when ||k~||^2 <= 2 (Su Jianlin's note,
    eq. (spec) with j = k; beta <= 1 gives ||k~||^2 <= 1)."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(13, T=12, dk=6, dv=6)
    S0b = S0 + _rng(14).standard_normal(S0.shape).astype(np.float32)
    Sa, Sb = S0.astype(np.float64), S0b.astype(np.float64)
    for t in range(q.shape[1]):
        sl = slice(t, t + 1)
        _, Na = oracle.gdn_seq(q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], beta[:, sl], Sa.astype(np.float32))
        _, Nb = oracle.gdn_seq(q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], beta[:, sl], Sb.astype(np.float32))
        for h in range(q.shape[2]):
            before = np.linalg.norm(Sa.astype(np.float32).astype(np.float64)[0, h]
                                    - Sb.astype(np.float32).astype(np.float64)[0, h], 2)
            after = np.linalg.norm(Na[0, h] - Nb[0, h], 2)
            assert after <= alpha[0, t, h].max() * before * (1 + 1e-12) + 1e-12
        Sa, Sb = Na, Nb


# --------------------------------------------------------------------------- transition spectrum
def _transition(k, alpha, beta):
    """One-step transition of the oracle, read off by applying it to S0 = I with v = 0."""
    dk = k.shape[-1]
    q = np.ones((1, 1, 1, dk), np.float32)
    S0 = np.eye(dk, dtype=np.float32)[None, None]
    _, S1 = oracle.gdn_seq(q, k.reshape(1, 1, 1, dk), np.zeros((1, 1, 1, dk), np.float32),
                           alpha.reshape(1, 1, 1, dk), beta.reshape(1, 1, 1, dk), S0, eps=0.0)
    return S1[0, 0]


def test_transition_is_dplr_with_secular_spectrum():
    """The oracle's transition equals Diag(alpha) + a b^T with a = -k~, b = k~ (.) alpha
    (reading notes sec. 2.4), i.e. diag(w) - kappa (a (.) kappa)^T with w = alpha, kappa = k~,
    a = alpha (secularmode README).  Its eigenvalues (numpy) are real, satisfy the secular
    equation, interlace the decay values and stay <= max alpha; its spectral norm (numpy SVD)
    is <= max alpha."""
    r = _rng(15)
    for d in (3, 5, 8):
        for _ in range(20):
            k = r.standard_normal(d).astype(np.float32)
            alpha = r.uniform(0.2, 1.0, d).astype(np.float32)
            beta = r.uniform(0.0, 1.0, d).astype(np.float32)
            M = _transition(k, alpha, beta)
            kt = np.sqrt(beta.astype(np.float64)) * _unit(k)
            a64 = alpha.astype(np.float64)
            np.testing.assert_allclose(M, spectral.dplr_matrix(a64, kt, a64), rtol=0, atol=1e-14)
            lam = np.linalg.eigvals(M)
            assert np.abs(lam.imag).max() < 1e-9
            lam = np.sort(lam.real)
            w = np.sort(a64)
            for x in lam:
                # det(M - x I) from the secular form vanishes (relative to the product scale)
                assert abs(spectral.secular_det(a64, kt, a64, x)) < 1e-9
            assert np.all(lam <= w + 1e-12)                       # lambda_i <= w_i
            assert np.all(lam[1:] >= w[:-1] - 1e-12)              # w_{i-1} <= lambda_i
            assert lam[-1] <= a64.max() + 1e-12
            assert np.linalg.norm(M, 2) <= a64.max() * (1 + 1e-12)


# --------------------------------------------------------------------------- closed-form spectra
def test_rank1_spectral_norm_golden():
    """Hand-worked values of the closed form (tests/golden/rank1_spectral_norm.txt) against
    both the oracle's closed-form function and numpy's SVD."""
    with open(os.path.join(GOLDEN, "rank1_spectral_norm.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 7
    for d, j, k, eta, want in rows:
        j = np.array([float(x) for x in j.split(",")])
        k = np.array([float(x) for x in k.split(",")])
        eta, want = float(eta), float(want)
        assert abs(spectral.rank1_spectral_norm(j, k, eta) - want) < 1e-14
        assert abs(np.linalg.norm(np.eye(int(d)) - eta * np.outer(j, k), 2) - want) < 1e-12


def test_rank1_spectral_norm_vs_svd():
    """Closed form of ||I - eta j k^T||_2 (Su Jianlin's note, eq. (spec); the unnormalised
    form in "Modifying Itself") against brute-force SVD on random tiny matrices, and the
    'iff' statement: <= 1 exactly when j = k and eta <= 2 (or eta = 0)."""
    r = _rng(16)
    for d in range(2, 9):
        for _ in range(30):
            j, k = r.standard_normal(d), r.standard_normal(d)
            eta = r.uniform(0, 3)
            want = np.linalg.norm(np.eye(d) - eta * np.outer(j, k), 2)
            assert abs(spectral.rank1_spectral_norm(j, k, eta) - want) < 1e-10 * max(1, want)
            ju, ku = _unit(j), _unit(k)
            assert spectral.rank1_spectral_norm(ju, ku, eta) > 1.0         # j != k, eta > 0
            assert spectral.rank1_spectral_norm(ku, ku, min(eta, 2.0)) <= 1.0 + 1e-12
            assert spectral.rank1_spectral_norm(ku, ku, 2.0 + eta + 1e-3) > 1.0


def test_gdn2_shrink_caps_norm():
    """Replacing j by j* = c k + lambda*(j - c k) keeps j*^T k = c and gives
    ||I - j* k^T||_2 = 1/gamma_max whenever lambda* < 1 (Su Jianlin's note, "Modifying
    Itself"); gamma_max = 1 collapses j* to c k (KDA)."""
    r = _rng(17)
    hits = 0
    for _ in range(200):
        d = r.integers(2, 8)
        k = _unit(r.standard_normal(d))
        j = k * r.uniform(0, 1, d)                 # GDN2's j = k (.) b, b in [0,1]^d: c in [0, 1]
        gmax = r.uniform(0.6, 1.0)
        c = j @ k
        assert (c - 1.0) * gmax + 1.0 / gmax >= c  # tau >= c, the note's solvability condition
        js, lam = spectral.gdn2_shrink(j, k, gmax)
        assert abs(js @ k - j @ k) < 1e-12
        n = np.linalg.norm(np.eye(d) - np.outer(js, k), 2)
        if lam < 1.0:
            hits += 1
            assert abs(n - 1.0 / gmax) < 1e-9
        else:
            assert n <= 1.0 / gmax + 1e-9
        js1, _ = spectral.gdn2_shrink(j, k, 1.0)
        np.testing.assert_allclose(js1, (j @ k) * k, atol=1e-7)  # lambda* = sqrt(rounding) ~ 1e-8
    assert hits > 8


def test_secular_equation_generic():
    """For diag(w) - kappa (a (.) kappa)^T with a >= 0 (secularmode README): the determinant
    identity against numpy det, a real spectrum interlacing w, the -1 boundary
    sum a kappa^2 / (w + 1) = 1, and the DeltaNet limit w = 1 where the moved eigenvalue is
    1 - beta (-1 at beta = 2)."""
    r = _rng(18)
    for d in (2, 4, 7):
        for _ in range(20):
            w = np.sort(r.uniform(0.05, 1.0, d))
            kap = _unit(r.standard_normal(d))
            a = r.uniform(0, 2, d)
            A = spectral.dplr_matrix(w, kap, a)
            for lam in r.uniform(-2, 2, 3):
                assert abs(spectral.secular_det(w, kap, a, lam) - np.linalg.det(A - lam * np.eye(d))) < 1e-10
            ev = np.sort(np.linalg.eigvals(A).real)
            assert np.abs(np.linalg.eigvals(A).imag).max() < 1e-9
            assert np.all(ev <= w + 1e-10) and np.all(ev[1:] >= w[:-1] - 1e-10)
            # scale the removal so the budget is exactly 1: -1 becomes an eigenvalue
            a1 = a / spectral.over_removal_budget(w, kap, a)
            ev1 = np.sort(np.linalg.eigvals(spectral.dplr_matrix(w, kap, a1)).real)
            assert abs(ev1[0] + 1.0) < 1e-9
    for beta in (0.3, 1.0, 2.0):
        kap = _unit(r.standard_normal(5))
        ev = np.sort(np.linalg.eigvals(spectral.dplr_matrix(np.ones(5), kap, beta * np.ones(5))).real)
        assert abs(ev[0] - (1 - beta)) < 1e-12 and np.allclose(ev[1:], 1.0)


# --------------------------------------------------------------------------- DeltaProduct
def _dp_inputs(seed, B=1, T=9, H=2, nh=2, d=5, s0=True):
    r = _rng(seed)
    q = r.standard_normal((B, T, H, d)).astype(np.float32)
    k = r.standard_normal((B, T, H, nh, d)).astype(np.float32)
    v = r.standard_normal((B, T, H, nh, d)).astype(np.float32)
    beta = r.uniform(0, 2, (B, T, H, nh)).astype(np.float32)
    gamma = r.uniform(0.5, 1.0, (B, T, H)).astype(np.float32)
    S0 = r.standard_normal((B, H, d, d)).astype(np.float32) if s0 else None
    return q, k, v, gamma, beta, S0


def test_deltaproduct_second_step_off_is_gated_deltanet():
    """beta_{t,2} = 0 leaves one Householder step per token: gated DeltaNet (GDN with
    scalar gate gamma and scalar beta)."""
    q, k, v, gamma, beta, S0 = _dp_inputs(19)
    beta[..., 1] = 0.0
    o, s = oracle.deltaproduct_seq(q, k, v, gamma, beta, S0)
    o2, s2 = oracle.gdn_seq(q, k[:, :, :, 0], v[:, :, :, 0], gamma, beta[..., 0], S0,
                            alpha_scalar=True, beta_scalar=True)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s, s2, rtol=0, atol=1e-12)


def test_deltaproduct_without_gate_is_interleaved_deltanet():
    """gamma = 1: DeltaProduct_n_h is DeltaNet (eq. (6)) run over the n_h T sub-steps,
    read at the last sub-step of every token (DeltaProduct summary, "Approach")."""
    q, k, v, gamma, beta, S0 = _dp_inputs(20, nh=3)
    gamma = np.ones_like(gamma)
    o, s = oracle.deltaproduct_seq(q, k, v, gamma, beta, S0, eps=0.0)
    B, T, H, nh, d = k.shape
    for h in range(H):
        ks = k[0, :, h].reshape(T * nh, d)
        vs = v[0, :, h].reshape(T * nh, d)
        bs = beta[0, :, h].reshape(T * nh).astype(np.float64)
        qs = np.repeat(q[0, :, h], nh, axis=0)
        ot, St = _textbook(qs, ks, vs, np.ones((T * nh, d)), bs, S0[0, h])
        np.testing.assert_allclose(o[0, :, h], ot[nh - 1::nh], rtol=0, atol=1e-11)
        np.testing.assert_allclose(s[0, h], St, rtol=0, atol=1e-11)


def test_deltaproduct_beta_two_is_a_reflection():
    """beta = 2 with a unit key gives the Householder reflection I - 2 k k^T: orthogonal,
    with eigenvalue -1 (DeltaProduct summary, eigenvalues in [-1, 1]; secularmode README,
    'at beta = 2 the minimum eigenvalue is -1')."""
    d = 6
    r = _rng(21)
    k = r.standard_normal((1, 1, 1, 1, d)).astype(np.float32)
    S0 = np.eye(d, dtype=np.float32)[None, None]
    _, M = oracle.deltaproduct_seq(np.ones((1, 1, 1, d), np.float32), k,
                                   np.zeros((1, 1, 1, 1, d), np.float32),
                                   np.ones((1, 1, 1), np.float32), np.full((1, 1, 1, 1), 2.0, np.float32),
                                   S0, eps=0.0)
    M = M[0, 0]
    np.testing.assert_allclose(M @ M.T, np.eye(d), atol=1e-12)
    ev = np.sort(np.linalg.eigvals(M).real)
    assert abs(ev[0] + 1) < 1e-12 and np.allclose(ev[1:], 1.0)


def test_deltaproduct_as_interleaved_gdn_sequence():
    """DeltaProduct equals the FG^2-GDN recurrence over the interleaved sub-step sequence
    with scalar beta, decay gamma_t on the first sub-step and 1 on the others, read at the
    last sub-step of each token (the mapping the chunked kernels use)."""
    q, k, v, gamma, beta, S0 = _dp_inputs(22, T=11, nh=2, d=6)
    o, s = oracle.deltaproduct_seq(q, k, v, gamma, beta, S0)
    B, T, H, nh, d = k.shape
    ks = np.transpose(k, (0, 1, 3, 2, 4)).reshape(B, T * nh, H, d)
    vs = np.transpose(v, (0, 1, 3, 2, 4)).reshape(B, T * nh, H, d)
    bs = np.transpose(beta, (0, 1, 3, 2)).reshape(B, T * nh, H)
    al = np.ones((B, T, nh, H), np.float32)
    al[:, :, 0, :] = gamma
    al = al.reshape(B, T * nh, H)
    qs = np.repeat(q, nh, axis=1)
    for chunk in (4, 7, 64):
        o2, s2 = oracle.gdn_chunked(qs, ks, vs, al, bs, S0, chunk=chunk, alpha_scalar=True,
                                    beta_scalar=True)
        np.testing.assert_allclose(o2[:, nh - 1::nh], o, rtol=0, atol=1e-11)
        np.testing.assert_allclose(s2, s, rtol=0, atol=1e-11)


# --------------------------------------------------------------------------- FG^2-GDN+
def _plus_inputs(seed, T=10, dk=6, dv=9):
    q, k, v, alpha, beta_k, S0 = _gdn_inputs(seed, T=T, dk=dk, dv=dv)
    beta_v = _rng(seed + 1000).uniform(0.0, 1.0, (1, T, 2, dv)).astype(np.float32)
    return q, k, v, alpha, beta_k, beta_v, S0


def test_plus_with_equal_rates_is_fg2():
    """FG^2-GDN+ with beta^v = beta^k is FG^2-GDN (FG^2-GDN summary, "FG2-GDN+ Variant";
    reading notes sec. 2.3 eq. (13) against eq. (11))."""
    q, k, v, alpha, beta, S0 = _gdn_inputs(30, T=11)
    o1, s1 = oracle.gdn_seq(q, k, v, alpha, beta, S0)
    o2, s2 = oracle.gdn_seq(q, k, v, alpha, beta, S0, beta_v=beta.copy())
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-14)


def test_plus_write_identity_and_gradient_step():
    """Eq. (13): S_t = X + k^ (v~ - X^T k^)^T with k^ = sqrt(beta^k) (.) k and
    v~ = sqrt(beta^v) (.) v, i.e. one gradient step on 1/2 ||X^T k^ - v~||^2 (autograd);
    with ||k^|| = 1 the write is exact: S_t^T k^ = v~."""
    q, k, v, alpha, beta_k, beta_v, S0 = _plus_inputs(31, T=1, dk=5, dv=7)
    _, S1 = oracle.gdn_seq(q, k, v, alpha, beta_k, S0, beta_v=beta_v, eps=0.0)
    for h in range(2):
        kh = torch.tensor(np.sqrt(beta_k[0, 0, h].astype(np.float64)) * _unit(k[0, 0, h]))
        vt = torch.tensor(np.sqrt(beta_v[0, 0, h].astype(np.float64)) * v[0, 0, h].astype(np.float64))
        X = torch.tensor(alpha[0, 0, h][:, None].astype(np.float64) * S0[0, h], requires_grad=True)
        (grad,) = torch.autograd.grad(0.5 * ((X.T @ kh - vt) ** 2).sum(), X)
        np.testing.assert_allclose(S1[0, h], (X - grad).detach().numpy(), rtol=0, atol=1e-12)
    ones = np.ones_like(beta_k)
    _, S1 = oracle.gdn_seq(q, k, v, alpha, ones, S0, beta_v=beta_v, eps=0.0)
    for h in range(2):
        vt = np.sqrt(beta_v[0, 0, h].astype(np.float64)) * v[0, 0, h]
        np.testing.assert_allclose(S1[0, h].T @ _unit(k[0, 0, h]), vt, rtol=0, atol=1e-12)


def test_plus_value_rate_scales_linearly():
    """With S0 = 0 the state and output are linear in v~ = sqrt(beta^v) (.) v, so
    multiplying beta^v by c^2 multiplies them by c (eq. (13))."""
    q, k, v, alpha, beta_k, beta_v, _ = _plus_inputs(32, T=12)
    o1, s1 = oracle.gdn_seq(q, k, v, alpha, beta_k, None, beta_v=beta_v)
    o2, s2 = oracle.gdn_seq(q, k, v, alpha, beta_k, None, beta_v=4.0 * beta_v)
    np.testing.assert_allclose(o2, 2.0 * o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, 2.0 * s1, rtol=0, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 4, 16])
def test_plus_sequential_equals_chunked(chunk):
    """FG^2-GDN+ with dk != dv: token-by-token and chunkwise forms agree."""
    q, k, v, alpha, beta_k, beta_v, S0 = _plus_inputs(33, T=37, dk=6, dv=9)
    o1, s1 = oracle.gdn_seq(q, k, v, alpha, beta_k, S0, beta_v=beta_v)
    o2, s2 = oracle.gdn_chunked(q, k, v, alpha, beta_k, S0, chunk=chunk, beta_v=beta_v)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.sqrt(np.mean(o1 ** 2))
    assert np.abs(s1 - s2).max() <= 1e-12 * np.sqrt(np.mean(s1 ** 2))

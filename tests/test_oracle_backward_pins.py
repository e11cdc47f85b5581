"""Pins of the oracle's gradients (oracle.backward) to facts that do not come from
autograd: central finite differences of the independent C forward (oracle.gdn_seq),
and a closed form for one token from a zero state."""
import numpy as np
import pytest

import oracle
from oracle.backward import gdn_grads

H_FD = 2.0 ** -10      # inputs are float32 of magnitude < 2, so x +- H_FD is exact


def _inputs(seed, T=5, dk=3, dv=3, alpha_scalar=False, beta_scalar=False, plus=False):
    r = np.random.default_rng(seed)
    f = np.float32
    x = dict(q=r.standard_normal((1, T, 2, dk)).astype(f), k=r.standard_normal((1, T, 2, dk)).astype(f),
             v=r.uniform(-1, 1, (1, T, 2, dv)).astype(f),
             alpha=r.uniform(0.5, 0.95, (1, T, 2) if alpha_scalar else (1, T, 2, dk)).astype(f),
             beta=r.uniform(0.2, 0.9, (1, T, 2) if beta_scalar else (1, T, 2, dk)).astype(f),
             S0=r.uniform(-1, 1, (1, 2, dk, dv)).astype(f))
    if plus:
        x["beta_v"] = r.uniform(0.2, 0.9, (1, T, 2) if beta_scalar else (1, T, 2, dv)).astype(f)
    dO = r.standard_normal((1, T, 2, dv)).astype(f)
    dS = r.standard_normal((1, 2, dk, dv)).astype(f)
    return x, dO, dS


def _loss(x, dO, dS, kw):
    o, s = oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                          beta_v=x.get("beta_v"), **kw)
    return float(np.sum(o * dO) + np.sum(s * dS))


@pytest.mark.parametrize("mode", ["fg2", "kda", "gdn", "plus", "plus_rect"])
def test_gradients_match_finite_differences_of_c_forward(mode):
    kw = dict(alpha_scalar=mode == "gdn", beta_scalar=mode in ("kda", "gdn"))
    plus = mode.startswith("plus")
    x, dO, dS = _inputs(40 + len(mode), dv=4 if mode == "plus_rect" else 3, plus=plus, **kw)
    g = gdn_grads(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], dO, dS,
                  beta_v=x.get("beta_v"), **kw)
    for name in ["q", "k", "v", "alpha", "beta", "S0"] + (["beta_v"] if plus else []):
        fd = np.zeros(x[name].shape)
        for idx in np.ndindex(x[name].shape):
            xp = {n: a.copy() for n, a in x.items()}
            xm = {n: a.copy() for n, a in x.items()}
            xp[name][idx] += np.float32(H_FD)
            xm[name][idx] -= np.float32(H_FD)
            step = float(xp[name][idx]) - float(xm[name][idx])
            fd[idx] = (_loss(xp, dO, dS, kw) - _loss(xm, dO, dS, kw)) / step
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(g[name], fd, rtol=0, atol=2e-5 * scale, err_msg=name)


def test_one_token_zero_state_closed_form():
    """T = 1, S0 = 0: o = v~ (k~ . q^), so dL/dv = sqrt(beta) (.) dO (k~ . q^) and
    dL/dq = (I - q^ q^^T) k~ (dO . v~) / ||q|| (eps = 0)."""
    x, dO, _ = _inputs(50, T=1, dk=4, dv=4)
    g = gdn_grads(x["q"], x["k"], x["v"], x["alpha"], x["beta"], None, dO, eps=0.0)
    for h in range(2):
        q, k, v, b = (x[n][0, 0, h].astype(np.float64) for n in ("q", "k", "v", "beta"))
        d = dO[0, 0, h].astype(np.float64)
        qh = q / np.linalg.norm(q)
        kt = np.sqrt(b) * k / np.linalg.norm(k)
        vt = np.sqrt(b) * v
        np.testing.assert_allclose(g["v"][0, 0, h], np.sqrt(b) * d * (kt @ qh), rtol=1e-12, atol=1e-14)
        dq = (np.eye(4) - np.outer(qh, qh)) @ kt * (d @ vt) / np.linalg.norm(q)
        np.testing.assert_allclose(g["q"][0, 0, h], dq, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(g["o"][0, 0, h], vt * (kt @ qh), rtol=1e-12, atol=1e-14)


def test_checkpointed_segments_change_nothing():
    """Long sequences are differentiated segment by segment; the result equals the
    unsegmented one (the segments only bound memory)."""
    import torch
    from oracle.backward import gdn_forward_torch
    x, _, _ = _inputs(60, T=37, dk=4, dv=4)
    t = {n: torch.from_numpy(a.astype(np.float64)).requires_grad_(True) for n, a in x.items()}
    outs = []
    for seg in (5, 1000):
        o, s = gdn_forward_torch(t["q"], t["k"], t["v"], t["alpha"], t["beta"], t["S0"], segment=seg)
        gs = torch.autograd.grad(o.sum() + (s * s).sum(), list(t.values()))
        outs.append([gg.numpy() for gg in gs] + [o.detach().numpy()])
    for a, b in zip(*outs):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)

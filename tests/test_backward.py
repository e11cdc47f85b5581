"""GPU parity of the chunkwise backward (gdn_chunk_bwd) against the oracle's fp64
autograd gradients, for every input: gate modes, FG^2-GDN+ rates, ragged tails,
T < chunk, both dtypes and chunk sizes, dk != dv, and sampled heads of a long
sequence."""
import numpy as np
import pytest

from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
from oracle.backward import gdn_grads
from _util import parity, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

# Gradients are computed in float32 from inputs the oracle reads exactly, so both
# dtypes meet the float32 bound up to the conditioning of (I + A)^{-1} and of the
# normalisations; 1e-3 of the RMS leaves room for that amplification.
TOL_GRAD = 1e-3


def run(cfg, x, dO, dS, chunk):
    from gated_delta_rule_fg_b200 import ops
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    g = ops.chunk_bwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt), to_dev(x["alpha"]),
                      to_dev(x["beta"]), to_dev(x["S0"]), to_dev(dO, dt), to_dev(dS),
                      beta_v=to_dev(x.get("beta_v")), chunk=chunk, alpha_scalar=cfg.alpha_scalar,
                      beta_scalar=cfg.beta_scalar)
    torch.cuda.synchronize()
    return {n: t.cpu().numpy() for n, t in g.items()}


def cotangents(cfg, x, seed):
    r = np.random.default_rng(seed)
    B, T, H, _ = x["q"].shape
    dO = r.standard_normal((B, T, H, cfg.dv)).astype(np.float32)
    if cfg.dtype == "bf16":
        from gated_delta_rule_fg_b200.inputs import round_bf16
        dO = round_bf16(dO)
    dS = r.standard_normal((B, H, cfg.dk, cfg.dv)).astype(np.float32)
    return dO, dS


def compare(cfg, x, got, ref, pairs=None):
    names = ["q", "k", "v", "alpha", "beta", "S0"] + (["beta_v"] if "beta_v" in x else [])
    for n in names:
        a, b = got[n], ref[n]
        if pairs is not None:
            if n == "S0":
                a = np.stack([a[bb, hh] for bb, hh in pairs])
                b = np.stack([b[bb, hh] for bb, hh in pairs])
            else:
                a = np.stack([a[bb, :, hh] for bb, hh in pairs])
                b = np.stack([b[bb, :, hh] for bb, hh in pairs])
        try:
            parity(a, b, TOL_GRAD)
        except AssertionError as e:
            raise AssertionError(f"d{n}: {e}") from None


CASES = [("fg2", "f32", 64, 64, 16, 40), ("fg2", "bf16", 128, 128, 32, 100),
         ("kda", "f32", 64, 128, 32, 70), ("gdn", "bf16", 64, 64, 16, 33),
         ("deltanet", "f32", 32, 32, 16, 20), ("plus", "f32", 64, 32, 32, 45),
         ("plus", "bf16", 128, 128, 32, 64), ("plus_scalar", "f32", 64, 64, 16, 7),
         ("fg2", "f32", 128, 128, 32, 1)]


@pytest.mark.parametrize("mode,dtype,dk,dv,chunk,T", CASES)
def test_backward_small(mode, dtype, dk, dv, chunk, T):
    cfg = GdnConfig("bwd", B=2, H=2, T=T, dk=dk, dv=dv, chunk=chunk, dtype=dtype,
                    alpha_scalar=mode == "gdn", beta_scalar=mode in ("kda", "gdn", "deltanet", "plus_scalar"),
                    plus=mode.startswith("plus"), s0_std=0.1, seed=4000 + T + dk)
    x = make_inputs(cfg)
    if mode == "deltanet":
        x["alpha"] = np.ones_like(x["alpha"])
    dO, dS = cotangents(cfg, x, 4100 + T)
    ref = gdn_grads(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], dO, dS,
                    beta_v=x.get("beta_v"), alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar)
    compare(cfg, x, run(cfg, x, dO, dS, chunk), ref)


def test_backward_chunk_size_invariance_and_zero_state():
    """Chunks 16 and 32 agree (the result does not depend on the backward's chunk), with
    S0 = None and dS_final = None."""
    cfg = GdnConfig("bwd_inv", B=1, H=3, T=90, dk=64, dv=64, chunk=16, dtype="f32", seed=4200)
    x = make_inputs(cfg)
    dO, _ = cotangents(cfg, x, 4201)
    a = run(cfg, x, dO, None, 16)
    b = run(cfg, x, dO, None, 32)
    ref = gdn_grads(x["q"], x["k"], x["v"], x["alpha"], x["beta"], None, dO, None)
    compare(cfg, x, a, ref)
    for n in a:
        parity(a[n], b[n], TOL_GRAD)


def test_backward_long_sequence_sampled_heads():
    """4096 tokens x 16 heads at d = 128 (the training configuration's shape per
    sequence); two heads checked against the oracle."""
    cfg = GdnConfig("bwd_long", B=1, H=16, T=4096, dk=128, dv=128, chunk=32, dtype="bf16",
                    alpha_scale=0.02, s0_std=0.01, seed=4300)
    x = make_inputs(cfg)
    dO, dS = cotangents(cfg, x, 4301)
    pairs = [(0, 0), (0, 15)]
    ref = gdn_grads(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], dO, dS, pairs=pairs)
    compare(cfg, x, run(cfg, x, dO, dS, 32), ref, pairs=pairs)

"""GPU parity of the single-token recurrent step (gdn_recurrent_step) against the
fp64 oracle: one step from a random state, every gate mode, FG^2-GDN+ rates, in-place
updates, and a prefill (gdn_chunk_fwd) continued by decode steps, which must match the
oracle run over the whole sequence."""
import numpy as np
import pytest

import oracle
from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
from _util import TOL_BF16, TOL_F32, parity, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _ops():
    from gated_delta_rule_fg_b200 import ops
    return ops


def _tok(a, t):
    """Token t of a [B,T,H,...] array (or None)."""
    return None if a is None else np.ascontiguousarray(a[:, t])


def step_gpu(cfg, x, t, S, in_place=False):
    ops = _ops()
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out, S_out = ops.recurrent_step(to_dev(_tok(x["q"], t), dt), to_dev(_tok(x["k"], t), dt),
                                    to_dev(_tok(x["v"], t), dt), to_dev(_tok(x["alpha"], t)),
                                    to_dev(_tok(x["beta"], t)), S,
                                    beta_v=to_dev(_tok(x.get("beta_v"), t)),
                                    alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar,
                                    in_place=in_place)
    return out, S_out


def oracle_run(cfg, x, S0):
    return oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0, beta_v=x.get("beta_v"),
                          alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar)


MODES = ["fg2", "kda", "gdn", "deltanet", "plus", "plus_scalar"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (32, 128), (128, 32)])
def test_single_step(dtype, mode, dk, dv):
    scalar_b = mode in ("kda", "gdn", "deltanet", "plus_scalar")
    if dk != dv and not (scalar_b or mode.startswith("plus")):
        pytest.skip("channel-wise beta on v needs dk == dv")
    cfg = GdnConfig("dec", B=3, H=5, T=1, dk=dk, dv=dv, chunk=16, dtype=dtype,
                    alpha_scalar=mode == "gdn", beta_scalar=scalar_b, plus=mode.startswith("plus"),
                    s0_std=0.3, seed=dk * 7 + dv + len(mode))
    x = make_inputs(cfg)
    if mode == "deltanet":
        x["alpha"] = np.ones_like(x["alpha"])
    out, S_out = step_gpu(cfg, x, 0, to_dev(x["S0"]))
    torch.cuda.synchronize()
    ro, rs = oracle_run(cfg, x, x["S0"])
    parity(out.float().cpu().numpy(), ro[:, 0], TOL_F32, out_bf16=dtype == "bf16")
    parity(S_out.cpu().numpy(), rs, TOL_F32)


def test_zero_state_and_empty_batch():
    cfg = GdnConfig("dec0", B=2, H=3, T=1, dk=128, dv=128, chunk=16, seed=5)
    x = make_inputs(cfg)
    out, S_out = step_gpu(cfg, x, 0, None)
    torch.cuda.synchronize()
    ro, rs = oracle_run(cfg, x, None)
    parity(out.float().cpu().numpy(), ro[:, 0], TOL_F32, out_bf16=True)
    parity(S_out.cpu().numpy(), rs, TOL_F32)
    ops = _ops()
    e = torch.empty((0, 3, 128), dtype=torch.bfloat16, device="cuda")
    a = torch.empty((0, 3, 128), dtype=torch.float32, device="cuda")
    o, s = ops.recurrent_step(e, e, e, a, a, None)
    assert o.shape == (0, 3, 128) and s.shape == (0, 3, 128, 128)


@pytest.mark.parametrize("dtype,plus", [("bf16", False), ("bf16", True), ("f32", False)])
def test_prefill_then_decode_in_place(dtype, plus):
    """Prefill T0 tokens with the chunked forward, then decode n more tokens in place;
    outputs and the final state match the oracle over the whole T0 + n tokens."""
    T0, n = 150, 6
    dk = dv = 128 if dtype == "bf16" else 64
    cfg = GdnConfig("pd", B=2, H=3, T=T0 + n, dk=dk, dv=dv, chunk=64 if dtype == "bf16" else 32,
                    dtype=dtype, plus=plus, s0_std=0.05, seed=77 + int(plus))
    x = make_inputs(cfg)
    ops = _ops()
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    pre = {key: (None if val is None else np.ascontiguousarray(val[:, :T0])) for key, val in x.items()}
    args = (to_dev(pre["q"], dt), to_dev(pre["k"], dt), to_dev(pre["v"], dt), to_dev(pre["alpha"]),
            to_dev(pre["beta"]))
    if plus:
        o_pre, S = ops.plus_chunk_fwd(*args, to_dev(pre["beta_v"]), to_dev(x["S0"]), chunk=cfg.chunk)
    else:
        o_pre, S = ops.chunk_fwd(*args, to_dev(x["S0"]), chunk=cfg.chunk)
    outs = []
    for t in range(T0, T0 + n):
        o, S2 = step_gpu(cfg, x, t, S, in_place=True)
        assert S2.data_ptr() == S.data_ptr()
        outs.append(o.float().cpu().numpy())
    torch.cuda.synchronize()
    ro, rs = oracle_run(cfg, x, x["S0"])
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    parity(o_pre.float().cpu().numpy(), ro[:, :T0], tol, out_bf16=dtype == "bf16")
    parity(np.stack(outs, axis=1), ro[:, T0:], tol, out_bf16=dtype == "bf16")
    parity(S.cpu().numpy(), rs, tol)

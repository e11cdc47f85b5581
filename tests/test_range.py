"""The fp16 operand range of the tensor-core path (bf16 inputs, chunk 64, d = 128).

The operator of eq. (11) accepts any bf16 v and any float32 S0, but the tensor-core path
rounds v~, b, PU' and the state copy it multiplies with to fp16 (largest finite value 65504).
Inputs that push one of them past that range must be reported as GDN_ERR_RANGE through the
workspace status word; inputs inside it must give GDN_OK and match the oracle."""
import numpy as np
import pytest

import oracle
from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs, round_bf16
from _util import TOL_BF16, parity, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _call(x, cfg):
    from gated_delta_rule_fg_b200 import ops
    dt = torch.bfloat16
    nws = ops.chunk_fwd_workspace_size(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.chunk, ops.GDN_BF16, 0)
    ws = ops.alloc_workspace(nws, "cuda")
    o, s = ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt), to_dev(x["alpha"]),
                         to_dev(x["beta"]), to_dev(x["S0"]), chunk=cfg.chunk, workspace=ws)
    st = ops.workspace_status(ws)
    return st, o.float().cpu().numpy(), s.cpu().numpy()


def _cfg(seed, s0=0.0):
    return GdnConfig("range", B=1, H=2, T=200, dk=128, dv=128, chunk=64, dtype="bf16", s0_std=s0, seed=seed)


def test_range_flag_large_initial_state():
    """S0 entries near 1e5 do not fit the fp16 state copy: GDN_ERR_RANGE."""
    from gated_delta_rule_fg_b200 import ops
    cfg = _cfg(501, s0=0.01)
    x = make_inputs(cfg)
    x["S0"] = (x["S0"] * 1e7).astype(np.float32)           # std 1e5
    st, _, _ = _call(x, cfg)
    assert st == ops.GDN_ERR_RANGE


def test_range_flag_large_values():
    """v near 1e5 (a legal bf16 value) does not fit the fp16 value operand: GDN_ERR_RANGE."""
    from gated_delta_rule_fg_b200 import ops
    cfg = _cfg(502)
    x = make_inputs(cfg)
    x["v"] = round_bf16(x["v"] * 1e5)
    st, _, _ = _call(x, cfg)
    assert st == ops.GDN_ERR_RANGE


def test_range_moderate_values_are_valid():
    """v near 3e3 stays inside the fp16 range everywhere: GDN_OK, and the result matches the
    oracle (so the check does not fire on valid inputs)."""
    from gated_delta_rule_fg_b200 import ops
    cfg = _cfg(503, s0=0.01)
    x = make_inputs(cfg)
    x["v"] = round_bf16(x["v"] * 3e3)
    x["S0"] = (x["S0"] * 3e3).astype(np.float32)
    st, o, s = _call(x, cfg)
    assert st == ops.GDN_OK
    ro, rs = oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    parity(o, ro, TOL_BF16, out_bf16=True)
    parity(s, rs, TOL_BF16)

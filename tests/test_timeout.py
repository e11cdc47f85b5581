"""Failure detection on the device: a bounded wait that runs out.

Every mbarrier wait of the tensor-core scan is bounded; one that runs out records
GDN_ERR_TIMEOUT in the workspace status word and its role unwinds (stops, lets the copies it
issued land, releases its tensor memory at the CTA's end).  The test knob
GDN_TEST_SCAN_SKIP_CHUNK (environment, read per call) makes the scan's producer leave one chunk
unloaded and shortens the bound to 1 ms, so the roles waiting for that chunk run out.  Nothing
faults: the call returns, the status says TIMEOUT, and the next call on the same device (which
needs the tensor memory the timed-out CTAs held) is correct again.

bf16 inputs at d = 128, chunk 64 (the tensor-core path), B1 H2 T2048 (32 chunks, one range)."""
import os

import numpy as np
import pytest

import oracle
from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
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


def test_scan_wait_runs_out_and_unwinds():
    from gated_delta_rule_fg_b200 import ops
    cfg = GdnConfig("timeout", B=1, H=2, T=2048, dk=128, dv=128, chunk=64, dtype="bf16", s0_std=0.01, seed=601)
    x = make_inputs(cfg)
    os.environ["GDN_TEST_SCAN_SKIP_CHUNK"] = "5"
    try:
        st, _, _ = _call(x, cfg)
    finally:
        del os.environ["GDN_TEST_SCAN_SKIP_CHUNK"]
    assert st == ops.GDN_ERR_TIMEOUT
    torch.cuda.synchronize()                     # the context is still usable
    st, o, s = _call(x, cfg)
    assert st == ops.GDN_OK
    ro, rs = oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    parity(o, ro, TOL_BF16, out_bf16=True)
    parity(s, rs, TOL_BF16)

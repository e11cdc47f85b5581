"""The bounds-checking build (-DGDN_DEBUG_BOUNDS, libgdn_b200_bounds.so) on the GPU: every
kernel checks the global-memory indices it forms against the extents of its buffers and records
GDN_ERR_BOUNDS instead of faulting.  On valid calls nothing may fire and the results must be the
normal build's bit for bit.  Run in a child process, since the library is chosen when the
binding is imported (environment GDN_DEBUG_BOUNDS=1)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from gated_delta_rule_fg_b200 import ops
from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
res = {"lib": ops.LIB_PATH, "cases": []}
cases = [GdnConfig("tc", B=1, H=2, T=64 * 70 + 9, dk=128, dv=128, chunk=64, s0_std=0.05, seed=71),
         GdnConfig("simt", B=2, H=2, T=300, dk=64, dv=64, chunk=32, dtype="f32", s0_std=0.05, seed=72)]
for cfg in cases:
    x = make_inputs(cfg)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    d = lambda a, t=None: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(t) if t is not None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    nws = ops.chunk_fwd_workspace_size(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.chunk,
                                       ops.GDN_BF16 if cfg.dtype == "bf16" else ops.GDN_F32, 0)
    ws = ops.alloc_workspace(nws, "cuda")
    o, s = ops.chunk_fwd(d(x["q"], dt), d(x["k"], dt), d(x["v"], dt), d(x["alpha"]), d(x["beta"]), d(x["S0"]),
                         chunk=cfg.chunk, workspace=ws)
    st = ops.workspace_status(ws)
    np.save(f"{sys.argv[2]}_{cfg.name}_o.npy", o.float().cpu().numpy())
    np.save(f"{sys.argv[2]}_{cfg.name}_s.npy", s.cpu().numpy())
    res["cases"].append({"name": cfg.name, "status": st})
print(json.dumps(res))
"""


def _run(tmp_path, bounds):
    env = dict(os.environ)
    env.pop("GDN_DEBUG_BOUNDS", None)
    if bounds:
        env["GDN_DEBUG_BOUNDS"] = "1"
    tag = str(tmp_path / ("bounds" if bounds else "normal"))
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT, tag], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1]), tag


def test_bounds_build_is_silent_and_bit_identical(tmp_path):
    import numpy as np
    from gated_delta_rule_fg_b200 import ops
    rb, tb = _run(tmp_path, True)
    rn, tn = _run(tmp_path, False)
    assert rb["lib"].endswith("libgdn_b200_bounds.so") and rn["lib"].endswith("libgdn_b200.so")
    for cb, cn in zip(rb["cases"], rn["cases"]):
        assert cb["status"] == ops.GDN_OK and cn["status"] == ops.GDN_OK, (cb, cn)
        for part in ("o", "s"):
            a = np.load(f"{tb}_{cb['name']}_{part}.npy")
            b = np.load(f"{tn}_{cn['name']}_{part}.npy")
            assert np.array_equal(a, b), (cb["name"], part)


CHILD_FIRE = r"""
import json, os, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from gated_delta_rule_fg_b200 import ops
from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
cfg = GdnConfig("fire", B=1, H=2, T=64 * 70 + 9, dk=128, dv=128, chunk=64, s0_std=0.05, seed=73)
x = make_inputs(cfg)
dt = torch.bfloat16
d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
args = (d(x["q"]).to(dt), d(x["k"]).to(dt), d(x["v"]).to(dt), d(x["alpha"]), d(x["beta"]), d(x["S0"]))
nws = ops.chunk_fwd_workspace_size(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.chunk, ops.GDN_BF16, 0)
ws = ops.alloc_workspace(nws, "cuda")
os.environ["GDN_TEST_BOUNDS_NC_OFF"] = "1"
ops.chunk_fwd(*args, chunk=64, workspace=ws)
fired = ops.workspace_status(ws)
del os.environ["GDN_TEST_BOUNDS_NC_OFF"]
o, s = ops.chunk_fwd(*args, chunk=64, workspace=ws)
after = ops.workspace_status(ws)
np.save(sys.argv[2] + "_o.npy", o.float().cpu().numpy())
print(json.dumps({"lib": ops.LIB_PATH, "fired": fired, "after": after}))
"""


def test_bounds_check_fires_and_skips(tmp_path):
    """With the bounds-checking build's test knob the kernels are told one chunk fewer than their
    grids cover: the checks on the last chunk's CTAs fire, the call reports GDN_ERR_BOUNDS without
    a fault, and the next call on the same context matches the oracle."""
    import numpy as np
    from gated_delta_rule_fg_b200 import ops
    env = dict(os.environ)
    env["GDN_DEBUG_BOUNDS"] = "1"
    env.pop("GDN_TEST_BOUNDS_NC_OFF", None)
    tag = str(tmp_path / "fire")
    out = subprocess.run([sys.executable, "-c", CHILD_FIRE, ROOT, tag], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    r = json.loads(out.stdout.strip().splitlines()[-1])
    assert r["lib"].endswith("libgdn_b200_bounds.so")
    assert r["fired"] == ops.GDN_ERR_BOUNDS and r["after"] == ops.GDN_OK
    import oracle
    from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
    from _util import TOL_BF16, parity
    cfg = GdnConfig("fire", B=1, H=2, T=64 * 70 + 9, dk=128, dv=128, chunk=64, s0_std=0.05, seed=73)
    x = make_inputs(cfg)
    ro, _ = oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    parity(np.load(tag + "_o.npy"), ro, TOL_BF16, out_bf16=True)

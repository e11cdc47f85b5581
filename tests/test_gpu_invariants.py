"""GPU-side invariants and edge cases of the library (through the C ABI):
chunk-size invariance, time-split resume, superposition, scale invariance, the
beta = 0 and T = 1 closed forms, empty inputs, NULL S0 / S_final, and the
device status word."""
import numpy as np
import pytest

from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
from _util import TOL_BF16, TOL_F32, parity, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _ops():
    from gated_delta_rule_fg_b200 import ops
    return ops


_FROM_X = object()


def _run(x, dtype, chunk, S0=_FROM_X, **kw):
    ops = _ops()
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    s0 = x["S0"] if S0 is _FROM_X else S0
    o, s = ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                         to_dev(x["alpha"]), to_dev(x["beta"]), to_dev(s0), chunk=chunk, **kw)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), s.cpu().numpy()


def _inputs(dtype="bf16", T=300, seed=3, s0=0.05, dk=128):
    cfg = GdnConfig("inv", B=1, H=4, T=T, dk=dk, dv=dk, chunk=64, dtype=dtype, s0_std=s0, seed=seed)
    return cfg, make_inputs(cfg)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_chunk_size_invariance(dtype):
    cfg, x = _inputs(dtype, dk=64)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    o64, s64 = _run(x, dtype, 64)
    for c in (16, 32):
        o, s = _run(x, dtype, c)
        parity(o, o64, 2 * tol, out_bf16=dtype == "bf16")
        parity(s, s64, 2 * tol)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_time_split_resume(dtype):
    cfg, x = _inputs(dtype)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    o, s = _run(x, dtype, 64)
    a = {k: (v[:, :137] if k != "S0" else v) for k, v in x.items()}
    b = {k: (v[:, 137:] if k != "S0" else v) for k, v in x.items()}
    o1, s1 = _run(a, dtype, 64)
    o2, s2 = _run(b, dtype, 64, S0=s1)
    parity(np.concatenate([o1, o2], axis=1), o, 2 * tol, out_bf16=dtype == "bf16")
    parity(s2, s, 2 * tol)


def test_superposition_fp32():
    """The output is linear in (S0, v) for fixed q, k, alpha, beta."""
    cfg, x = _inputs("f32")
    o, s = _run(x, "f32", 64)
    xa = dict(x, v=np.zeros_like(x["v"]))
    oa, sa = _run(xa, "f32", 64)
    ob, sb = _run(x, "f32", 64, S0=None)
    parity(oa + ob, o, 1e-5)
    parity(sa + sb, s, 1e-5)


def test_scale_invariance_fp32():
    cfg, x = _inputs("f32")
    o, s = _run(x, "f32", 64)
    o2, s2 = _run(dict(x, q=4.0 * x["q"], k=0.25 * x["k"]), "f32", 64)
    parity(o2, o, 1e-5)
    parity(s2, s, 1e-5)


def test_beta_zero_closed_form_fp32():
    cfg, x = _inputs("f32", T=70)
    x["beta"] = np.zeros_like(x["beta"])
    o, s = _run(x, "f32", 64)
    cum = np.cumprod(x["alpha"].astype(np.float64), axis=1)       # [B,T,H,dk]
    qn = x["q"] / np.sqrt((x["q"].astype(np.float64) ** 2).sum(-1, keepdims=True) + 1e-6)
    want = np.einsum("bthi,bhij,bthi->bthj", cum, x["S0"].astype(np.float64), qn)
    parity(o, want, TOL_F32)
    parity(s, cum[:, -1, :, :, None] * x["S0"], TOL_F32)


def test_single_token_closed_form_fp32():
    cfg, x = _inputs("f32", T=1, s0=0.0)
    o, s = _run(x, "f32", 16)
    k = x["k"].astype(np.float64)
    kt = np.sqrt(x["beta"]) * k / np.sqrt((k ** 2).sum(-1, keepdims=True) + 1e-6)
    vt = np.sqrt(x["beta"]) * x["v"]
    q = x["q"].astype(np.float64)
    qn = q / np.sqrt((q ** 2).sum(-1, keepdims=True) + 1e-6)
    parity(s, np.einsum("bthi,bthj->bhij", kt, vt), TOL_F32)
    parity(o, (kt * qn).sum(-1, keepdims=True) * vt, TOL_F32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_empty_sequence_passes_state_through(dtype):
    cfg, x = _inputs(dtype, T=0)
    o, s = _run(x, dtype, 64)
    assert o.shape[1] == 0
    np.testing.assert_array_equal(s, x["S0"])
    o, s = _run(x, dtype, 64, S0=None)
    np.testing.assert_array_equal(s, np.zeros_like(x["S0"]))


def test_null_final_state_and_zero_state():
    ops = _ops()
    cfg, x = _inputs("bf16", s0=0.0)
    dt = torch.bfloat16
    o1, s1 = ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                           to_dev(x["alpha"]), to_dev(x["beta"]), None, chunk=64)
    o2, s2 = ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                           to_dev(x["alpha"]), to_dev(x["beta"]),
                           torch.zeros_like(s1), chunk=64, want_state=False)
    assert s2 is None
    torch.testing.assert_close(o1, o2, rtol=0, atol=0)


def test_workspace_status_clean_after_runs():
    ops = _ops()
    cfg, x = _inputs("bf16")
    dt = torch.bfloat16
    B, T, H, dk = x["q"].shape
    ws = ops.alloc_workspace(ops.chunk_fwd_workspace_size(B, H, T, dk, dk, 64, ops.GDN_BF16, 0), "cuda")
    for _ in range(2):
        ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                      to_dev(x["alpha"]), to_dev(x["beta"]), None, chunk=64, workspace=ws)
    assert ops.workspace_status(ws) == ops.GDN_OK


def test_too_small_workspace_is_rejected_without_launch():
    ops = _ops()
    cfg, x = _inputs("bf16", T=64)
    dt = torch.bfloat16
    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.GdnError) as e:
        ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                      to_dev(x["alpha"]), to_dev(x["beta"]), None, chunk=64, workspace=ws)
    assert e.value.code == ops.GDN_ERR_WORKSPACE


def test_single_stream_flag_same_result():
    """GDN_SINGLE_STREAM keeps the whole call on the caller's stream (no fork onto the
    library's side stream); a sequence long enough to be cut into chunk ranges gives the
    default call's result bit for bit."""
    ops = _ops()
    cfg = GdnConfig("single", B=1, H=2, T=64 * 70 + 9, dk=128, dv=128, chunk=64, s0_std=0.05, seed=41)
    x = make_inputs(cfg)
    dt = torch.bfloat16
    args = (to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt), to_dev(x["alpha"]), to_dev(x["beta"]),
            to_dev(x["S0"]))
    o1, s1 = ops.chunk_fwd(*args, chunk=64)
    o2, s2 = ops.chunk_fwd(*args, chunk=64, single_stream=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("dtype,dk", [("bf16", 128), ("f32", 64)])
def test_chunk_128_is_chunk_64(dtype, dk):
    """chunk 128 is accepted and evaluated as 64-row chunks: bit for bit the chunk-64 result
    (tensor-core path at bf16 d 128, float32 path at d 64), and within the tolerance of the
    oracle's token-by-token recurrence."""
    import oracle
    cfg, x = _inputs(dtype, T=333, dk=dk)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    o64, s64 = _run(x, dtype, 64)
    o128, s128 = _run(x, dtype, 128)
    assert np.array_equal(o64, o128) and np.array_equal(s64, s128)
    ro, rs = oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"])
    parity(o128, ro, tol, out_bf16=dtype == "bf16")
    parity(s128, rs, tol)

"""GPU parity of gdn2_chunk_fwd (GDN2: non-tied erase / write with the token-wise
stability transforms of Su Jianlin's GDN2 stability note) against the fp64 oracle."""
import numpy as np
import pytest

from gated_delta_rule_fg_b200.inputs import make_gdn2_inputs
from oracle import gdn2 as oracle_gdn2
from _util import TOL_F32, parity, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

MODES = {"none": 0, "clip": 1, "shrink": 2}


def run(x, dtype, chunk, mode):
    from gated_delta_rule_fg_b200 import ops
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out, sf = ops.gdn2_chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt), to_dev(x["alpha"]),
                                 to_dev(x["eta"]), to_dev(x["b"]), to_dev(x["S0"]), mode=MODES[mode], chunk=chunk)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sf.cpu().numpy()


CASES = [(mode, dtype, dk, dv, chunk, T) for mode in MODES
         for (dtype, dk, dv, chunk, T) in (("f32", 64, 64, 16, 70), ("bf16", 128, 128, 32, 100),
                                           ("f32", 32, 128, 32, 33), ("bf16", 128, 64, 16, 17))]


@pytest.mark.parametrize("mode,dtype,dk,dv,chunk,T", CASES)
def test_gdn2_against_oracle(mode, dtype, dk, dv, chunk, T):
    x = make_gdn2_inputs(2, T, 2, dk, dv, dtype=dtype, seed=5000 + T + dk + len(mode))
    got = run(x, dtype, chunk, mode)
    ro, rs = oracle_gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], x["b"], x["S0"], mode=mode)
    parity(got[0], ro, TOL_F32, out_bf16=dtype == "bf16")
    parity(got[1], rs, TOL_F32)


def test_gdn2_tied_is_kda_call():
    """b = 1, no transform: gdn2_chunk_fwd equals gdn_chunk_fwd with scalar beta = eta."""
    from gated_delta_rule_fg_b200 import ops
    x = make_gdn2_inputs(1, 90, 3, 64, 64, seed=5100)
    x["b"] = np.ones_like(x["b"])
    o1, s1 = run(x, "f32", 16, "none")
    o2, s2 = ops.chunk_fwd(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), to_dev(x["alpha"]), to_dev(x["eta"]),
                           to_dev(x["S0"]), chunk=16, beta_scalar=True)
    torch.cuda.synchronize()
    parity(o1, o2.cpu().numpy(), TOL_F32)
    parity(s1, s2.cpu().numpy(), TOL_F32)


def test_gdn2_clip_keeps_state_bounded_where_plain_grows():
    """With eta near 2 and j far from k, the plain GDN2 state can grow; with the decay
    clipped, every transition has spectral norm <= 1, so ||S_T||_F <= ||S_0||_F plus the
    writes.  Checked against the oracle in both modes on a long sequence."""
    x = make_gdn2_inputs(1, 600, 2, 32, 32, seed=5200, alpha_scale=0.001, s0_std=1.0)
    x["eta"] = np.full_like(x["eta"], 1.9)
    x["v"] = np.zeros_like(x["v"])          # no writes: the state only evolves by the transitions
    for mode in ("none", "clip"):
        got = run(x, "f32", 32, mode)
        ro, rs = oracle_gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], x["b"], x["S0"], mode=mode)
        parity(got[1], rs, TOL_F32)
        if mode == "clip":
            assert np.linalg.norm(got[1]) <= np.linalg.norm(x["S0"]) * (1 + 1e-4)


TC = [(mode, T) for mode in MODES for T in (1, 63, 200)]


@pytest.mark.parametrize("mode,T", TC)
def test_gdn2_tensor_core(mode, T):
    """bf16, chunk 64, d = 128 runs on the tensor-core kernels (erase operand in the A rows and
    the state read); fp16 operands, so the bf16 bound of the tied path applies."""
    from _util import TOL_BF16
    x = make_gdn2_inputs(2, T, 2, 128, 128, dtype="bf16", seed=5300 + T + len(mode))
    got = run(x, "bf16", 64, mode)
    ro, rs = oracle_gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], x["b"], x["S0"], mode=mode)
    parity(got[0], ro, TOL_BF16, out_bf16=True)
    parity(got[1], rs, TOL_BF16)


@pytest.mark.parametrize("mode", list(MODES))
def test_gdn2_tensor_core_strong_decay_fallback(mode):
    """Chunks with a wide log-decay span take the element-wise fp32 Gram products, which read
    the erase rows the prep stored for them."""
    from _util import TOL_BF16
    x = make_gdn2_inputs(1, 200, 2, 128, 128, dtype="bf16", seed=5400 + len(mode))
    x["alpha"] = np.where(np.arange(200)[None, :, None, None] % 3 == 0, 1e-6, x["alpha"]).astype(np.float32)
    got = run(x, "bf16", 64, mode)
    ro, rs = oracle_gdn2.gdn2_seq(x["q"], x["k"], x["v"], x["alpha"], x["eta"], x["b"], x["S0"], mode=mode)
    parity(got[0], ro, TOL_BF16, out_bf16=True)
    parity(got[1], rs, TOL_BF16)

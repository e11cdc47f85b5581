"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Small cases run the oracle on everything; the full-size configurations run
the library exactly as bench.py does and compare every head (the oracle
handles (batch, head) pairs independently).
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_fg_b200.inputs import CONFIGS, GdnConfig, make_inputs
from _util import TOL_BF16, TOL_F32, parity, to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _ops():
    from gated_delta_rule_fg_b200 import ops
    return ops


def run_gdn(cfg, x, chunk=None):
    ops = _ops()
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out, sf = ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                            to_dev(x["alpha"]), to_dev(x["beta"]), to_dev(x["S0"]),
                            chunk=chunk or cfg.chunk, alpha_scalar=cfg.alpha_scalar,
                            beta_scalar=cfg.beta_scalar)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sf.cpu().numpy()


def run_dp(cfg, x, chunk=None):
    ops = _ops()
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out, sf = ops.deltaproduct_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                                   to_dev(x["gamma"]), to_dev(x["beta"]), to_dev(x["S0"]),
                                   chunk=chunk or cfg.chunk)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sf.cpu().numpy()


def oracle_gdn(cfg, x, pairs=None):
    return oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                          alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar, pairs=pairs)


def oracle_dp(x, pairs=None):
    return oracle.deltaproduct_seq(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["S0"], pairs=pairs)


def check(cfg, got, ref, pairs=None):
    tol = TOL_BF16 if cfg.dtype == "bf16" else TOL_F32
    (o, s), (ro, rs) = got, ref
    if pairs is not None:
        idx_b = [b for b, _ in pairs]
        idx_h = [h for _, h in pairs]
        o, ro = o[idx_b, :, idx_h], ro[idx_b, :, idx_h]
        s, rs = s[idx_b, idx_h], rs[idx_b, idx_h]
    eo = parity(o, ro, tol, out_bf16=cfg.dtype == "bf16")
    es = parity(s, rs, tol)
    return eo, es


# --------------------------------------------------------------------------- small, full oracle
def test_config_fp32_small_exact_size():
    """The float32 configuration at its stated size, every element."""
    cfg = CONFIGS["fg2_f32_small"]
    x = make_inputs(cfg)
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


SMALL = []
for dtype in ("f32", "bf16"):
    for mode in ("fg2", "kda", "gdn", "deltanet"):
        for T, chunk in ((1, 16), (15, 16), (64, 64), (250, 32), (250, 64), (131, 16)):
            SMALL.append((dtype, mode, T, chunk))


@pytest.mark.parametrize("dtype,mode,T,chunk", SMALL)
def test_small_modes(dtype, mode, T, chunk):
    """Every gate mode, ragged tails (T % chunk != 0), T < chunk and T = 1, both dtypes."""
    cfg = GdnConfig("small", B=2, H=3, T=T, dk=64, dv=64, chunk=chunk, dtype=dtype,
                    alpha_scalar=mode == "gdn", beta_scalar=mode in ("kda", "gdn", "deltanet"),
                    s0_std=0.1 if T % 2 else 0.0, seed=T * 7 + chunk)
    x = make_inputs(cfg)
    if mode == "deltanet":
        x["alpha"] = np.ones_like(x["alpha"])
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


@pytest.mark.parametrize("dk", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_head_dims(dk, dtype):
    cfg = GdnConfig("dims", B=1, H=2, T=200, dk=dk, dv=dk, chunk=64 if dk == 128 else 32,
                    dtype=dtype, s0_std=0.05, seed=dk)
    x = make_inputs(cfg)
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


def test_kda_unequal_head_dims():
    """Scalar beta allows dk != dv."""
    cfg = GdnConfig("kda_rect", B=1, H=2, T=100, dk=64, dv=128, chunk=32, beta_scalar=True,
                    s0_std=0.05, seed=9)
    x = make_inputs(cfg)
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("nh,T,chunk", [(2, 40, 16), (2, 100, 64), (3, 33, 32), (1, 50, 16), (4, 17, 64)])
def test_deltaproduct_small(dtype, nh, T, chunk):
    cfg = GdnConfig("dp", B=2, H=2, T=T, dk=64, dv=64, chunk=chunk, dtype=dtype,
                    deltaproduct_nh=nh, seed=nh * 100 + T)
    x = make_inputs(cfg)
    check(cfg, run_dp(cfg, x), oracle_dp(x))


def test_strong_decay_small_alpha():
    """Tiny alpha (log-decay span of hundreds inside a chunk) stays finite and exact."""
    for dtype in ("f32", "bf16"):
        cfg = GdnConfig("decay", B=1, H=2, T=130, dk=64, dv=64, chunk=64, dtype=dtype, seed=77)
        x = make_inputs(cfg)
        x["alpha"] = np.where(np.arange(130)[None, :, None, None] % 3 == 0, 1e-6,
                              x["alpha"]).astype(np.float32)
        check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


# --------------------------------------------------------------------------- full sizes
FULL = ["kda_bf16", "fg2_prefill_32k", "fg2_train_b8", "deltaproduct_nh2"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_all_heads(name):
    """Full-size configurations in the benchmark's launch configuration; the oracle
    recomputes every (batch, head) pair, so every output element and every state entry of
    the call is compared."""
    cfg = CONFIGS[name]
    x = make_inputs(cfg)
    if cfg.deltaproduct_nh:
        got = run_dp(cfg, x)
        ref = oracle_dp(x)
    else:
        got = run_gdn(cfg, x)
        ref = oracle_gdn(cfg, x)
    check(cfg, got, ref)


# --------------------------------------------------------------------------- tensor-core path shapes
TC = [(mode, T) for mode in ("fg2", "kda", "gdn", "deltanet") for T in (1, 63, 64, 65, 200)]


@pytest.mark.parametrize("mode,T", TC)
def test_tensor_core_shapes_modes(mode, T):
    """bf16, chunk 64, dk = dv = 128 (the tensor-core kernels): every gate mode, T < chunk,
    T = chunk, one past, ragged; nonzero S0 on odd T."""
    cfg = GdnConfig("tc", B=2, H=2, T=T, dk=128, dv=128, chunk=64, dtype="bf16",
                    alpha_scalar=mode == "gdn", beta_scalar=mode in ("kda", "gdn", "deltanet"),
                    s0_std=0.1 if T % 2 else 0.0, seed=1000 + T)
    x = make_inputs(cfg)
    if mode == "deltanet":
        x["alpha"] = np.ones_like(x["alpha"])
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


@pytest.mark.parametrize("nh,T", [(2, 100), (3, 70), (1, 130), (4, 50)])
def test_tensor_core_deltaproduct(nh, T):
    cfg = GdnConfig("tcdp", B=1, H=2, T=T, dk=128, dv=128, chunk=64, deltaproduct_nh=nh,
                    s0_std=0.05, seed=2000 + T)
    x = make_inputs(cfg)
    check(cfg, run_dp(cfg, x), oracle_dp(x))


def test_tensor_core_strong_decay_fallback():
    """Chunks whose log-decay span is too wide for the factored fp16 Gram products take the
    element-wise path; results stay exact."""
    cfg = GdnConfig("tcdecay", B=1, H=2, T=200, dk=128, dv=128, chunk=64, seed=78)
    x = make_inputs(cfg)
    x["alpha"] = np.where(np.arange(200)[None, :, None, None] % 3 == 0, 1e-6, x["alpha"]).astype(np.float32)
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


# --------------------------------------------------------------------------- FG^2-GDN+
def run_plus(cfg, x, chunk=None):
    ops = _ops()
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    out, sf = ops.plus_chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt),
                                 to_dev(x["alpha"]), to_dev(x["beta"]), to_dev(x["beta_v"]),
                                 to_dev(x["S0"]), chunk=chunk or cfg.chunk,
                                 alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), sf.cpu().numpy()


def oracle_plus(cfg, x, pairs=None):
    return oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], beta_v=x["beta_v"],
                          alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar, pairs=pairs)


PLUS = [("f32", 64, 64, 16, 131), ("f32", 32, 64, 32, 70), ("f32", 128, 32, 64, 100),
        ("bf16", 64, 64, 32, 250), ("bf16", 128, 128, 64, 1), ("bf16", 128, 128, 64, 63),
        ("bf16", 128, 128, 64, 65), ("bf16", 128, 128, 64, 200)]


@pytest.mark.parametrize("dtype,dk,dv,chunk,T", PLUS)
@pytest.mark.parametrize("scalar", [False, True])
def test_plus_small(dtype, dk, dv, chunk, T, scalar):
    """FG^2-GDN+ (separate beta^k / beta^v): CUDA-core and tensor-core shapes, dk != dv,
    ragged tails, scalar and channel-wise rates; nonzero S0 on odd T."""
    cfg = GdnConfig("plus", B=2, H=2, T=T, dk=dk, dv=dv, chunk=chunk, dtype=dtype, plus=True,
                    beta_scalar=scalar, s0_std=0.1 if T % 2 else 0.0, seed=3000 + T + dk)
    x = make_inputs(cfg)
    check(cfg, run_plus(cfg, x), oracle_plus(cfg, x))


def test_plus_equal_rates_matches_fg2_call():
    """gdn_plus_chunk_fwd with beta_v = beta_k returns gdn_chunk_fwd's result bit for bit."""
    cfg = GdnConfig("plus_eq", B=1, H=4, T=300, dk=128, dv=128, chunk=64, plus=True, s0_std=0.05,
                    seed=3100)
    x = make_inputs(cfg)
    x["beta_v"] = x["beta"].copy()
    o1, s1 = run_plus(cfg, x)
    o2, s2 = run_gdn(cfg, x)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_plus_full_size_all_heads():
    """FG^2-GDN+ on the 32K-token prefill shape; every head against the oracle."""
    base = CONFIGS["fg2_prefill_32k"]
    cfg = GdnConfig("plus_prefill_32k", B=base.B, H=base.H, T=base.T, dk=base.dk, dv=base.dv,
                    chunk=base.chunk, plus=True, seed=3200)
    x = make_inputs(cfg)
    check(cfg, run_plus(cfg, x), oracle_plus(cfg, x))


def test_tensor_core_segmented_call_uneven_ranges():
    """A sequence long enough for the call to be cut into chunk ranges whose intra and scan
    roles overlap on two streams (98 chunks: three uneven ranges) with a ragged last chunk
    and a nonzero initial state: every token and the final state match the oracle."""
    cfg = GdnConfig("tcseg", B=1, H=2, T=64 * 97 + 13, dk=128, dv=128, chunk=64, s0_std=0.05, seed=6100)
    x = make_inputs(cfg)
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x))


def test_tensor_core_large_offsets_sampled_heads():
    """B5 H16 T32768: the workspace (40,960 chunk blocks, 4.7 GB) passes 2^32 bytes, so every
    block offset must be 64-bit.  Sampled heads include every head of the last batch, whose
    blocks sit at the top of the workspace."""
    base = CONFIGS["fg2_prefill_32k"]
    cfg = GdnConfig("large", B=5, H=16, T=base.T, dk=128, dv=128, chunk=64, s0_std=0.01, seed=6200)
    x = make_inputs(cfg)
    pairs = [(0, 0), (3, 9)] + [(4, h) for h in range(cfg.H)]
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x, pairs=pairs), pairs=pairs)


@pytest.mark.parametrize("T,pairs", [(64 * 3 + 17, None), (64 * 70 + 5, [(0, 0), (5, 2), (9, 3)])])
def test_tensor_core_wide_scan_grid(T, pairs):
    """B10 H4: one 32-column slice per scan CTA would need 160 CTAs, more than one wave of
    SMs, so the scan carries two slices per CTA.  Short (every head checked) and segmented
    (sampled heads) calls, nonzero S0."""
    cfg = GdnConfig("tcw2", B=10, H=4, T=T, dk=128, dv=128, chunk=64, s0_std=0.05, seed=6300 + T)
    x = make_inputs(cfg)
    check(cfg, run_gdn(cfg, x), oracle_gdn(cfg, x, pairs=pairs), pairs=pairs)

"""gdn_chunk_fwd_noalloc: the entry point for callers that cannot allocate device
memory (framework allocators, fixed-memory runtimes, stream capture).  It must give
the same results as gdn_chunk_fwd with a caller workspace, on consecutive calls that
reuse its built-in scratch, and refuse sizes beyond that scratch without launching.
This file is collected last so that a run stopping at the first failure has already
run every other test."""
import ctypes

import numpy as np
import pytest

from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
from _util import to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _both(cfg, x):
    from gated_delta_rule_fg_b200 import ops
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    args = (to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt), to_dev(x["alpha"]),
            to_dev(x["beta"]), to_dev(x["S0"]))
    kw = dict(chunk=cfg.chunk, alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar)
    o_ref, s_ref = ops.chunk_fwd(*args, **kw)
    o_na, s_na = ops.chunk_fwd_noalloc(*args, **kw)
    torch.cuda.synchronize()
    return (o_na.float().cpu().numpy(), s_na.cpu().numpy()), (o_ref.float().cpu().numpy(), s_ref.cpu().numpy())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    """Both entry points run the same kernels on the same inputs, so the results are
    identical bit for bit, on two consecutive calls that reuse the shared scratch."""
    d = 128 if dtype == "bf16" else 32
    for call, T in enumerate((300, 177)):          # two calls in a row on the shared scratch
        cfg = GdnConfig("noalloc", B=1, H=4, T=T, dk=d, dv=d, chunk=64 if dtype == "bf16" else 16,
                        dtype=dtype, s0_std=0.05 * call, seed=90 + call)
        x = make_inputs(cfg)
        (o, s), (ro, rs) = _both(cfg, x)
        np.testing.assert_array_equal(o, ro)
        np.testing.assert_array_equal(s, rs)


def test_noalloc_binding_rejects_wrong_output_dtype():
    """A caller-supplied output of the wrong dtype is refused before the library is called
    (a float32 q with a bfloat16 out would otherwise be written past its end)."""
    from gated_delta_rule_fg_b200 import ops
    cfg = GdnConfig("noalloc_dtype", B=1, H=2, T=32, dk=32, dv=32, chunk=16, dtype="f32", seed=97)
    x = make_inputs(cfg)
    q, k, v = (to_dev(x[n], torch.float32) for n in ("q", "k", "v"))
    a, b = to_dev(x["alpha"]), to_dev(x["beta"])
    bad_out = torch.empty((1, 32, 2, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        ops.chunk_fwd_noalloc(q, k, v, a, b, out=bad_out, chunk=16)
    bad_s = torch.empty((1, 2, 32, 32), dtype=torch.float64, device="cuda")
    with pytest.raises(TypeError):
        ops.chunk_fwd_noalloc(q, k, v, a, b, S_final=bad_s, chunk=16)


def test_noalloc_rejected_call_enqueues_nothing():
    """Argument errors are found before the scratch status word is cleared: a misaligned
    pointer returns GDN_ERR_INVALID_ARG and leaves the stream without new work."""
    from gated_delta_rule_fg_b200 import ops
    L = ops.lib()
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10004)
    torch.cuda.synchronize()
    st = L.gdn_chunk_fwd_noalloc(fake, fake, odd, fake, fake, None, fake, None, 1, 2, 64, 128, 128,
                                 64, ops.GDN_BF16, 0, None)
    assert st == ops.GDN_ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from gated_delta_rule_fg_b200 import ops
    L = ops.lib()
    fake = ctypes.c_void_p(0x10000)
    # 32K tokens x 16 heads needs ~0.9 GB of scratch, far beyond the built-in 64 MiB
    st = L.gdn_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, None, 1, 16, 32768, 128, 128,
                                 64, ops.GDN_BF16, 0, None)
    assert st == ops.GDN_ERR_WORKSPACE
    st = L.gdn_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, None, 1, 1, 64, 96, 96,
                                 64, ops.GDN_BF16, 0, None)
    assert st == ops.GDN_ERR_UNSUPPORTED

"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/gdn.h declares, sizes the workspace, and validates arguments before
touching the device."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_fg_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

FAKE = 0x10000            # an aligned, never dereferenced stand-in for a device pointer
FAKE_ODD = 0x10008        # 8-byte aligned only


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_fg_b200 import build
    build.build()
    return ops.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"gdn_chunk_fwd", "gdn_deltaproduct_fwd", "gdn_workspace_status"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in gdn.h but not exported"
        assert n in ops.SIGNATURES, f"{n} has no ctypes signature in ops.py"


def test_version_and_status_strings(L):
    assert L.gdn_version() >= 100
    for code in range(8):
        assert len(ops.status_string(code)) > 0
    assert ops.status_string(ops.GDN_ERR_BOUNDS) != "unknown status"
    assert ops.status_string(99) == "unknown status"


def test_path_query(L):
    """gdn_chunk_fwd_tensor_cores says which path a call takes (no device access)."""
    tc = ops.chunk_fwd_tensor_cores
    assert tc(1, 16, 32768, 128, 128, 64, ops.GDN_BF16) == 1
    assert tc(1, 16, 32768, 128, 128, 128, ops.GDN_BF16) == 1      # chunk 128: 64-row chunks
    assert tc(1, 2, 0, 128, 128, 64, ops.GDN_BF16) == 1             # empty sequence: same path
    assert tc(1, 16, 4096, 128, 128, 32, ops.GDN_BF16) == 0         # chunk 32: CUDA cores
    assert tc(1, 16, 4096, 64, 64, 64, ops.GDN_BF16) == 0           # d 64: CUDA cores
    assert tc(1, 16, 4096, 64, 64, 64, ops.GDN_F32) == 0            # float32: CUDA cores
    assert tc(1, 16, 4096, 96, 96, 64, ops.GDN_BF16) == -1          # unsupported head dim
    assert tc(1, 16, 4096, 128, 128, 48, ops.GDN_BF16) == -1        # unsupported chunk


def test_bounds_checking_build_exports_the_same_abi():
    """The bounds-checking build (-DGDN_DEBUG_BOUNDS) is the same ABI in another file."""
    from gated_delta_rule_fg_b200 import build
    path = build.build(debug_bounds=True)
    assert path == ops.BOUNDS_LIB_PATH and os.path.exists(path)
    B = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(B, n), f"{n} declared in gdn.h but not exported by the bounds-checking build"
    B.gdn_chunk_fwd_workspace_size.restype = ctypes.c_size_t
    B.gdn_chunk_fwd_workspace_size.argtypes = ops.SIGNATURES["gdn_chunk_fwd_workspace_size"][1]
    assert B.gdn_chunk_fwd_workspace_size(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0) == \
        ops.chunk_fwd_workspace_size(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0)


def test_workspace_sizes(L):
    ws = ops.chunk_fwd_workspace_size
    assert ws(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0) > 0
    assert ws(1, 2, 256, 32, 32, 16, ops.GDN_F32, 0) > 0
    assert ws(1, 1, 0, 64, 64, 64, ops.GDN_F32, 0) > 0          # T = 0 is valid
    assert ws(1, 1, 10, 48, 48, 64, ops.GDN_F32, 0) == 0        # unsupported head dim
    assert ws(1, 1, 10, 64, 64, 48, ops.GDN_F32, 0) == 0        # unsupported chunk
    assert ws(1, 1, 10, 64, 128, 64, ops.GDN_F32, 0) == 0       # channel-wise beta, dk != dv
    assert ws(1, 1, 10, 64, 128, 64, ops.GDN_F32, ops.GDN_BETA_SCALAR) > 0
    assert ws(-1, 1, 10, 64, 64, 64, ops.GDN_F32, 0) == 0
    a = ws(1, 4, 1000, 64, 64, 32, ops.GDN_F32, 0)
    b = ws(1, 4, 2000, 64, 64, 32, ops.GDN_F32, 0)
    assert b > a                                                # grows with T
    dws = ops.deltaproduct_fwd_workspace_size
    assert dws(2, 8, 8192, 2, 128, 128, 64, ops.GDN_BF16) > 0
    assert dws(2, 8, 8192, 5, 128, 128, 64, ops.GDN_BF16) == 0  # n_h > 4


def _call(L, q=FAKE, k=FAKE, v=FAKE, alpha=FAKE, beta=FAKE, S0=None, out=FAKE, Sf=None,
          B=1, H=1, T=8, dk=64, dv=64, chunk=64, dtype=ops.GDN_F32, flags=0,
          ws=FAKE, wsb=1 << 30):
    return L.gdn_chunk_fwd(q, k, v, alpha, beta, S0, out, Sf, B, H, T, dk, dv, chunk, dtype,
                           flags, ws, wsb, None)


def test_argument_validation_before_launch(L):
    assert _call(L, q=None) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, beta=None) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, out=None) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, k=FAKE_ODD) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, Sf=FAKE_ODD) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, B=-1) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, dtype=7) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, flags=8) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, dk=64, dv=128) == ops.GDN_ERR_INVALID_ARG
    assert _call(L, dk=96, dv=96) == ops.GDN_ERR_UNSUPPORTED
    assert _call(L, chunk=256) == ops.GDN_ERR_UNSUPPORTED
    # chunk 128 is accepted and evaluated as 64-row chunks: same workspace and launches as chunk 64
    for dt, d in ((ops.GDN_BF16, 128), (ops.GDN_F32, 64)):
        assert L.gdn_chunk_fwd_workspace_size(1, 4, 1000, d, d, 128, dt, 0) == \
            L.gdn_chunk_fwd_workspace_size(1, 4, 1000, d, d, 64, dt, 0) > 0
        assert L.gdn_chunk_fwd_launches(1, 4, 1000, d, d, 128, dt, 0) == L.gdn_chunk_fwd_launches(1, 4, 1000, d, d, 64, dt, 0)
    assert _call(L, chunk=0) == ops.GDN_ERR_UNSUPPORTED
    assert _call(L, ws=None) == ops.GDN_ERR_WORKSPACE
    assert _call(L, ws=FAKE + 16) == ops.GDN_ERR_WORKSPACE       # not 256-byte aligned
    assert _call(L, wsb=1024) == ops.GDN_ERR_WORKSPACE           # too small
    # empty batch: valid, nothing to do, no device access
    assert _call(L, B=0) == ops.GDN_OK
    assert _call(L, H=0) == ops.GDN_OK
    assert _call(L, B=0, flags=ops.GDN_SINGLE_STREAM) == ops.GDN_OK   # the single-stream flag is accepted
    assert L.gdn_chunk_fwd_workspace_size(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, ops.GDN_SINGLE_STREAM) > 0


def test_deltaproduct_validation(L):
    f = L.gdn_deltaproduct_fwd
    args = [FAKE] * 5 + [None, FAKE, None]
    assert f(*args, 1, 1, 8, 0, 64, 64, 64, ops.GDN_BF16, FAKE, 1 << 30, None) == ops.GDN_ERR_UNSUPPORTED
    assert f(*args, 1, 1, 8, 5, 64, 64, 64, ops.GDN_BF16, FAKE, 1 << 30, None) == ops.GDN_ERR_UNSUPPORTED
    bad = [None] + [FAKE] * 4 + [None, FAKE, None]
    assert f(*bad, 1, 1, 8, 2, 64, 64, 64, ops.GDN_BF16, FAKE, 1 << 30, None) == ops.GDN_ERR_INVALID_ARG
    assert f(*args, 1, 1, 8, 2, 64, 64, 64, ops.GDN_BF16, None, 0, None) == ops.GDN_ERR_WORKSPACE


def test_status_query_needs_workspace(L):
    assert L.gdn_workspace_status(None, None) == ops.GDN_ERR_WORKSPACE


def test_plus_validation(L):
    """gdn_plus_chunk_fwd: channel-wise rates allow dk != dv; beta_v is required and
    checked for alignment; errors come back before anything is enqueued."""
    pws = ops.plus_chunk_fwd_workspace_size
    assert pws(1, 2, 100, 64, 128, 32, ops.GDN_F32, 0) > 0       # dk != dv with channel-wise rates
    assert ops.chunk_fwd_workspace_size(1, 2, 100, 64, 128, 32, ops.GDN_F32, 0) == 0
    assert pws(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0) == \
        ops.chunk_fwd_workspace_size(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0)
    # 512 chunks: four chunk ranges, each an intra and a scan launch
    assert ops.plus_chunk_fwd_launches(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0) == 8
    assert ops.chunk_fwd_launches(1, 16, 32768, 128, 128, 64, ops.GDN_BF16, 0) == 8
    assert ops.chunk_fwd_launches(1, 16, 2048, 128, 128, 64, ops.GDN_BF16, 0) == 2      # 32 chunks: one range
    assert pws(1, 1, 10, 96, 96, 64, ops.GDN_F32, 0) == 0

    def call(beta_v=FAKE, **kw):
        a = dict(B=1, H=1, T=8, dk=64, dv=64, chunk=64, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.gdn_plus_chunk_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, beta_v, None, FAKE, None,
                                    a["B"], a["H"], a["T"], a["dk"], a["dv"], a["chunk"],
                                    ops.GDN_F32, 0, a["ws"], a["wsb"], None)

    assert call(beta_v=None) == ops.GDN_ERR_INVALID_ARG
    assert call(beta_v=FAKE_ODD) == ops.GDN_ERR_INVALID_ARG
    assert call(dk=96, dv=96) == ops.GDN_ERR_UNSUPPORTED
    assert call(ws=None) == ops.GDN_ERR_WORKSPACE
    assert call(B=0) == ops.GDN_OK


def test_recurrent_step_validation(L):
    f = L.gdn_recurrent_step

    def call(q=FAKE, beta_v=None, S_in=None, S_out=FAKE, out=FAKE, B=1, H=1, dk=64, dv=64, flags=0,
             dtype=ops.GDN_F32):
        return f(q, FAKE, FAKE, FAKE, FAKE, beta_v, S_in, S_out, out, B, H, dk, dv, dtype, flags, None)

    assert call(q=None) == ops.GDN_ERR_INVALID_ARG
    assert call(S_out=None) == ops.GDN_ERR_INVALID_ARG
    assert call(out=FAKE_ODD) == ops.GDN_ERR_INVALID_ARG
    assert call(dk=64, dv=128) == ops.GDN_ERR_INVALID_ARG              # channel-wise beta on v
    assert call(dk=96, dv=96) == ops.GDN_ERR_UNSUPPORTED
    assert call(dtype=5) == ops.GDN_ERR_INVALID_ARG
    assert call(flags=4) == ops.GDN_ERR_INVALID_ARG
    assert call(S_in=FAKE + 256, S_out=FAKE) == ops.GDN_ERR_INVALID_ARG  # partial overlap
    assert call(B=-1) == ops.GDN_ERR_INVALID_ARG
    assert call(B=0) == ops.GDN_OK


def test_backward_validation(L):
    bws = ops.chunk_bwd_workspace_size
    assert bws(1, 2, 100, 64, 64, 32, ops.GDN_F32, 0) > 0
    assert bws(1, 2, 100, 64, 64, 64, ops.GDN_F32, 0) == 0          # chunk 64 not in the backward
    assert bws(1, 2, 100, 128, 128, 16, ops.GDN_BF16, 0) > 0
    assert ops.chunk_bwd_launches(1, 2, 100, 64, 64, 32, ops.GDN_F32, 0) == 4
    assert ops.chunk_bwd_launches(1, 2, 0, 64, 64, 32, ops.GDN_F32, 0) == 1

    def call(dbeta_v=None, beta_v=None, dout=FAKE, chunk=32, ws=FAKE):
        return L.gdn_chunk_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, beta_v, None, dout, None, FAKE, FAKE,
                               FAKE, FAKE, FAKE, dbeta_v, FAKE, 1, 1, 8, 64, 64, chunk, ops.GDN_F32, 0,
                               ws, 1 << 30, None)

    assert call(dout=None) == ops.GDN_ERR_INVALID_ARG
    assert call(dbeta_v=FAKE) == ops.GDN_ERR_INVALID_ARG              # dbeta_v without beta_v
    assert call(chunk=64) == ops.GDN_ERR_UNSUPPORTED
    assert call(ws=None) == ops.GDN_ERR_WORKSPACE
    assert call(dout=FAKE_ODD) == ops.GDN_ERR_INVALID_ARG


def test_gdn2_validation(L):
    ws = ops.gdn2_chunk_fwd_workspace_size
    assert ws(1, 2, 100, 64, 64, 32, ops.GDN_F32, 0) > 0
    assert ws(1, 2, 100, 128, 128, 64, ops.GDN_F32, 0) == 0           # float32 path: chunk 64 at d 128 does not fit
    assert ws(1, 2, 100, 128, 128, 64, ops.GDN_BF16, 0) > 0           # ... the tensor-core path takes it
    assert ws(1, 2, 100, 64, 64, 32, ops.GDN_F32, ops.GDN_BETA_SCALAR) == 0
    assert L.gdn2_chunk_fwd_launches(1, 2, 100, 64, 64, 32, ops.GDN_F32, 0) == 2

    def call(eta=FAKE, mode=0, chunk=32):
        return L.gdn2_chunk_fwd(FAKE, FAKE, FAKE, FAKE, eta, FAKE, None, FAKE, None, 1, 1, 8, 64, 64, chunk,
                                ops.GDN_F32, 0, mode, FAKE, 1 << 30, None)

    assert call(eta=None) == ops.GDN_ERR_INVALID_ARG
    assert call(mode=3) == ops.GDN_ERR_INVALID_ARG
    assert call(chunk=48) == ops.GDN_ERR_UNSUPPORTED

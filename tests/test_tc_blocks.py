"""Unit check of the tensor-core intra-chunk kernel: decode the per-chunk blocks it
writes into the workspace (N = -K'^T W, Qe, b = K'^T U', PU', e^{g_last}) and compare them with the
same quantities formed in fp64 numpy from their definitions (chunk-local cumulative
log-decay g, A and P with the decay taken element by element, T = (I + A)^{-1}).
The block layout is the library's internal contract between its two kernels (Qe is stored
K-major, rows of 128 channels, for the scan's tensor-memory copy)."""
import numpy as np
import pytest

from gated_delta_rule_fg_b200.inputs import GdnConfig, make_inputs
from _util import to_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

C, D, NS = 64, 128, 32
BLOCK = 115200
OFF_N, OFF_QE, OFF_B, OFF_PU, OFF_GC = 0, 32768, 49152, 81920, 98304


def off_mn(mn, k, sbo, lbo):
    return (mn % 8) * 2 + (k % 8) * 16 + (mn // 8) * sbo + (k // 8) * lbo


def off_k(mn, k, sbo, lbo):
    return (mn % 8) * 16 + (k % 8) * 2 + (mn // 8) * sbo + (k // 8) * lbo


def grp(row, j, nrows):
    # group-major slice: 16-byte groups (8 columns) of consecutive rows are consecutive
    return ((j // 8) * nrows + row) * 8 + j % 8


def decode(blk):
    h = blk.view(np.float16)
    f = blk.view(np.float32)
    i2, c2 = np.meshgrid(np.arange(128), np.arange(128), indexing="ij")
    N = h[(OFF_N + off_k(i2, c2, 2048, 128)) // 2].astype(np.float64)
    r2, c3 = np.meshgrid(np.arange(64), np.arange(128), indexing="ij")
    Qe = h[(OFF_QE + off_k(r2, c3, 2048, 128)) // 2].astype(np.float64)
    jj = np.arange(128)
    bi, bj = np.meshgrid(np.arange(128), jj, indexing="ij")
    b = h[OFF_B // 2 + (bj // NS) * 128 * NS + grp(bi, bj % NS, 128)].astype(np.float64)
    pr, pj = np.meshgrid(np.arange(64), jj, indexing="ij")
    PU = h[OFF_PU // 2 + (pj // NS) * 64 * NS + grp(pr, pj % NS, 64)].astype(np.float64)
    gC = f[OFF_GC // 4:OFF_GC // 4 + D]
    return dict(N=N, Qe=Qe, b=b, PUp=PU, gC=gC)


def expected(x, h, c0, n, beta_scalar=False):
    q = x["q"][0, c0:c0 + n, h].astype(np.float64)
    k = x["k"][0, c0:c0 + n, h].astype(np.float64)
    v = x["v"][0, c0:c0 + n, h].astype(np.float64)
    al = x["alpha"][0, c0:c0 + n, h].astype(np.float64)
    be = x["beta"][0, c0:c0 + n, h].astype(np.float64)
    if beta_scalar:
        be = np.repeat(be[:, None], D, axis=1)
    pad = C - n
    qh = q / np.sqrt((q ** 2).sum(-1, keepdims=True) + 1e-6)
    kt = np.sqrt(be) * k / np.sqrt((k ** 2).sum(-1, keepdims=True) + 1e-6)
    vt = np.sqrt(be) * v
    la = np.log(al)
    qh, kt, vt, la = (np.pad(a, ((0, pad), (0, 0))) for a in (qh, kt, vt, la))
    g = np.cumsum(la, axis=0)
    low = np.tril(np.ones((C, C), bool))
    Dm = np.exp(np.where(low[:, :, None], g[:, None, :] - g[None, :, :], -np.inf))
    A = np.einsum("rc,ic,ric->ri", kt, kt, Dm) * np.tril(np.ones((C, C)), -1)
    P = np.einsum("rc,ic,ric->ri", qh, kt, Dm)
    T = np.linalg.inv(np.eye(C) + A)
    W = T @ (kt * np.exp(g))
    Up = T @ vt
    Kp = kt * np.exp(g[-1] - g)
    return dict(N=-Kp.T @ W, Qe=qh * np.exp(g) - P @ W, b=Kp.T @ Up, PUp=P @ Up, gC=np.exp(g[-1]))


def _rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)


@pytest.mark.parametrize("alpha_mode", ["normal", "strong"])
def test_intra_blocks(alpha_mode):
    from gated_delta_rule_fg_b200 import ops
    T, H = 150, 2
    cfg = GdnConfig("blk", B=1, H=H, T=T, dk=D, dv=D, chunk=C, seed=31)
    x = make_inputs(cfg)
    if alpha_mode == "strong":      # a chunk whose log-decay half-span exceeds the factored range
        x["alpha"][:, 64:128] = np.where(np.arange(D)[None, None, None, :] % 2 == 0, 0.6, 0.95)
    dt = torch.bfloat16
    need = ops.chunk_fwd_workspace_size(1, H, T, D, D, C, ops.GDN_BF16, 0)
    ws = ops.alloc_workspace(need, "cuda")
    ops.chunk_fwd(to_dev(x["q"], dt), to_dev(x["k"], dt), to_dev(x["v"], dt), to_dev(x["alpha"]),
                  to_dev(x["beta"]), None, chunk=C, workspace=ws)
    torch.cuda.synchronize()
    raw = ws.cpu().numpy()[256:]
    NC = (T + C - 1) // C
    for h in range(H):
        for c in range(NC):
            n = min(C, T - c * C)
            got = decode(raw[(h * NC + c) * BLOCK:(h * NC + c + 1) * BLOCK])
            want = expected(x, h, c * C, n)
            for key, tol in (("N", 3e-3), ("Qe", 3e-3), ("b", 3e-3), ("PUp", 3e-3), ("gC", 1e-5)):
                assert _rel(got[key], want[key]) < tol, (h, c, key, _rel(got[key], want[key]))

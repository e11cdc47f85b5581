"""Checks the tensor-core conventions the library's sm_100a kernels rely on
(shared-memory canonical layouts, descriptor LBO/SBO roles, instruction
descriptor fields, TMEM lane mapping for M = 64 / 128, operand negation) with
a test-only kernel built from tests/csrc/umma_probe.cu, against torch."""
import ctypes
import itertools
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "umma_probe.cu")
SO = os.path.join(HERE, "_build", "umma_probe.so")


@pytest.fixture(scope="module")
def probe():
    os.makedirs(os.path.dirname(SO), exist_ok=True)
    if not os.path.exists(SO) or os.path.getmtime(SO) < os.path.getmtime(SRC):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2",
                               "-Xcompiler", "-fPIC", "-shared", "-o", SO, SRC])
    L = ctypes.CDLL(SO)
    L.umma_probe.restype = ctypes.c_int
    L.umma_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    return L


CASES = [c for c in itertools.product([64, 128], [32, 64, 256], [64, 128], [0, 1], [0, 1], [0, 1], [0, 1])
         if not (c[2] == 64 and c[1] == 256)]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,a_order,b_order", CASES)
def test_umma_layouts(probe, M, N, K, a_mn, b_mn, a_order, b_order):
    g = torch.Generator().manual_seed(M * 1000 + N * 10 + K + a_mn + 2 * b_mn)
    A = torch.randn(M, K, generator=g).half().cuda()
    B = torch.randn(K, N, generator=g).half().cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for neg in (0, 1):
        rc = probe.umma_probe(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, a_mn, b_mn, a_order,
                              b_order, neg, err.data_ptr())
        assert rc == 0
        torch.cuda.synchronize()
        assert int(err.item()) == 0, "MMA completion wait timed out"
        ref = (A.float() @ B.float()) * (-1.0 if neg else 1.0)
        torch.testing.assert_close(D, ref, rtol=1e-3, atol=1e-3)


def _probe_sw(probe):
    probe.umma_probe_sw.restype = ctypes.c_int
    probe.umma_probe_sw.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p]
    return probe.umma_probe_sw


SW_CASES = [c for c in itertools.product([64, 128], [64, 128], [64, 128], [0, 1], [0, 1])]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn", SW_CASES)
def test_umma_swizzle128_layouts(probe, M, N, K, a_mn, b_mn):
    """128-byte-swizzled operands as a TMA load writes them (K-major: +32 B per K step inside a
    64-element box; MN-major: LBO = box stride, +2048 B per K step) give the plain product."""
    f = _probe_sw(probe)
    g = torch.Generator().manual_seed(M + N + K + a_mn + 2 * b_mn)
    A = torch.randn(M, K, generator=g).half().cuda()
    B = torch.randn(K, N, generator=g).half().cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert f(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, a_mn, b_mn, err.data_ptr()) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0, "MMA completion wait timed out"
    torch.testing.assert_close(D, A.float() @ B.float(), rtol=1e-3, atol=1e-3)


TA_CASES = [(M, N, K, b_mn) for M in (64, 128) for N in (32, 64, 128, 256) for K in (64, 128) for b_mn in (0, 1)]


@pytest.mark.parametrize("M,N,K,b_mn", TA_CASES)
def test_umma_tmem_a_operand(probe, M, N, K, b_mn):
    """A operand in tensor memory: row m of A in the lane its D row would use (m for M = 128,
    (m % 16) + 32 (m / 16) for M = 64), two fp16 per 32-bit column (even k low), K / 2 columns
    and 8 columns per K step of 16."""
    probe.umma_probe_ta.restype = ctypes.c_int
    probe.umma_probe_ta.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    g = torch.Generator().manual_seed(M + N + K + b_mn)
    A = torch.randn(M, K, generator=g).half().cuda()
    B = torch.randn(K, N, generator=g).half().cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    row_map = 0 if M == 128 else 1
    assert probe.umma_probe_ta(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, K, b_mn, 0, row_map,
                               err.data_ptr()) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0, "MMA completion wait timed out"
    torch.testing.assert_close(D, A.float() @ B.float(), rtol=1e-3, atol=1e-3)

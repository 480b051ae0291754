"""GPU self-test of the hand-written tcgen05 wrappers (descriptor encodings,
operand majorness, TMEM data layout) on single bf16 GEMMs against torch fp32."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "cuda", "tc_selftest.cu")
SO = os.path.join(HERE, "cuda", "libtcselftest.so")


def _lib():
    hdr = os.path.join(ROOT, "gated_delta_rule_99_b200", "csrc", "tc_ptx.cuh")
    if not os.path.exists(SO) or os.path.getmtime(SO) < max(os.path.getmtime(SRC),
                                                           os.path.getmtime(hdr)):
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-O2", "-std=c++17", "-shared",
                               "-Xcompiler", "-fPIC", "-gencode", "arch=compute_100a,code=sm_100a",
                               "-I", os.path.dirname(hdr), "-o", SO, SRC])
    L = ctypes.CDLL(SO)
    L.tc_selftest_run.restype = ctypes.c_int
    L.tc_selftest_run.argtypes = ([ctypes.c_void_p] * 3 + [ctypes.c_int] * 6 + [ctypes.c_void_p] +
                                  [ctypes.c_int])
    return L


def run(A, B, M, N, Kd, a_mn, b_mn, swap=0, a_tmem=0):
    L = _lib()
    D = torch.full((128, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.tc_selftest_run(A.data_ptr(), B.data_ptr(), D.data_ptr(), M, N, Kd, a_mn, b_mn, swap,
                           err.data_ptr(), a_tmem)
    assert rc == 0, rc
    assert int(err.item()) == 0, "mbarrier wait timed out"
    return D.cpu()


CASES = [(128, 64, 128, 0, 0), (128, 128, 64, 0, 1), (128, 64, 128, 1, 0), (128, 128, 128, 1, 1),
         (128, 256, 128, 0, 0), (128, 64, 64, 1, 1), (128, 128, 64, 0, 0)]


@pytest.mark.parametrize("M,N,Kd,a_mn,b_mn", CASES)
def test_mma_m128(M, N, Kd, a_mn, b_mn):
    g = torch.Generator().manual_seed(M * 7 + N + Kd + a_mn * 3 + b_mn)
    A = torch.randn(M, Kd, generator=g).to(torch.bfloat16)
    B = torch.randn(N, Kd, generator=g).to(torch.bfloat16)
    ref = A.float() @ B.float().T
    results = {}
    for swap in ((0, 1) if (a_mn or b_mn) else (0,)):
        D = run(A.cuda(), B.cuda(), M, N, Kd, a_mn, b_mn, swap)
        err = float((D[:M] - ref).abs().max() / ref.abs().max())
        results[swap] = err
    print("mma M=%d N=%d K=%d a_mn=%d b_mn=%d: err by lbo/sbo variant %s" % (M, N, Kd, a_mn, b_mn,
                                                                            results))
    assert results[0] < 1e-3, results


@pytest.mark.parametrize("N,Kd,b_mn", [(64, 128, 0), (128, 64, 1), (64, 64, 0), (128, 128, 1)])
def test_mma_a_from_tmem(N, Kd, b_mn):
    """A (128 x K, K-major) taken from TMEM as packed bf16 pairs, B from shared memory."""
    g = torch.Generator().manual_seed(900 + N + Kd + b_mn)
    A = torch.randn(128, Kd, generator=g).to(torch.bfloat16)
    B = torch.randn(N, Kd, generator=g).to(torch.bfloat16)
    ref = A.float() @ B.float().T
    D = run(A.cuda(), B.cuda(), 128, N, Kd, 0, b_mn, 0, a_tmem=1)
    err = float((D - ref).abs().max() / ref.abs().max())
    print("mma with A in TMEM, N=%d K=%d b_mn=%d: err %.2e" % (N, Kd, b_mn, err))
    assert err < 1e-3, err


def test_tmem_layout_m64():
    """Locates every element of a 64 x N accumulator in the TMEM dump."""
    M, N, Kd = 64, 64, 64
    A = torch.eye(M, Kd).to(torch.bfloat16)
    rows = (torch.arange(Kd).float() + 1).repeat(N, 1).to(torch.bfloat16)     # D[m][n] = m + 1
    cols = (torch.arange(N).float() + 1)[:, None].repeat(1, Kd).to(torch.bfloat16)  # D[m][n] = n + 1
    Dr = run(A.cuda(), rows.cuda(), M, N, Kd, 0, 0).numpy()
    Dc = run(A.cuda(), cols.cuda(), M, N, Kd, 0, 0).numpy()
    where = {}
    for lane in range(128):
        for c in range(N):
            r, n = Dr[lane, c], Dc[lane, c]
            if np.isfinite(r) and r >= 1 and abs(r - round(r)) == 0 and np.isfinite(n) and n >= 1:
                where.setdefault((int(r) - 1, int(n) - 1), []).append((lane, c))
    found = sum(1 for m in range(M) for n in range(N) if (m, n) in where)
    sample = {k: where.get(k) for k in [(0, 0), (1, 0), (15, 0), (16, 0), (31, 5), (32, 0),
                                        (48, 63), (63, 63), (0, 32)]}
    print("M=64 layout: %d/%d elements located; samples %s" % (found, M * N, sample))
    hyp = all(where.get((m, n)) and (m // 16 * 32 + m % 16, n) in where[(m, n)]
              for m in range(M) for n in range(N))
    print("hypothesis lane = 32*(m//16) + m%%16, column = n: %s" % hyp)
    assert found == M * N

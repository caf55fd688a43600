"""The tensor-core operand layouts and MMA-issue helpers of the chunk kernel,
each checked alone: operands written in the kernel's swizzled shared-memory
layouts, one MMA per layout form, compared with a host GEMM of the same
bf16-rounded operands."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "umma_layout_check.cu")
INC = os.path.join(os.path.dirname(HERE), "chunk_delta_rule_b200", "csrc")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("umma") / "libumma_check.so")
    subprocess.check_call(["nvcc", "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC", "-shared", "-I", INC, "-o", out, SRC])
    l = ctypes.CDLL(out)
    l.umma_layout_check.argtypes = [ctypes.c_int] + [ctypes.c_void_p] * 5
    l.umma_layout_check.restype = ctypes.c_int
    return l


@pytest.mark.parametrize("mode,M,N,K,wrapB", [
    (0, 128, 64, 128, False),   # [K;Q] K^T
    (1, 128, 64, 64, False),    # K^T Tc^T   (A MN-major, atoms 16 KB apart)
    (2, 128, 64, 64, False),    # V^T Eb^T   (A MN-major, atoms 8 KB apart)
    (3, 128, 64, 128, False),   # S W^T      (B MN-major)
    (4, 128, 128, 128, True),   # (D X)^T K  (B MN-major, K rows re-read for hi|lo)
    (5, 128, 64, 128, True),    # X^T P^T accumulated onto an initial D
    (6, 128, 64, 64, False),    # tf32: X (TMEM) P^T, P K-major fp32
    (7, 128, 128, 64, False),   # tf32: X (TMEM) (D K), (D K)^T K-major fp32, N = 128
    (8, 128, 64, 128, False),   # bf16: S (TMEM, packed pairs) Qh^T, Qh K-major
    (9, 128, 64, 128, False),   # bf16: S (TMEM, packed pairs) (-W)^T, W MN-major
])
def test_mma_layout(lib, mode, M, N, K, wrapB):
    g = torch.Generator().manual_seed(mode)
    A = torch.randn(M, K, generator=g)
    B = torch.randn(N, K, generator=g)
    if wrapB:
        B[:, 64:] = B[:, :64]
    D0 = torch.randn(M, N, generator=g) if mode == 5 else torch.zeros(M, N)
    Ad, Bd, D0d = A.cuda(), B.cuda(), D0.cuda()
    D = torch.full((M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.umma_layout_check(mode, Ad.data_ptr(), Bd.data_ptr(), D0d.data_ptr(), D.data_ptr(),
                               status.data_ptr())
    assert rc == 0 and int(status.item()) == 0
    if mode in (6, 7):
        # tf32 keeps 10 explicit mantissa bits of each operand
        want = A.double() @ B.double().T
        tol = 2e-3 * (A.abs() @ B.abs().T).double().max().item()
    else:
        Ab = A.bfloat16().double()
        Bb = B.bfloat16().double()
        want = Ab @ Bb.T + (D0.double() if mode == 5 else 0)
        tol = 1e-3 * max(1.0, want.abs().max().item())
    got = D.double().cpu()
    err = (got - want).abs().max().item()
    assert err < tol, f"mode {mode}: max err {err}"

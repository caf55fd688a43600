"""The chunk kernel rounds fp32 to tf32 with two integer operations; this checks
it against the hardware conversion (cvt.rna.tf32.f32) bit for bit on non-NaN
inputs."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "tf32_round_check.cu")
INC = os.path.join(os.path.dirname(HERE), "chunk_delta_rule_b200", "csrc")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("tf32") / "libtf32_check.so")
    subprocess.check_call(["nvcc", "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC", "-shared", "-I", INC, "-o", out, SRC])
    l = ctypes.CDLL(out)
    l.tf32_round_check.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    l.tf32_round_check.restype = ctypes.c_int
    return l


def run(lib, bits: torch.Tensor):
    bits = bits.to(torch.int64).to(torch.int32).cuda()   # same 32 bits, any sign
    mism = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    assert lib.tf32_round_check(bits.data_ptr(), mism.data_ptr(), first.data_ptr(), bits.numel()) == 0
    return int(mism.item()), int(first.item()) & 0xffffffff


def test_every_pattern_around_rounding_boundaries(lib):
    # all 2^13 low-bit patterns (ties included) for a spread of sign/exponent/high
    # mantissa prefixes, zeros, denormals, the largest finite values, infinities, NaNs
    patterns = torch.tensor([0x00000000, 0x00002000, 0x007fe000, 0x3f800000, 0x3f9ab000, 0x7f7fe000,
                             0x7f800000, 0x80000000, 0x80246000, 0xbf800000, 0xff7fe000, 0xff800000,
                             0x4b7fe000, 0x0c0de000, 0x9abcd000], dtype=torch.int64)
    prefixes = patterns >> 13
    low = torch.arange(1 << 13, dtype=torch.int64)
    bits = ((prefixes[:, None] << 13) | low[None, :]).reshape(-1)
    assert run(lib, bits) == (0, 0xffffffff)


def test_random_patterns(lib):
    g = torch.Generator().manual_seed(7)
    bits = torch.randint(0, 1 << 32, (1 << 22,), generator=g, dtype=torch.int64)
    assert run(lib, bits) == (0, 0xffffffff)

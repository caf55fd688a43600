"""The tensor-core kernel's failure path, made to run without faulting the GPU: one
of its bounded waits is on a barrier phase that nothing completes (the stall test
entry), with a per-wait limit of a few microseconds.  The kernel must latch
COMBA_ETIMEOUT, drain what it has issued, release its tensor memory and return;
the device then runs the next, normal call correctly."""
import ctypes

import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, make_chunk_inputs
from tests.gpu_util import TOL_BF16, assert_close, to_dev

pytestmark = pytest.mark.gpu

COMBA_ETIMEOUT = -4
p = lambda t: ctypes.c_void_p(0 if t is None else t.data_ptr())


def _inputs():
    cfg = CONFIGS["layer340m_bf16"].replace(B=1, H=1, T=256, s0_std=0.02)
    return make_chunk_inputs(cfg, seed=909)


@pytest.mark.parametrize("timeout_ns", [2000, 1_000_000])
def test_wait_that_runs_out_latches_timeout_and_the_device_recovers(timeout_ns):
    x = _inputs()
    xd = to_dev(x)
    lib = cdr.library()
    assert lib.comba_get_last_error() == 0
    out = torch.zeros((1, 256, 1, 128), dtype=torch.bfloat16, device="cuda")
    Sf = torch.zeros((1, 1, 128, 128), dtype=torch.float32, device="cuda")
    st = lib.comba_chunk_fwd_stall_test(p(xd["q"]), p(xd["k"]), p(xd["v"]), p(xd["log_alpha"]), p(xd["beta"]),
                                        p(xd["d"]), p(xd["S0"]), p(out), p(Sf), 1, 256, 1, 128, 128, 64,
                                        ctypes.c_ulonglong(timeout_ns), 1,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0                     # launched
    torch.cuda.synchronize()           # the kernel returned
    assert lib.comba_get_last_error() == COMBA_ETIMEOUT
    assert lib.comba_get_last_error() == 0   # read and cleared
    # the same problem with the default limit, on the same device and process
    o, S = cdr.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"], xd["S0"], chunk=64)
    torch.cuda.synchronize()
    assert lib.comba_get_last_error() == 0
    ro, rS = oracle.recurrence(**x)
    assert_close("out", o.double().cpu().numpy(), ro, TOL_BF16)
    assert_close("S_final", S.double().cpu().numpy(), rS, TOL_BF16)


def test_generous_limit_changes_nothing():
    x = _inputs()
    xd = to_dev(x)
    lib = cdr.library()
    out = torch.empty((1, 256, 1, 128), dtype=torch.bfloat16, device="cuda")
    Sf = torch.empty((1, 1, 128, 128), dtype=torch.float32, device="cuda")
    st = lib.comba_chunk_fwd_stall_test(p(xd["q"]), p(xd["k"]), p(xd["v"]), p(xd["log_alpha"]), p(xd["beta"]),
                                        p(xd["d"]), p(xd["S0"]), p(out), p(Sf), 1, 256, 1, 128, 128, 64,
                                        ctypes.c_ulonglong(2_000_000_000), 0,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    o, S = cdr.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"], xd["S0"], chunk=64,
                         segment=False)
    torch.cuda.synchronize()
    assert lib.comba_get_last_error() == 0
    assert torch.equal(out, o) and torch.equal(Sf, S)

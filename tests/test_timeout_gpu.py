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


def test_backward_state_pass_wait_that_runs_out_and_the_device_recovers():
    """The same for the backward's tensor-core state passes (bf16, dk = dv = 128)."""
    from comba_workloads import make_cotangents
    cfg = CONFIGS["layer340m_bf16"].replace(B=1, H=2, T=200, dk=128, dv=128, s0_std=0.1)
    x = make_chunk_inputs(cfg, seed=919)
    cot = make_cotangents(cfg, seed=929)
    xd = {k: (None if v is None else v.cuda()) for k, v in {**x, **cot}.items()}
    lib = cdr.library()
    assert lib.comba_get_last_error() == 0
    B, T, H = 1, 200, 2
    f32 = lambda *s: torch.zeros(*s, dtype=torch.float32, device="cuda")
    g = dict(dq=f32(B, T, H, 128), dk=f32(B, T, H, 128), dv=f32(B, T, H, 128), dla=f32(B, T, H),
             dbt=f32(B, T, H), dd=f32(H), dS0=f32(B, H, 128, 128))
    need = int(lib.comba_chunk_bwd_workspace_size(B, T, H, 128, 128))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = lib.comba_chunk_bwd_stall_test(
        p(xd["q"]), p(xd["k"]), p(xd["v"]), p(xd["log_alpha"]), p(xd["beta"]), p(xd["d"]), p(xd["S0"]),
        p(xd["dout"]), p(xd["dS_final"]), p(g["dq"]), p(g["dk"]), p(g["dv"]), p(g["dla"]), p(g["dbt"]),
        p(g["dd"]), p(g["dS0"]), B, T, H, 128, 128, 0, p(ws), ctypes.c_size_t(need), ctypes.c_ulonglong(50_000),
        1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert lib.comba_get_last_error() == COMBA_ETIMEOUT
    assert lib.comba_get_last_error() == 0
    # a normal backward on the same device and process
    res = cdr.chunk_bwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"], xd["dout"],
                        S0=xd["S0"], dS_final=xd["dS_final"])
    torch.cuda.synchronize()
    assert lib.comba_get_last_error() == 0
    ref = oracle.recurrence_bwd_np(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["d"], x["S0"],
                                   cot["dout"], cot["dS_final"])
    for n in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        assert_close(n, res[n].double().cpu().numpy(), ref[n], dict(rel=5e-3, abs=None))

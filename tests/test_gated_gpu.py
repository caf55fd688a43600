"""comba_chunk_fwd_gated (q/k L2 normalisation and gates formed inside the kernel
from raw projections) against the oracle's gate_inputs followed by its recurrence."""
import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, make_gated_inputs
from tests.gpu_util import TOL_BF16, assert_close

pytestmark = pytest.mark.gpu

EPS = 1e-6


def run_and_check(x, chunk):
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    out, S = cdr.chunk_fwd_gated(xd["q_raw"], xd["k_raw"], xd["v"], xd["a_raw"], xd["b_raw"], xd["A_log"],
                                 xd["dt_bias"], xd["d"], xd["S0"], chunk=chunk, norm_eps=EPS)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    q, k, la, be = oracle.gate_inputs(x["q_raw"], x["k_raw"], x["a_raw"], x["b_raw"], x["A_log"],
                                      x["dt_bias"], eps=EPS)
    ro, rS = oracle.recurrence(q, k, x["v"], la, be, x["d"], x["S0"])
    assert_close("out", out.double().cpu().numpy(), ro, TOL_BF16)
    assert_close("S_final", S.double().cpu().numpy(), rS, TOL_BF16)
    return la


@pytest.mark.parametrize("B,H,T,dk,dv,chunk", [
    (2, 3, 200, 128, 128, 64),     # tensor-core kernel, ragged tail
    (1, 2, 64, 128, 128, 64),
    (2, 2, 77, 64, 32, 32),        # general kernel
    (1, 2, 50, 32, 64, 16),
])
def test_gated_against_oracle(B, H, T, dk, dv, chunk):
    cfg = CONFIGS["layer340m_bf16"].replace(B=B, H=H, T=T, dk=dk, dv=dv, chunk=chunk, s0_std=0.05)
    run_and_check(make_gated_inputs(cfg, seed=321 + T + dk, dt_bias_std=0.5), chunk)


def test_gated_strong_decay_takes_the_exact_path():
    # A_log = ln 3: log-decays of about -2 per token, so chunks total well below -80
    cfg = CONFIGS["layer340m_bf16"].replace(B=1, H=2, T=192, s0_std=0.5)
    x = make_gated_inputs(cfg, seed=99)
    x["A_log"] = torch.full((2,), 1.0986123, dtype=torch.float32)
    la = run_and_check(x, 64)
    assert la.reshape(1, 3, 64, 2).sum(2).max() < -80


def test_gated_zero_length_copies_state():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=2, T=1, s0_std=0.05)
    x = make_gated_inputs(cfg, seed=5)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    empty = lambda t: t[:, :0].contiguous()
    out, S = cdr.chunk_fwd_gated(empty(xd["q_raw"]), empty(xd["k_raw"]), empty(xd["v"]), empty(xd["a_raw"]),
                                 empty(xd["b_raw"]), xd["A_log"], None, xd["d"], xd["S0"], chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(S, xd["S0"])


def test_gated_full_size_sampled_chains():
    # the benchmark's raw-projection workload (1.3B layer), run whole; two (b, h) chains
    # against the oracle
    cfg = CONFIGS["layer1p3b_bf16"]
    x = make_gated_inputs(cfg)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    out, S = cdr.chunk_fwd_gated(xd["q_raw"], xd["k_raw"], xd["v"], xd["a_raw"], xd["b_raw"], xd["A_log"],
                                 xd["dt_bias"], xd["d"], xd["S0"], chunk=cfg.chunk, norm_eps=EPS)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    q, k, la, be = oracle.gate_inputs(x["q_raw"], x["k_raw"], x["a_raw"], x["b_raw"], x["A_log"],
                                      x["dt_bias"], eps=EPS)
    for b, h in [(0, 0), (7, 15)]:
        sl = lambda a: a[b:b + 1, :, h:h + 1]
        ro, rS = oracle.recurrence(sl(q), sl(k), sl(x["v"]), sl(la), sl(be), x["d"][h:h + 1],
                                   x["S0"][b:b + 1, h:h + 1])
        assert_close(f"out {b},{h}", out[b, :, h].double().cpu().numpy(), ro[0, :, 0], TOL_BF16)
        assert_close(f"S_final {b},{h}", S[b, h].double().cpu().numpy(), rS[0, 0], TOL_BF16)

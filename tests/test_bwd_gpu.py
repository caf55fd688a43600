"""comba_chunk_bwd (the chunk backward) against the float64 oracle's gradients of the
token recurrence, element by element on seeded inputs: ragged tails, every
supported dk x dv pair, bf16 and fp32 inputs, strong decay, T = 0 and 1, and
sampled chains of the full 1.3B-layer shape."""
import numpy as np
import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, make_chunk_inputs, make_cotangents
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu

# fp32 arithmetic over 32-token chunks on the exact (widened) input values: every
# gradient within rel-L2 1e-4 of the float64 gradients (the forward's fp32 bar is
# 1e-5; the backward chains two triangular solves and the state passes per chunk,
# about an order of magnitude more rounding steps per result).
TOL_BWD = dict(rel=1e-4, abs=None)
# bf16 inputs with dk = dv = 128 take the tensor-core form of the state passes and
# of the five state contractions of the grads kernel, with the states, W, X and dR
# rounded to bf16 as MMA operands: every gradient, dS0 included, is held to the
# bf16 workload bound of the forward, rel-L2 5e-3.
TOL_BWD_TC = dict(rel=5e-3, abs=None)


def tol_for(dtype, dk, dv):
    return TOL_BWD_TC if (dtype == "bf16" and dk == 128 and dv == 128) else TOL_BWD
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dd", "dS0")


def run(x, cot, need_dd=True, need_dS0=True):
    xd = {k: (None if v is None else v.cuda()) for k, v in {**x, **cot}.items()}
    g = cdr.chunk_bwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"], xd["dout"],
                      S0=xd["S0"], dS_final=xd["dS_final"], need_dd=need_dd, need_dS0=need_dS0)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    return {k: (None if v is None else v.double().cpu().numpy()) for k, v in g.items()}


def check(x, cot, g, tol=TOL_BWD, names=GRADS):
    ref = oracle.recurrence_bwd_np(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["d"], x["S0"],
                                   cot["dout"], cot["dS_final"])
    for n in names:
        assert_close(n, g[n], ref[n], tol)


@pytest.mark.parametrize("B,H,T,dk,dv,dtype", [
    (2, 2, 100, 64, 64, "fp32"),      # 3 chunks + a 4-token tail
    (1, 3, 257, 128, 128, "fp32"),
    (2, 2, 96, 128, 128, "bf16"),      # whole chunks
    (1, 2, 77, 32, 128, "fp32"),
    (1, 2, 45, 128, 32, "bf16"),
    (2, 1, 64, 64, 32, "fp32"),
    (1, 2, 33, 32, 64, "bf16"),
])
def test_bwd_against_oracle(B, H, T, dk, dv, dtype):
    cfg = CONFIGS["layer340m_bf16"].replace(B=B, H=H, T=T, dk=dk, dv=dv, dtype=dtype, s0_std=0.1,
                                            decay="mamba")
    x = make_chunk_inputs(cfg, seed=1000 + T + dk)
    cot = make_cotangents(cfg, seed=2000 + T)
    check(x, cot, run(x, cot), tol=tol_for(dtype, dk, dv))


def test_bwd_strong_decay_and_no_state_cotangent():
    cfg = CONFIGS["layer340m_bf16"].replace(B=1, H=2, T=130, dk=64, dv=64, dtype="fp32", s0_std=0.5,
                                            decay="uniform", decay_lo=-2.5, decay_hi=-1.5)
    x = make_chunk_inputs(cfg, seed=7)
    cot = make_cotangents(cfg, seed=8, dS_std=0.0)
    check(x, cot, run(x, cot))


def test_bwd_zero_initial_state_and_optional_outputs():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=2, T=40, dk=64, dv=64, dtype="bf16", s0_std=0.0)
    x = make_chunk_inputs(cfg, seed=11)
    assert x["S0"] is None
    cot = make_cotangents(cfg, seed=12)
    g = run(x, cot, need_dd=False, need_dS0=False)
    assert g["dd"] is None and g["dS0"] is None
    check(x, cot, g, names=("dq", "dk", "dv", "dlog_alpha", "dbeta"))


def test_bwd_single_token_and_empty_sequence():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=3, T=1, dk=32, dv=32, dtype="fp32", s0_std=0.3)
    x = make_chunk_inputs(cfg, seed=13)
    cot = make_cotangents(cfg, seed=14)
    check(x, cot, run(x, cot))
    empty = {k: (v[:, :0].contiguous() if (v is not None and v.dim() >= 3 and k not in ("S0",)) else v)
             for k, v in x.items()}
    cot0 = {"dout": cot["dout"][:, :0].contiguous(), "dS_final": cot["dS_final"]}
    g = run(empty, cot0)
    assert np.array_equal(g["dS0"], cot["dS_final"].double().numpy())
    assert np.array_equal(g["dd"], np.zeros(3))


@pytest.mark.parametrize("T", [1, 32, 33, 45, 257])
def test_bwd_tensor_core_form_edge_lengths(T):
    """bf16, dk = dv = 128 (the tensor-core form): one token (the forward walk has no
    update step), exactly one chunk, a ragged second chunk, and longer ragged tails;
    with and without an initial state and a state cotangent."""
    for s0, ds in ((0.0, 1.0), (0.2, 0.0), (0.2, 1.0)):
        cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=2, T=T, dk=128, dv=128, dtype="bf16", s0_std=s0,
                                                decay="mamba")
        x = make_chunk_inputs(cfg, seed=300 + T)
        cot = make_cotangents(cfg, seed=400 + T, dS_std=ds)
        check(x, cot, run(x, cot), tol=TOL_BWD_TC)


def test_bwd_tensor_core_form_empty_sequence():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=3, T=1, dk=128, dv=128, dtype="bf16", s0_std=0.3)
    x = make_chunk_inputs(cfg, seed=13)
    cot = make_cotangents(cfg, seed=14)
    empty = {k: (v[:, :0].contiguous() if (v is not None and v.dim() >= 3 and k not in ("S0",)) else v)
             for k, v in x.items()}
    cot0 = {"dout": cot["dout"][:, :0].contiguous(), "dS_final": cot["dS_final"]}
    g = run(empty, cot0)
    assert np.array_equal(g["dS0"], cot["dS_final"].double().numpy())
    assert np.array_equal(g["dd"], np.zeros(3))


def test_bwd_full_layer_sampled_chains():
    """The 1.3B layer (B=8, T=4096, H=16, dk=dv=128, bf16): every output of three
    sampled (b, h) chains against the oracle run on those chains alone (chains are
    independent; dd sums over all of them and is covered above)."""
    cfg = CONFIGS["layer1p3b_bf16"]
    x = make_chunk_inputs(cfg)
    cot = make_cotangents(cfg)
    g = run(x, cot)
    for (b, h) in [(0, 0), (3, 7), (7, 15)]:
        xs = {k: (None if v is None else (v[b:b + 1, :, h:h + 1] if v.dim() >= 3 and k != "S0" else v))
              for k, v in x.items()}
        xs["d"] = x["d"][h:h + 1]
        xs["S0"] = None if x["S0"] is None else x["S0"][b:b + 1, h:h + 1]
        cs = {"dout": cot["dout"][b:b + 1, :, h:h + 1], "dS_final": cot["dS_final"][b:b + 1, h:h + 1]}
        ref = oracle.recurrence_bwd_np(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], xs["d"],
                                       xs["S0"], cs["dout"], cs["dS_final"])
        for n in ("dq", "dk", "dv"):
            assert_close(f"{n}[{b},{h}]", g[n][b:b + 1, :, h:h + 1], ref[n], TOL_BWD_TC)
        for n in ("dlog_alpha", "dbeta"):
            assert_close(f"{n}[{b},{h}]", g[n][b:b + 1, :, h:h + 1], ref[n], TOL_BWD_TC)
        assert_close(f"dS0[{b},{h}]", g["dS0"][b:b + 1, h:h + 1], ref["dS0"], TOL_BWD_TC)


def test_bwd_deterministic():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=2, T=150, dk=128, dv=128, dtype="bf16", s0_std=0.1)
    x = make_chunk_inputs(cfg, seed=21)
    cot = make_cotangents(cfg, seed=22)
    g1, g2 = run(x, cot), run(x, cot)
    for n in GRADS:
        assert np.array_equal(g1[n], g2[n]), n

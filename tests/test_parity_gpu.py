"""CUDA path against the float64 oracle, element by element, on seeded inputs.

Small cases span several chunks and a ragged tail and are compared in full;
the full-size workloads run in the launch configuration the benchmark times
and are compared on sampled (b, h) chains, which the oracle computes one by
one (chains are independent)."""
import numpy as np
import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, make_chunk_inputs
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, chain_slice, gpu_chunk, to_dev)

pytestmark = pytest.mark.gpu


def test_tiny_fp32_workload():
    cfg = CONFIGS["tiny_fp32"]
    x = make_chunk_inputs(cfg)
    o, S = gpu_chunk(x, cfg.chunk)
    ro, rS = oracle.recurrence(**x)
    assert_close("out", o, ro, TOL_F32)
    assert_close("S_final", S, rS, TOL_F32)


SMALL = [
    # (B, H, T, dk, dv, chunk, dtype)
    (2, 3, 200, 128, 128, 64, "bf16"),    # tensor-core shape, ragged tail (3 chunks + 8)
    (1, 2, 64, 128, 128, 64, "bf16"),     # exactly one chunk
    (1, 1, 1, 128, 128, 64, "bf16"),      # single token
    (2, 2, 63, 128, 128, 64, "bf16"),     # T < chunk
    (1, 2, 77, 64, 32, 32, "bf16"),
    (2, 1, 50, 32, 128, 16, "bf16"),
    (1, 2, 130, 16, 48, 64, "bf16"),
    (1, 2, 200, 128, 128, 64, "fp32"),
    (2, 1, 91, 64, 64, 16, "fp32"),
    (1, 3, 33, 48, 80, 32, "fp32"),
]


@pytest.mark.parametrize("B,H,T,dk,dv,chunk,dt", SMALL)
def test_small_shapes_against_oracle(B, H, T, dk, dv, chunk, dt):
    base = CONFIGS["layer340m_bf16"] if dt == "bf16" else CONFIGS["tiny_fp32"]
    cfg = base.replace(B=B, H=H, T=T, dk=dk, dv=dv, chunk=chunk, s0_std=0.02)
    x = make_chunk_inputs(cfg, seed=1000 + T + dk)
    o, S = gpu_chunk(x, chunk)
    ro, rS = oracle.recurrence(**x)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    assert_close("out", o, ro, tol)
    assert_close("S_final", S, rS, tol)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_strong_decay_mixes_exact_and_factored_chunks(dt):
    # log a ~ U(-2, -0.5): a chunk's total log-decay spreads around -80 (about -89 to
    # -75 for this seed, half of the chunks on either side), so chunks take both the
    # factored e^{g_r} e^{-g_s} form and the exact per-entry exponent, and in-chunk
    # decays reach the limits of fp32.
    base = CONFIGS["layer340m_bf16"] if dt == "bf16" else CONFIGS["tiny_fp32"]
    cfg = base.replace(B=2, H=2, T=320, dk=128, dv=128, chunk=64, decay="uniform",
                       decay_lo=-2.0, decay_hi=-0.5, s0_std=0.5)
    x = make_chunk_inputs(cfg, seed=4242)
    g = x["log_alpha"].double().reshape(2, 5, 64, 2).sum(2)
    assert bool((g > -80).any()) and bool((g <= -80).any())
    o, S = gpu_chunk(x, 64)
    ro, rS = oracle.recurrence(**x)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    assert_close("out", o, ro, tol)
    assert_close("S_final", S, rS, tol)


@pytest.mark.parametrize("with_s0,in_place", [(False, False), (True, False), (True, True)])
def test_segmented_long_sequence_matches_oracle_and_unsegmented(with_s0, in_place):
    # Two chains of 4096 tokens leave most of the GPU idle, so the library cuts each
    # chain into segments joined by their state transitions (comba_chunk_fwd_ws).
    cfg = CONFIGS["layer340m_bf16"].replace(B=1, H=2, T=4096, s0_std=0.05 if with_s0 else 0.0)
    x = make_chunk_inputs(cfg, seed=777)
    if not with_s0:
        x["S0"] = None
    lib = cdr.library()
    assert lib.comba_chunk_fwd_workspace_size(1, 4096, 2, 128, 128, 64) > 0
    xd = to_dev(x)
    args = {k: xd[k] for k in ("q", "k", "v", "log_alpha", "beta", "d")}
    S0 = xd["S0"]
    o_plain, S_plain = cdr.chunk_fwd(**args, S0=S0, chunk=64, segment=False)
    if in_place:
        Sc = S0.clone()
        o_seg, S_seg = cdr.chunk_fwd(**args, S0=Sc, S_final=Sc, chunk=64)
    else:
        o_seg, S_seg = cdr.chunk_fwd(**args, S0=S0, chunk=64)
    torch.cuda.synchronize()
    assert cdr.library().comba_get_last_error() == 0
    ro, rS = oracle.recurrence(**x)
    np64 = lambda t: t.double().cpu().numpy()
    assert_close("out (segmented)", np64(o_seg), ro, TOL_BF16)
    assert_close("S_final (segmented)", np64(S_seg), rS, TOL_BF16)
    assert_close("out (unsegmented)", np64(o_plain), ro, TOL_BF16)
    # the two groupings of the same computation agree to well inside the bf16 bound
    d_o = (o_seg.float() - o_plain.float()).norm() / o_plain.float().norm()
    d_S = (S_seg - S_plain).norm() / S_plain.norm()
    assert float(d_o) < 2e-3 and float(d_S) < 2e-3


@pytest.mark.parametrize("name,chains", [
    ("layer340m_bf16", [(0, 0), (3, 5), (7, 7)]),
    ("layer1p3b_bf16", [(0, 0), (4, 9), (7, 15)]),
    ("long64k_bf16", [(0, 3), (0, 14)]),
])
def test_full_size_workloads_sampled_chains(name, chains):
    cfg = CONFIGS[name]
    x = make_chunk_inputs(cfg)
    xd = to_dev(x)
    out, S = cdr.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"],
                           xd["S0"], chunk=cfg.chunk)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(S).all()
    for b, h in chains:
        xs = chain_slice(x, b, h)
        ro, rS = oracle.recurrence(**xs)
        assert_close(f"out[{b},:,{h}]", out[b, :, h].double().cpu().numpy(), ro[0, :, 0], TOL_BF16)
        assert_close(f"S_final[{b},{h}]", S[b, h].double().cpu().numpy(), rS[0, 0], TOL_BF16)


def test_zero_length_sequence_copies_state():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=2, T=0)
    x = to_dev(make_chunk_inputs(cfg.replace(T=1)))
    q = x["q"][:, :0]
    g = x["log_alpha"][:, :0].contiguous()
    out, S = cdr.chunk_fwd(q.contiguous(), q.contiguous(), x["v"][:, :0].contiguous(), g, g,
                           x["d"], x["S0"], chunk=64)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(S, x["S0"])
    _, Sz = cdr.chunk_fwd(q.contiguous(), q.contiguous(), x["v"][:, :0].contiguous(), g, g,
                          x["d"], None, chunk=64)
    torch.cuda.synchronize()
    assert torch.count_nonzero(Sz) == 0


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_state_carry_split_equals_one_call(dt):
    """Two calls with S_final -> S0 (in place) equal one call over the whole
    sequence when the split falls on a chunk boundary."""
    base = CONFIGS["layer340m_bf16"] if dt == "bf16" else CONFIGS["tiny_fp32"]
    cfg = base.replace(B=2, H=2, T=256, dk=128, dv=128, chunk=64, s0_std=0.02)
    x = to_dev(make_chunk_inputs(cfg, seed=77))
    o_full, S_full = cdr.chunk_fwd(**{k: x[k] for k in ("q", "k", "v", "log_alpha", "beta", "d", "S0")}, chunk=64)
    S = x["S0"].clone()
    outs = []
    for a, b in ((0, 128), (128, 256)):
        sl = {k: x[k][:, a:b].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        o, _ = cdr.chunk_fwd(**sl, d=x["d"], S0=S, S_final=S, chunk=64)
        outs.append(o)
    torch.cuda.synchronize()
    o2 = torch.cat(outs, dim=1)
    tol = 1e-6 if dt == "fp32" else 1e-2
    assert (o2.float() - o_full.float()).abs().max().item() <= tol
    assert (S - S_full).abs().max().item() <= tol


def test_output_is_affine_in_d_and_linear_in_v_S0():
    cfg = CONFIGS["tiny_fp32"].replace(B=1, H=2, T=96, dk=32, dv=32, chunk=32, s0_std=0.1)
    x = to_dev(make_chunk_inputs(cfg, seed=5))
    args = {k: x[k] for k in ("q", "k", "v", "log_alpha", "beta", "d", "S0")}
    o, S = cdr.chunk_fwd(**args, chunk=32)
    o2, S2 = cdr.chunk_fwd(**dict(args, v=-3.0 * x["v"], S0=-3.0 * x["S0"]), chunk=32)
    torch.cuda.synchronize()
    assert torch.allclose(o2, -3.0 * o, rtol=1e-5, atol=1e-5)
    assert torch.allclose(S2, -3.0 * S, rtol=1e-5, atol=1e-5)
    z = dict(args, d=torch.zeros_like(x["d"]))
    o0, Sz = cdr.chunk_fwd(**z, chunk=32)
    okk, _ = cdr.chunk_fwd(**dict(z, q=x["k"]), chunk=32)
    torch.cuda.synchronize()
    want = o0 - x["d"][None, None, :, None] * okk
    assert torch.allclose(o, want, rtol=1e-4, atol=1e-5)
    assert torch.allclose(Sz, S, rtol=1e-6, atol=1e-6)


def test_outputs_stay_inside_their_buffers():
    """Guard bands around out and S_final keep their canary values."""
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=3, T=150, s0_std=0.02)
    x = to_dev(make_chunk_inputs(cfg, seed=9))
    B, T, H, dv, dk = cfg.B, cfg.T, cfg.H, cfg.dv, cfg.dk
    pad = 4096
    ob = torch.full((pad + B * T * H * dv + pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    sb = torch.full((pad + B * H * dv * dk + pad,), -5.0, dtype=torch.float32, device="cuda")
    out = ob[pad:pad + B * T * H * dv].view(B, T, H, dv)
    Sf = sb[pad:pad + B * H * dv * dk].view(B, H, dv, dk)
    cdr.chunk_fwd(**{k: x[k] for k in ("q", "k", "v", "log_alpha", "beta", "d", "S0")},
                  chunk=64, out=out, S_final=Sf)
    torch.cuda.synchronize()
    assert bool((ob[:pad] == 7.0).all()) and bool((ob[-pad:] == 7.0).all())
    assert bool((sb[:pad] == -5.0).all()) and bool((sb[-pad:] == -5.0).all())
    ro, rS = oracle.recurrence(**{k: (None if v is None else v.cpu()) for k, v in x.items()})
    assert_close("out", out.double().cpu().numpy(), ro, TOL_BF16)


def test_deterministic_across_calls():
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=4, T=256)
    x = to_dev(make_chunk_inputs(cfg, seed=3))
    args = {k: x[k] for k in ("q", "k", "v", "log_alpha", "beta", "d", "S0")}
    o1, S1 = cdr.chunk_fwd(**args, chunk=64)
    o2, S2 = cdr.chunk_fwd(**args, chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)

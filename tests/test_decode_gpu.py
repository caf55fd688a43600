"""comba_recurrent_step (decode) against the float64 oracle and against the chunk path."""
import numpy as np
import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, DECODE, decode_step_inputs, make_chunk_inputs, make_decode_state
from tests.gpu_util import TOL_BF16, assert_close, to_dev

pytestmark = pytest.mark.gpu


def test_decode_workload_512_steps_sampled_heads():
    """Full decode workload (B=256, H=32, 512 tokens, state resident and updated in
    place); the oracle follows a sample of (b, h) heads through all 512 steps."""
    cfg = DECODE
    st = make_decode_state(cfg)
    gen, scale = st["gen"], st["decay_scale"]
    d = st["d"].cuda()
    S = st["S"].cuda()
    heads = [(0, 0), (17, 5), (128, 31), (255, 16)]
    S_ref = np.stack([st["S"][b, h].double().numpy() for b, h in heads])[None]   # [1, n, dv, dk]
    d_ref = np.array([float(st["d"][h]) for _, h in heads])
    worst_o = []
    for t in range(cfg.steps):
        x = decode_step_inputs(gen, scale, cfg)
        xd = to_dev(x)
        o = cdr.recurrent_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], d, S)
        pick = lambda a: np.stack([a[b, h].double().numpy() for b, h in heads])[None, None]
        ro, S_ref_new = oracle.recurrence(pick(x["q"]), pick(x["k"]), pick(x["v"]),
                                          pick(x["log_alpha"]), pick(x["beta"]), d_ref, S_ref)
        S_ref = S_ref_new
        if t % 64 == 63 or t == 0:
            og = o.double().cpu().numpy()
            got = np.stack([og[b, h] for b, h in heads])
            worst_o.append(assert_close(f"out step {t}", got, ro[0, 0], TOL_BF16))
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    got_S = np.stack([S[b, h].double().cpu().numpy() for b, h in heads])
    assert_close("S after 512 steps", got_S, S_ref[0], TOL_BF16)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 128), (128, 48)])
def test_decode_steps_equal_chunk_forward(dk, dv):
    """T single-token steps equal one chunk-wise forward over the same T tokens."""
    cfg = CONFIGS["layer340m_bf16"].replace(B=3, H=2, T=100, dk=dk, dv=dv, s0_std=0.02)
    x = to_dev(make_chunk_inputs(cfg, seed=11))
    o_chunk, S_chunk = cdr.chunk_fwd(**{k: x[k] for k in ("q", "k", "v", "log_alpha", "beta", "d", "S0")}, chunk=64)
    S = x["S0"].clone()
    outs = []
    for t in range(cfg.T):
        outs.append(cdr.recurrent_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(),
                                       x["v"][:, t].contiguous(), x["log_alpha"][:, t].contiguous(),
                                       x["beta"][:, t].contiguous(), x["d"], S))
    torch.cuda.synchronize()
    o_step = torch.stack(outs, dim=1)
    ro, rS = oracle.recurrence(**{k: (None if v is None else v.cpu()) for k, v in x.items()})
    assert_close("step out", o_step.double().cpu().numpy(), ro, TOL_BF16)
    assert_close("step S", S.double().cpu().numpy(), rS, TOL_BF16)
    assert_close("chunk vs step out", o_chunk.double().cpu().numpy(), o_step.double().cpu().numpy(), TOL_BF16)

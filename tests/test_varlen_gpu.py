"""Packed variable-length sequences with q / k heads shared by groups of value
heads (comba_chunk_fwd_varlen) against the float64 oracle, sequence by sequence.

Each (sequence, value head) is an independent chain of the same recurrence, so
the expected values are the oracle's on each sequence alone, with q / k of value
head h taken from head h // (H // Hqk)."""
import numpy as np
import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, make_chunk_inputs
from tests.gpu_util import TOL_BF16, assert_close

pytestmark = pytest.mark.gpu


def packed_inputs(lengths, H, Hqk, dk, dv, seed, s0_std=0.05):
    """Packed inputs [total_T, heads, d] of len(lengths) sequences and cu_seqlens."""
    total = int(sum(lengths))
    base = CONFIGS["layer340m_bf16"].replace(B=1, T=max(total, 1), dk=dk, dv=dv, s0_std=0.0)
    xv = make_chunk_inputs(base.replace(H=H), seed=seed)
    xq = make_chunk_inputs(base.replace(H=Hqk), seed=seed + 1)
    gen = torch.Generator().manual_seed(seed + 2)
    N = len(lengths)
    S0 = (s0_std * torch.randn((N, H, dv, dk), generator=gen)).float() if s0_std > 0 else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    x = {
        "q": xq["q"][0, :total].contiguous(), "k": xq["k"][0, :total].contiguous(),
        "v": xv["v"][0, :total].contiguous(),
        "log_alpha": xv["log_alpha"][0, :total].contiguous(), "beta": xv["beta"][0, :total].contiguous(),
        "d": xv["d"], "S0": S0, "cu": cu,
    }
    return x


def oracle_packed(x, H, Hqk):
    """Expected out [total_T, H, dv] and S_final [N, H, dv, dk], one sequence at a time."""
    cu = x["cu"].numpy()
    G = H // Hqk
    heads = np.arange(H) // G
    total, dv = x["v"].shape[0], x["v"].shape[2]
    dk = x["q"].shape[2]
    N = len(cu) - 1
    out = np.zeros((total, H, dv))
    S = np.zeros((N, H, dv, dk))
    for n in range(N):
        s0, s1 = int(cu[n]), int(cu[n + 1])
        S0n = None if x["S0"] is None else x["S0"][n:n + 1]
        if s1 == s0:
            S[n] = 0.0 if S0n is None else S0n[0].double().numpy()
            continue
        sl = slice(s0, s1)
        o, Sn = oracle.recurrence(
            q=x["q"][sl][:, heads][None], k=x["k"][sl][:, heads][None], v=x["v"][sl][None],
            log_alpha=x["log_alpha"][sl][None], beta=x["beta"][sl][None], d=x["d"], S0=S0n)
        out[s0:s1] = o[0]
        S[n] = Sn[0]
    return out, S


def run_varlen(x, chunk):
    dev = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    out, S = cdr.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                  dev["d"], dev["cu"], S0=dev["S0"], chunk=chunk)
    torch.cuda.synchronize()
    return out, S


CASES = [
    # lengths, H, Hqk, dk, dv, chunk
    ([130, 0, 64, 1, 200, 63, 257], 4, 2, 128, 128, 64),   # tensor-core kernel, 2 v-heads per q/k head
    ([64, 128, 192], 2, 1, 128, 128, 64),                   # whole tiles only
    ([5, 77, 0, 300], 3, 3, 128, 128, 64),                   # plain per-head layout
    ([130, 0, 33, 200], 4, 1, 64, 32, 32),                   # general kernel, 4 v-heads per q/k head
    ([17, 64, 90], 2, 2, 32, 64, 16),
]


@pytest.mark.parametrize("lengths,H,Hqk,dk,dv,chunk", CASES)
def test_packed_sequences_against_oracle(lengths, H, Hqk, dk, dv, chunk):
    x = packed_inputs(lengths, H, Hqk, dk, dv, seed=9000 + sum(lengths) + H)
    out, S = run_varlen(x, chunk)
    assert cdr.get_last_error() == 0
    ro, rS = oracle_packed(x, H, Hqk)
    assert_close("out", out.double().cpu().numpy(), ro, TOL_BF16)
    assert_close("S_final", S.double().cpu().numpy(), rS, TOL_BF16)


@pytest.mark.parametrize("T", [256, 200])
def test_uniform_lengths_match_the_fixed_length_call(T):
    # N sequences of one length through the packed entry point are the [N, T, H, d]
    # problem of comba_chunk_fwd: same kernel arithmetic, same bits.
    N, H = 3, 4
    cfg = CONFIGS["layer340m_bf16"].replace(B=N, T=T, H=H, s0_std=0.05)
    x = make_chunk_inputs(cfg, seed=31337 + T)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    fo, fS = cdr.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"], xd["S0"],
                           chunk=64, segment=False)
    cu = torch.arange(0, (N + 1) * T, T, dtype=torch.int32, device="cuda")
    flat = lambda t: t.reshape(N * T, *t.shape[2:]).contiguous()
    vo, vS = cdr.chunk_fwd_varlen(flat(xd["q"]), flat(xd["k"]), flat(xd["v"]), flat(xd["log_alpha"]),
                                  flat(xd["beta"]), xd["d"], cu, S0=xd["S0"], chunk=64)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    assert torch.equal(vo.reshape(N, T, H, -1), fo)
    assert torch.equal(vS, fS)


def test_malformed_bounds_skip_the_sequence_and_report():
    # Sequence 1 ends past the packed tokens and sequence 2 runs backwards: both are
    # skipped (no outputs, S_final = S0) and COMBA_EINVAL is latched; sequence 0 is
    # computed as usual.
    x = packed_inputs([100, 100], 2, 2, 128, 128, seed=4711)
    x["cu"] = torch.tensor([0, 100, 300, 200], dtype=torch.int32)
    x["S0"] = torch.cat([x["S0"], x["S0"][:1]])
    dev = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    out = torch.full((200, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    cdr.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev["d"],
                         dev["cu"], S0=dev["S0"], chunk=64, out=out)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == -1
    assert cdr.get_last_error() == 0     # read and cleared
    y = dict(x)
    y["cu"] = torch.tensor([0, 100], dtype=torch.int32)
    y["S0"] = x["S0"][:1]
    ro, _ = oracle_packed(y, 2, 2)
    assert_close("out", out[:100].double().cpu().numpy(), ro[:100], TOL_BF16)
    assert bool((out[100:] == 7.0).all())


def test_bench_workload_sampled_chains():
    # The benchmark's packed workload (25 sequences, 16 value heads on one q / k head),
    # run whole; sampled (sequence, head) chains against the oracle one by one.
    from comba_workloads import VARLEN, make_varlen_inputs
    x = make_varlen_inputs(VARLEN)
    dev = {k: v.cuda() for k, v in x.items()}
    out, S = cdr.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                  dev["d"], dev["cu_seqlens"], S0=dev["S0"], chunk=VARLEN.chunk)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    cu = x["cu_seqlens"].tolist()
    lengths = np.diff(cu)
    G = VARLEN.H // VARLEN.Hqk
    for n, h in [(0, 0), (len(lengths) - 1, VARLEN.H - 1), (int(np.argmax(lengths)), 7),
                 (int(np.argmin(lengths)), 3)]:
        s0, s1 = cu[n], cu[n + 1]
        o, Sn = oracle.recurrence(
            q=x["q"][s0:s1, h // G][None, :, None], k=x["k"][s0:s1, h // G][None, :, None],
            v=x["v"][s0:s1, h][None, :, None], log_alpha=x["log_alpha"][s0:s1, h][None, :, None],
            beta=x["beta"][s0:s1, h][None, :, None], d=x["d"][h:h + 1], S0=x["S0"][n:n + 1, h:h + 1])
        assert_close(f"out seq {n} head {h}", out[s0:s1, h].double().cpu().numpy(), o[0, :, 0], TOL_BF16)
        assert_close(f"S_final seq {n} head {h}", S[n, h].double().cpu().numpy(), Sn[0, 0], TOL_BF16)


def test_mamba_form_prefill_then_grouped_decode():
    # Packed prefill of 3 sequences (4 value heads on one q / k head), then 5 decode
    # steps per sequence from its final state with the grouped step; the oracle runs
    # each sequence's prefill and decode tokens as one chain.
    lengths, H, Hqk, D, steps = [100, 37, 64], 4, 1, 128, 5
    x = packed_inputs(lengths, H, Hqk, D, D, seed=2024)
    _, S = run_varlen(x, 64)
    g = torch.Generator().manual_seed(99)
    N = len(lengths)
    dec = []
    for _ in range(steps):
        qk = torch.nn.functional.normalize(torch.randn(2, N, Hqk, D, generator=g), dim=-1).bfloat16()
        dec.append({"q": qk[0], "k": qk[1], "v": torch.randn(N, H, D, generator=g).bfloat16(),
                    "log_alpha": -0.05 * torch.rand(N, H, generator=g),
                    "beta": torch.rand(N, H, generator=g)})
    d = x["d"].cuda()
    outs = []
    for t in range(steps):
        xd = {k: v.cuda() for k, v in dec[t].items()}
        outs.append(cdr.recurrent_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], d, S))
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    cu = x["cu"].tolist()
    heads = np.arange(H) // (H // Hqk)
    for n in range(N):
        s0, s1 = cu[n], cu[n + 1]
        cat = lambda pre, key: torch.cat([pre[s0:s1]] + [dec[t][key][n:n + 1] for t in range(steps)])
        qn, kn = cat(x["q"], "q")[:, heads], cat(x["k"], "k")[:, heads]
        o, Sn = oracle.recurrence(q=qn[None], k=kn[None], v=cat(x["v"], "v")[None],
                                  log_alpha=cat(x["log_alpha"], "log_alpha")[None],
                                  beta=cat(x["beta"], "beta")[None], d=x["d"], S0=x["S0"][n:n + 1])
        got = torch.stack([outs[t][n] for t in range(steps)]).double().cpu().numpy()
        assert_close(f"decode out seq {n}", got, o[0, s1 - s0:], TOL_BF16)
        assert_close(f"state seq {n}", S[n].double().cpu().numpy(), Sn[0], TOL_BF16)


def test_grouped_decode_equals_the_step_on_expanded_heads():
    g = torch.Generator().manual_seed(5)
    B, H, Hqk, D = 3, 8, 2, 128
    q = torch.nn.functional.normalize(torch.randn(B, Hqk, D, generator=g), dim=-1).bfloat16().cuda()
    k = torch.nn.functional.normalize(torch.randn(B, Hqk, D, generator=g), dim=-1).bfloat16().cuda()
    v = torch.randn(B, H, D, generator=g).bfloat16().cuda()
    la = (-0.1 * torch.rand(B, H, generator=g)).cuda()
    be = torch.rand(B, H, generator=g).cuda()
    d = torch.rand(H, generator=g).cuda()
    S0 = (0.05 * torch.randn(B, H, D, D, generator=g)).cuda()
    S1, S2 = S0.clone(), S0.clone()
    o1 = cdr.recurrent_step(q, k, v, la, be, d, S1)
    rep = lambda t: t.repeat_interleave(H // Hqk, dim=1).contiguous()
    o2 = cdr.recurrent_step(rep(q), rep(k), v, la, be, d, S2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)

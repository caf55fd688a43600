"""Host logic of the context-parallel forward on CPU: gloo ranks (2 and 3), each
holding one contiguous piece of every chain, exchange their pieces' affine state
transitions and rerun from the composed start states.  The library calls are
replaced by float64 oracle stand-ins (CPU, test only), so this checks the
exchange, the rank order and the composition against the oracle over the whole
sequence; the kernels themselves are covered by the GPU parity tests."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from chunk_delta_rule_b200.context_parallel import chunk_fwd_context_parallel
from comba_workloads import CONFIGS, make_chunk_inputs

PIECE = 12   # tokens per rank


class OracleOps:
    """Stand-ins for the library calls: the float64 recurrence and a plain fold."""

    @staticmethod
    def fwd(q, k, v, log_alpha, beta, d, S0, chunk):
        o, S = oracle.recurrence(q, k, v, log_alpha, beta, d, S0)
        return torch.from_numpy(o), torch.from_numpy(S)

    @staticmethod
    def transition(q, k, v, log_alpha, beta, d, chunk):
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        _, R = oracle.recurrence(q, k, v, log_alpha, beta, d, None)
        eye = torch.eye(dv, dk, dtype=torch.float64).expand(B, H, dv, dk).contiguous()
        _, M = oracle.recurrence(q, k, torch.zeros_like(v), log_alpha, beta, d, eye)
        return torch.from_numpy(R), torch.from_numpy(M)

    @staticmethod
    def compose(R, M, S0):
        B, P, H = R.shape[:3]
        S = torch.zeros_like(R[:, 0]) if S0 is None else S0.to(torch.float64)
        out = torch.empty_like(R)
        for p in range(P):
            out[:, p] = S
            S = S @ M[:, p] + R[:, p]
        return out


def _inputs(world, s0):
    cfg = CONFIGS["tiny_fp32"].replace(B=2, H=2, T=world * PIECE, dk=128, dv=128, s0_std=s0)
    return make_chunk_inputs(cfg, seed=17 + world)


def _worker(rank, world, port, s0, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _inputs(world, s0)
        sl = slice(rank * PIECE, (rank + 1) * PIECE)
        piece = {n: x[n][:, sl].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
        out, S_end = chunk_fwd_context_parallel(**piece, d=x["d"], S0=x["S0"], ops=OracleOps)
        q.put((rank, out.numpy(), S_end.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,s0", [(2, 0.3), (3, 0.3), (3, 0.0)])
def test_context_parallel_pieces_join_to_the_whole_sequence(world, s0):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() % 800) + 7 * world
    procs = [ctx.Process(target=_worker, args=(r, world, port, s0, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = _inputs(world, s0)
    ro, rS = oracle.recurrence(**x)
    out = np.concatenate([r[1] for r in res], axis=1)
    assert np.abs(out - ro).max() <= 1e-12 * max(1.0, np.abs(ro).max())
    assert np.abs(res[-1][2] - rS).max() <= 1e-12 * max(1.0, np.abs(rS).max())
    # every other rank's end state is the chain's state after its piece
    _, S_mid = oracle.recurrence(**{n: (x[n][:, :PIECE] if x[n] is not None and x[n].dim() >= 3 else x[n])
                                    for n in x})
    assert np.abs(res[0][2] - S_mid).max() <= 1e-12 * max(1.0, np.abs(S_mid).max())


def test_context_parallel_requires_128_wide_heads():
    x = make_chunk_inputs(CONFIGS["tiny_fp32"])   # dk = dv = 32
    with pytest.raises(ValueError, match="dk = dv = 128"):
        chunk_fwd_context_parallel(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["d"], ops=OracleOps)

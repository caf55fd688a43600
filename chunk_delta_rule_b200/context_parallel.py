"""Context-parallel chunk forward: the sequence of every (b, h) chain is cut into
one contiguous piece per rank of a process group, one rank per GPU.

The state pass is affine in the state.  Over a piece it maps a start state S to
S M + R, where R is the end state from S = 0 and M is the end state from S = I
with V = 0.  This is the write-up's "recurrent across blocks, parallel inside"
form (section "硬件高效的分块并行计算") one level up, as in the segmented
single-GPU path.  Each rank:
  1. runs the chunk kernel twice over its piece, for R (from S = 0) and M (from
     S = I, V = 0);
  2. all-gathers R and M over the group: the path's one exchange, 2 x 64 KiB per
     chain per rank;
  3. composes the start states of all pieces with the library's compose kernel
     (S_start(0) = S0, S_start(p+1) = S_start(p) M_p + R_p) and keeps its own;
  4. reruns the chunk kernel over its piece from that state, for its outputs.
Step 1 is one launch of the chunk kernel over the piece's chains twice stacked,
with no outputs (comba_chunk_fwd_transition), so a rank runs the kernel's state
pass twice and writes its outputs once.  Every step of the computation runs in
the library's kernels; torch.distributed carries the exchange (NCCL between
GPUs).  dk = dv = 128.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["chunk_fwd_context_parallel"]


class _LibraryOps:
    """The three library calls the context-parallel forward is built from."""

    @staticmethod
    def transition(q, k, v, log_alpha, beta, d, chunk):
        from . import chunk_fwd_transition
        return chunk_fwd_transition(q, k, v, log_alpha, beta, d, chunk=chunk)

    @staticmethod
    def fwd(q, k, v, log_alpha, beta, d, S0, chunk):
        from . import chunk_fwd
        return chunk_fwd(q, k, v, log_alpha, beta, d, S0, chunk=chunk)

    @staticmethod
    def compose(R, M, S0):
        from . import state_compose
        return state_compose(R, M, S0)


def chunk_fwd_context_parallel(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                               beta: torch.Tensor, d: torch.Tensor, S0: Optional[torch.Tensor] = None,
                               chunk: int = 64, group=None, ops=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's piece of a context-parallel chunk forward.

    q, k [B, T_r, H, 128], v [B, T_r, H, 128], log_alpha, beta [B, T_r, H]: tokens
    r T_r .. (r + 1) T_r - 1 of every chain on rank r of ``group`` (all ranks the
    same T_r); d [H]; S0 [B, H, 128, 128] or None, the chains' initial state
    (read on rank 0's behalf by every rank; pass the same tensor everywhere).
    Returns (out for this piece, this piece's end state); on the last rank the end
    state is the chains' final state.  Every rank must make the call (collective).
    ``ops`` replaces the library calls (transition, fwd, compose); it exists for the
    host tests of the exchange."""
    ops = ops or _LibraryOps()
    B, Tr, H, dk = q.shape
    dv = v.shape[-1]
    if dk != 128 or dv != 128:
        raise ValueError("context-parallel forward: dk = dv = 128")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    # 1. this piece's transition
    R, M = ops.transition(q, k, v, log_alpha, beta, d, chunk)
    # 2. the exchange
    Rs = [torch.empty_like(R) for _ in range(world)]
    Ms = [torch.empty_like(M) for _ in range(world)]
    dist.all_gather(Rs, R.contiguous(), group=group)
    dist.all_gather(Ms, M.contiguous(), group=group)
    # 3. start states of all pieces; this rank's
    S_start = ops.compose(torch.stack(Rs, dim=1), torch.stack(Ms, dim=1), S0)
    S_mine = S_start[:, rank].contiguous()
    # 4. this piece's outputs from its true start state
    return ops.fwd(q, k, v, log_alpha, beta, d, S_mine, chunk)

"""comba_chunk_fwd_host (host buffers in and out, copies and kernels pipelined over
groups of batch rows) gives the same bits as the device-buffer entry point."""
import pytest
import torch

import chunk_delta_rule_b200 as cdr
from comba_workloads import CONFIGS, make_chunk_inputs

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "beta", "d", "S0")


@pytest.mark.parametrize("B,T,H,dk,dv,chunk,slices", [
    (6, 200, 3, 128, 128, 64, 1),
    (6, 200, 3, 128, 128, 64, 4),     # uneven slices (2, 1, 2, 1 rows)
    (5, 130, 2, 128, 128, 64, 16),    # more slices than rows
    (4, 77, 2, 64, 32, 32, 3),        # general kernel
])
def test_host_entry_equals_device_entry(B, T, H, dk, dv, chunk, slices):
    cfg = CONFIGS["layer340m_bf16"].replace(B=B, T=T, H=H, dk=dk, dv=dv, chunk=chunk, s0_std=0.05)
    x = make_chunk_inputs(cfg, seed=606 + B + T)
    xd = {k: x[k].cuda() for k in NAMES}
    ro, rS = cdr.chunk_fwd(**xd, chunk=chunk, segment=False)
    xh = {k: x[k].pin_memory() for k in NAMES}
    stream = torch.cuda.current_stream()
    ho, hS = cdr.chunk_fwd_host(**xh, chunk=chunk, slices=slices, stream=stream)
    stream.synchronize()
    assert cdr.get_last_error() == 0
    assert torch.equal(ho, ro.cpu())
    assert torch.equal(hS, rS.cpu())


def test_host_entry_back_to_back_calls_reuse_the_workspace():
    cfg = CONFIGS["layer340m_bf16"].replace(B=4, T=256, H=2, s0_std=0.05)
    xs = [make_chunk_inputs(cfg, seed=s) for s in (1, 2, 3)]
    refs = [cdr.chunk_fwd(**{k: x[k].cuda() for k in NAMES}, chunk=64, segment=False) for x in xs]
    # the pinned inputs must outlive the asynchronous copies: kept until the sync
    pinned = [{k: x[k].pin_memory() for k in NAMES} for x in xs]
    outs = [cdr.chunk_fwd_host(**xh, chunk=64, slices=4) for xh in pinned]
    torch.cuda.synchronize()
    for (ro, rS), (ho, hS) in zip(refs, outs):
        assert torch.equal(ho, ro.cpu()) and torch.equal(hS, rS.cpu())

"""comba_chunk_fwd_noalloc: the segmented chunk forward with its scratch in the
library's static device memory, against the workspace entry point and the oracle."""
import pytest
import torch

import chunk_delta_rule_b200 as cdr
import oracle
from comba_workloads import CONFIGS, make_chunk_inputs
from tests.gpu_util import TOL_BF16, assert_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,T", [(1, 2, 4096), (2, 4, 320)])
def test_noalloc_matches_workspace_path_and_oracle(B, H, T):
    # (1, 2, 4096) runs segmented (its workspace fits the static scratch);
    # (2, 4, 320) is short and runs unsegmented.
    cfg = CONFIGS["layer340m_bf16"].replace(B=B, H=H, T=T)
    x = make_chunk_inputs(cfg, seed=31 + T)
    xd = to_dev(x)
    args = {k: xd[k] for k in ("q", "k", "v", "log_alpha", "beta", "d")}
    out = torch.empty_like(xd["v"])
    S_final = torch.empty_like(xd["S0"])
    cdr.chunk_fwd_noalloc(**args, S0=xd["S0"], out=out, S_final=S_final, chunk=64)
    o_ws, S_ws = cdr.chunk_fwd(**args, S0=xd["S0"], chunk=64)
    torch.cuda.synchronize()
    assert cdr.library().comba_get_last_error() == 0
    # same arithmetic in the same order as the workspace entry point
    assert torch.equal(out, o_ws) and torch.equal(S_final, S_ws)
    ro, rS = oracle.recurrence(**x)
    assert_close("out", out.double().cpu().numpy(), ro, TOL_BF16)
    assert_close("S_final", S_final.double().cpu().numpy(), rS, TOL_BF16)

"""Helpers shared by the GPU parity tests: run the CUDA path on seeded inputs and
compare with the float64 oracle at the tolerances the workloads fix."""
from __future__ import annotations

import numpy as np
import torch

import chunk_delta_rule_b200 as cdr

# Tolerances: fp32 workloads rel-L2 <= 1e-5; bf16 workloads rel-L2 <= 5e-3 and
# max-abs <= 2e-2, each on out and on S_final.
TOL_F32 = dict(rel=1e-5, abs=None)
TOL_BF16 = dict(rel=5e-3, abs=2e-2)


def rel_l2(a, ref) -> float:
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (den if den > 0 else 1.0))


def max_abs(a, ref) -> float:
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(a - ref))) if a.size else 0.0


def assert_close(name, got, ref, tol):
    r = rel_l2(got, ref)
    m = max_abs(got, ref)
    assert np.isfinite(np.asarray(got, dtype=np.float64)).all(), f"{name}: non-finite values"
    assert r <= tol["rel"], f"{name}: rel-L2 {r:.3e} > {tol['rel']:.1e} (max-abs {m:.3e})"
    if tol["abs"] is not None:
        assert m <= tol["abs"], f"{name}: max-abs {m:.3e} > {tol['abs']:.1e} (rel-L2 {r:.3e})"
    return r, m


def to_dev(x: dict, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in x.items()}


def gpu_chunk(x: dict, chunk: int, device="cuda"):
    """Runs comba_chunk_fwd(_f32) on CPU-resident inputs; returns float64 numpy."""
    xd = to_dev(x, device)
    out, S = cdr.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["d"],
                           xd["S0"], chunk=chunk)
    torch.cuda.synchronize()
    assert cdr.get_last_error() == 0
    return out.double().cpu().numpy(), S.double().cpu().numpy()


def chain_slice(x: dict, b: int, h: int) -> dict:
    """Inputs of the single (b, h) chain, as a B=1, H=1 problem."""
    return {
        "q": x["q"][b:b + 1, :, h:h + 1], "k": x["k"][b:b + 1, :, h:h + 1],
        "v": x["v"][b:b + 1, :, h:h + 1],
        "log_alpha": x["log_alpha"][b:b + 1, :, h:h + 1], "beta": x["beta"][b:b + 1, :, h:h + 1],
        "d": x["d"][h:h + 1],
        "S0": None if x["S0"] is None else x["S0"][b:b + 1, h:h + 1],
    }

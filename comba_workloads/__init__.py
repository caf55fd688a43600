"""Seeded synthetic inputs for the Comba chunk-wise forward and its decode step.

This module is shared by the float64 oracle side (tests, CPU baseline) and the
CUDA side (tests, bench).  It holds only the input recipes (shapes, value
distributions, seeds and draw order) and none of the recurrence's arithmetic:
the L2 normalisation of q/k, the sigmoid that makes beta and the softplus that
makes log(alpha) are how the inputs are distributed, not steps of the method.

Layouts (row-major, contiguous):
  q, k      [B, T, H, dk]    bf16 or fp32 (the configuration's dtype)
  v         [B, T, H, dv]    same dtype as q
  log_alpha [B, T, H]        fp32, always < 0 (alpha_t = exp(log_alpha_t) in (0, 1))
  beta      [B, T, H]        fp32 in (0, 1)
  d         [H]              fp32, the per-head output-correction factor d_h
  S0        [B, H, dv, dk]   fp32 or None (zero initial state)

Draw order for one workload (one torch CPU generator seeded with the workload
seed): q, k, v, the log(alpha) pieces, beta, d, S0.  Values are drawn in
float64 and then rounded once to their storage dtype; consumers that need
float64 (the oracle) widen the rounded values, which is exact.

The configurations mirror the five workloads the method is measured on: a tiny
fp32 parity case, a 340M-model-layer shape, a 1.3B-model-layer shape (the
headline), a 64K-token long-context case with slow decay, and a batched decode
step repeated for 512 tokens.  The 0.02 in "S0 ~ N(0, 0.02)" is read as the
standard deviation, and the exp(U(-4,-1)) decay scale is drawn once per head
(the per-head time-constant reading); the softplus(N(0,1)) factor is drawn per
(b, t, h).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

__all__ = [
    "ChunkConfig", "DecodeConfig", "CONFIGS", "DECODE", "chunk_config",
    "make_chunk_inputs", "make_decode_state", "decode_step_inputs",
    "head_token_count", "VarlenConfig", "VARLEN", "varlen_lengths", "make_varlen_inputs",
    "make_gated_inputs", "make_cotangents",
]


@dataclasses.dataclass(frozen=True)
class ChunkConfig:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str            # "fp32" or "bf16": storage/compute dtype of q, k, v, out
    decay: str            # "uniform": log a ~ U(lo, hi);  "mamba": -softplus(N)*exp(U(-4,-1))
    decay_lo: float = -0.2
    decay_hi: float = -0.01
    s0_std: float = 0.0   # 0 means S0 = 0 (passed as None)
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def replace(self, **kw) -> "ChunkConfig":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    steps: int
    s0_std: float
    seed: int


CONFIGS: Dict[str, ChunkConfig] = {
    "tiny_fp32": ChunkConfig("tiny_fp32", B=1, H=2, T=128, dk=32, dv=32, chunk=32,
                             dtype="fp32", decay="uniform", decay_lo=-0.2, decay_hi=-0.01,
                             s0_std=0.0, seed=0),
    "layer340m_bf16": ChunkConfig("layer340m_bf16", B=8, H=8, T=2048, dk=128, dv=128, chunk=64,
                                  dtype="bf16", decay="mamba", s0_std=0.02, seed=1),
    "layer1p3b_bf16": ChunkConfig("layer1p3b_bf16", B=8, H=16, T=4096, dk=128, dv=128, chunk=64,
                                  dtype="bf16", decay="mamba", s0_std=0.02, seed=2),
    "long64k_bf16": ChunkConfig("long64k_bf16", B=1, H=16, T=65536, dk=128, dv=128, chunk=64,
                                dtype="bf16", decay="uniform", decay_lo=-0.01, decay_hi=-0.0001,
                                s0_std=0.02, seed=3),
}

DECODE = DecodeConfig("decode_b256_h32", B=256, H=32, dk=128, dv=128, steps=512,
                      s0_std=0.02, seed=4)


@dataclasses.dataclass(frozen=True)
class VarlenConfig:
    """Packed variable-length sequences whose value heads share q / k heads."""
    name: str
    total_T: int          # packed tokens per step
    H: int                # value heads
    Hqk: int              # q / k heads (divides H)
    dk: int
    dv: int
    chunk: int
    len_median: float     # sequence lengths: log-normal, clipped to [len_min, len_max]
    len_sigma: float
    len_min: int
    len_max: int
    s0_std: float
    seed: int


# The 1.3B layer's tokens per step in the mamba form (16 value heads sharing one
# 128-dim q / k head), as a mix of sequence lengths.
VARLEN = VarlenConfig("varlen_mamba1p3b_bf16", total_T=32768, H=16, Hqk=1, dk=128, dv=128, chunk=64,
                      len_median=1024.0, len_sigma=1.0, len_min=64, len_max=8192, s0_std=0.02, seed=5)


def varlen_lengths(cfg: VarlenConfig):
    """Seeded sequence lengths summing to cfg.total_T (the last one trimmed)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed)
    lengths, total = [], 0
    while total < cfg.total_T:
        z = float(torch.randn((), generator=gen))
        n = int(round(cfg.len_median * math.exp(cfg.len_sigma * z)))
        n = max(cfg.len_min, min(cfg.len_max, n))
        n = min(n, cfg.total_T - total)
        lengths.append(n)
        total += n
    return lengths


def make_varlen_inputs(cfg: VarlenConfig) -> Dict[str, torch.Tensor]:
    """Packed inputs of one varlen workload, CPU tensors: q, k [total_T, Hqk, dk] and
    v [total_T, H, dv] bf16, log_alpha / beta [total_T, H] and d [H] fp32 (draws of the
    chunk workloads), S0 [N, H, dv, dk] fp32, cu_seqlens [N+1] int32."""
    lengths = varlen_lengths(cfg)
    base = ChunkConfig(cfg.name, B=1, H=cfg.H, T=cfg.total_T, dk=cfg.dk, dv=cfg.dv, chunk=cfg.chunk,
                       dtype="bf16", decay="mamba", s0_std=0.0, seed=cfg.seed)
    xv = make_chunk_inputs(base)
    xq = make_chunk_inputs(base.replace(H=cfg.Hqk), seed=cfg.seed + 1)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed + 2)
    N = len(lengths)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    return {
        "q": xq["q"][0].contiguous(), "k": xq["k"][0].contiguous(), "v": xv["v"][0].contiguous(),
        "log_alpha": xv["log_alpha"][0].contiguous(), "beta": xv["beta"][0].contiguous(),
        "d": xv["d"],
        "S0": (cfg.s0_std * _normal(gen, (N, cfg.H, cfg.dv, cfg.dk))).to(torch.float32).contiguous(),
        "cu_seqlens": torch.tensor(cu, dtype=torch.int32),
    }


def make_gated_inputs(cfg: ChunkConfig, seed: Optional[int] = None, dt_bias_std: float = 0.0) -> Dict[str, torch.Tensor]:
    """Raw-projection inputs of a chunk workload, CPU tensors: q_raw, k_raw [B,T,H,dk]
    bf16 drawn N(0,1) and scaled per row by exp(U(-1,1)) (not normalised); v bf16 as
    the chunk workloads; a_raw, b_raw [B,T,H] ~ N(0,1); A_log [H] ~ U(-4,-1) (the
    per-head log scale of the chunk workloads' decay draws); dt_bias [H] ~ N(0,
    dt_bias_std^2); d [H] ~ U(0,1); S0 as cfg.s0_std."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed + 7919 if seed is None else seed)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    scale_q = torch.exp(_uniform(gen, (B, T, H, 1), -1.0, 1.0))
    scale_k = torch.exp(_uniform(gen, (B, T, H, 1), -1.0, 1.0))
    q = (_normal(gen, (B, T, H, dk)) * scale_q).to(torch.bfloat16)
    k = (_normal(gen, (B, T, H, dk)) * scale_k).to(torch.bfloat16)
    v = _normal(gen, (B, T, H, dv)).to(torch.bfloat16)
    a = _normal(gen, (B, T, H)).to(torch.float32)
    b = _normal(gen, (B, T, H)).to(torch.float32)
    A_log = _uniform(gen, (H,), -4.0, -1.0).to(torch.float32)
    dt_bias = (dt_bias_std * _normal(gen, (H,))).to(torch.float32)
    d = _uniform(gen, (H,), 0.0, 1.0).to(torch.float32)
    S0 = (cfg.s0_std * _normal(gen, (B, H, dv, dk))).to(torch.float32) if cfg.s0_std > 0 else None
    return {"q_raw": q.contiguous(), "k_raw": k.contiguous(), "v": v.contiguous(), "a_raw": a.contiguous(),
            "b_raw": b.contiguous(), "A_log": A_log.contiguous(), "dt_bias": dt_bias.contiguous(),
            "d": d.contiguous(), "S0": None if S0 is None else S0.contiguous()}


def chunk_config(name: str) -> ChunkConfig:
    return CONFIGS[name]


def head_token_count(cfg: ChunkConfig) -> int:
    return cfg.B * cfg.T * cfg.H


def _normal(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float64)


def _uniform(gen: torch.Generator, shape, lo: float, hi: float) -> torch.Tensor:
    return lo + (hi - lo) * torch.rand(shape, generator=gen, dtype=torch.float64)


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # Input recipe: q and k are unit vectors per (b, t, h).
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def _decay_scale(gen, H):
    # Per-head decay time constant of the "mamba" recipe, drawn once per head.
    return torch.exp(_uniform(gen, (H,), -4.0, -1.0))


def _gates(gen, shape_bth, H, decay, lo, hi, scale=None):
    if decay == "uniform":
        log_alpha = _uniform(gen, shape_bth, lo, hi)
    elif decay == "mamba":
        sp = torch.nn.functional.softplus(_normal(gen, shape_bth))
        if scale is None:
            scale = _decay_scale(gen, H)
        log_alpha = -sp * scale
    else:
        raise ValueError(decay)
    beta = torch.sigmoid(_normal(gen, shape_bth))
    return log_alpha, beta


def make_chunk_inputs(cfg: ChunkConfig, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All inputs of one chunk-forward workload, as CPU tensors in storage dtypes."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed if seed is None else seed)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    dt = cfg.torch_dtype
    q = _unit_rows(_normal(gen, (B, T, H, dk))).to(dt)
    k = _unit_rows(_normal(gen, (B, T, H, dk))).to(dt)
    v = _normal(gen, (B, T, H, dv)).to(dt)
    log_alpha, beta = _gates(gen, (B, T, H), H, cfg.decay, cfg.decay_lo, cfg.decay_hi)
    d = _uniform(gen, (H,), 0.0, 1.0)
    S0 = None
    if cfg.s0_std > 0:
        S0 = (cfg.s0_std * _normal(gen, (B, H, dv, dk))).to(torch.float32)
    return {
        "q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
        "log_alpha": log_alpha.to(torch.float32).contiguous(),
        "beta": beta.to(torch.float32).contiguous(),
        "d": d.to(torch.float32).contiguous(),
        "S0": None if S0 is None else S0.contiguous(),
    }


def make_cotangents(cfg: ChunkConfig, seed: Optional[int] = None, dS_std: float = 1.0) -> Dict[str, torch.Tensor]:
    """Cotangents for the backward: dout [B,T,H,dv] ~ N(0,1) in the workload's storage
    dtype and dS_final [B,H,dv,dk] ~ N(0, dS_std^2) fp32 (None when dS_std == 0), as
    CPU tensors."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed((cfg.seed if seed is None else seed) + 7919)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    dout = _normal(gen, (B, T, H, dv)).to(cfg.torch_dtype).contiguous()
    dS = None
    if dS_std > 0:
        dS = (dS_std * _normal(gen, (B, H, dv, dk))).to(torch.float32).contiguous()
    return {"dout": dout, "dS_final": dS}


def make_decode_state(cfg: DecodeConfig = DECODE, B: Optional[int] = None,
                      H: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The per-head d, the per-head decay scale and the resident fp32 state
    S [B, H, dv, dk] of the decode workload (draw order: d, scale, S).

    Returns the generator too, positioned after these draws, so that per-step
    inputs follow in a fixed order."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed)
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    d = _uniform(gen, (H,), 0.0, 1.0).to(torch.float32)
    scale = _decay_scale(gen, H)
    S = (cfg.s0_std * _normal(gen, (B, H, cfg.dv, cfg.dk))).to(torch.float32)
    return {"d": d.contiguous(), "S": S.contiguous(), "decay_scale": scale, "gen": gen}


def decode_step_inputs(gen: torch.Generator, decay_scale: torch.Tensor,
                       cfg: DecodeConfig = DECODE, B: Optional[int] = None,
                       H: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """One decode token for every (b, h): q, k [B, H, dk] bf16, v [B, H, dv] bf16,
    log_alpha, beta [B, H] fp32.  Draw order per step: q, k, v, softplus factor, beta.
    ``decay_scale`` is the per-head scale from ``make_decode_state``."""
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    q = _unit_rows(_normal(gen, (B, H, cfg.dk))).to(torch.bfloat16)
    k = _unit_rows(_normal(gen, (B, H, cfg.dk))).to(torch.bfloat16)
    v = _normal(gen, (B, H, cfg.dv)).to(torch.bfloat16)
    log_alpha, beta = _gates(gen, (B, H), H, "mamba", 0.0, 0.0, scale=decay_scale)
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "log_alpha": log_alpha.to(torch.float32).contiguous(),
            "beta": beta.to(torch.float32).contiguous()}

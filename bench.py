"""Benchmark of the Comba chunk-wise forward on B200.

One step = one chunk-wise forward over the whole workload (every (b, h) chain,
every token), i.e. one pass of the hot path.  Default workload: the 1.3B-model
layer shape (B=8, H=16, T=4096, dk=dv=128, chunk=64, bf16 q/k/v/out, fp32
gates and state), seeded synthetic inputs.

Prints ONE JSON line (rank 0).  ``value`` is device-timed throughput with the
inputs resident in HBM; ``e2e`` is the same metric through the public Python
API with the step's inputs copied from pinned host memory and its outputs
copied back inside the timed region.  Multi-GPU (torchrun): the (b, h) chains
are independent, so every rank runs its own batch (weak scaling, no
collective on the data path); time is the max over ranks.

``--impl reference`` times the float64 CPU oracle (the plain token-by-token
recurrence) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from comba_workloads import (CONFIGS, DECODE, VARLEN, make_cotangents, make_gated_inputs, make_varlen_inputs,  # noqa: E402
                             decode_step_inputs, make_chunk_inputs,
                             make_decode_state)

METRIC = "Comba chunk-fwd tokens/s and TFLOP/s on 1 B200, % of roofline"
L2_BYTES = 126 * 2 ** 20


def algorithmic_counts(cfg):
    """Per-launch algorithmic FLOPs and bytes of the chunk-wise forward.

    FLOPs per head-token (triangle-aware): C(3dk + 2dv) + 6 dk dv
      (K K^T and Q K^T lower halves, the inverse applied to [K | V], P X lower
       half; W S^T, (Q - dK) S^T and the X^T K state update).
    Bytes per head-token: q, k, v and out at their element size plus fp32
      log(alpha) and beta; plus the fp32 S0 read and S_final write once per chain."""
    C, dk, dv = cfg.chunk, cfg.dk, cfg.dv
    el = 2 if cfg.dtype == "bf16" else 4
    ht = cfg.B * cfg.T * cfg.H
    flops = ht * (C * (3 * dk + 2 * dv) + 6 * dk * dv)
    bytes_ = ht * ((2 * dk + 2 * dv) * el + 8) + cfg.B * cfg.H * dv * dk * 4 * 2
    return flops, bytes_


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# The sources that define the profiled chunk kernel (its device code and the
# helpers it includes); host-side files do not change the kernel.
KERNEL_SOURCES = ("chunk_tc.cuh", "tc_primitives.cuh", "common.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "chunk_delta_rule_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    or None when the summary is missing or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", f"chunk_fwd_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m_t or not m_h or m_h.group(1) != kernel_source_hash():
        return None
    return float(m_t.group(1))


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi.  Started before
    the timed region; ``summary(t0, t1)`` keeps the samples taken between the
    host times t0 and t1 (at least the first one after t0)."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 20):
        self.gpu = gpu_index
        self.interval = interval_ms
        self.proc = None
        self.samples = []   # (host time, fields)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.interval)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t_end = time.time() + 5.0
            while not self.samples and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def wait_after(self, t: float, timeout: float = 2.0):
        t_end = time.time() + timeout
        while self.proc is not None and time.time() < t_end:
            if any(ts >= t for ts, _ in self.samples):
                return
            time.sleep(0.01)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        inside = [p for ts, p in self.samples if t0 <= ts <= t1]
        if not inside:
            after = [p for ts, p in self.samples if ts >= t0]
            inside = after[:1]
        sm, mx, reasons = [], None, set()
        for parts in inside:
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def weak_scaling_value(tokens_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: every rank processes its own batch; time is the
    slowest rank's."""
    return world * tokens_per_rank / (ms_per_step_max / 1e3)


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time (all ranks must call)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg, rank: int) -> int:
    """Each rank draws its own batch (weak scaling over independent chains)."""
    return cfg.seed + 1000 * rank


def cpu_baseline(cfg, x, target_s: float = 10.0):
    """Times the float64 oracle (as it stands) on the host cores on a bounded
    sample of the workload's (b, h) chains -- the whole workload, repeated,
    when it takes less than ``target_s`` -- and returns the baseline record."""
    import oracle
    threads = oracle.num_threads()
    B, H = cfg.B, cfg.H

    def run(chains):
        sl = [(c // H, c % H) for c in chains]
        xs = {
            "q": torch.stack([x["q"][b, :, h] for b, h in sl], dim=1)[None],
            "k": torch.stack([x["k"][b, :, h] for b, h in sl], dim=1)[None],
            "v": torch.stack([x["v"][b, :, h] for b, h in sl], dim=1)[None],
            "log_alpha": torch.stack([x["log_alpha"][b, :, h] for b, h in sl], dim=1)[None],
            "beta": torch.stack([x["beta"][b, :, h] for b, h in sl], dim=1)[None],
            "d": torch.stack([x["d"][h] for _, h in sl]),
            "S0": None if x["S0"] is None else torch.stack([x["S0"][b, h] for b, h in sl])[None],
        }
        t0 = time.perf_counter()
        oracle.recurrence(**xs, threads=threads)
        return time.perf_counter() - t0

    probe = run([0])
    n = max(1, min(B * H, int(target_s / max(probe, 1e-6)) * threads))
    chains = list(range(n))
    el, reps = 0.0, 0
    while True:
        el += run(chains)
        reps += 1
        if el >= target_s or n < B * H:
            break
    tokens = reps * n * cfg.T / H  # a token carries all H heads
    return {"value": tokens / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {B * H} (b,h) chains x {cfg.T} tokens of {cfg.name}"
                      f"{'' if reps == 1 else f', {reps} passes'}; float64 C recurrence, OpenMP "
                      f"over chains; {el:.1f} s",
            "seconds": el}


def run_reference(args, cfg):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = make_chunk_inputs(cfg)
    per_step = max(1.0, min(10.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(cfg, x, target_s=0.2)
    vals, secs, rec = [], 0.0, None
    for _ in range(args.steps):
        rec = cpu_baseline(cfg, x, target_s=per_step)
        vals.append(rec["value"])
        secs += rec["seconds"]
    value = sum(vals) / len(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_record(cfg),
        "cpu_baseline": {"kind": "oracle", "cores": rec["cores"], "sample": rec["sample"],
                         "value": value, "unit": "tokens/s"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def config_record(cfg):
    return {"workload": cfg.name, "B": cfg.B, "T": cfg.T, "H": cfg.H, "dk": cfg.dk, "dv": cfg.dv,
            "chunk": cfg.chunk, "tokens_per_step": cfg.B * cfg.T,
            "l2": "inputs larger than L2 (q,k,v,out %.0f MiB vs 126 MiB L2); no flush"
                  % (cfg.B * cfg.T * cfg.H * (2 * cfg.dk + 2 * cfg.dv) * (2 if cfg.dtype == "bf16" else 4) / 2 ** 20)}


def decode_counts(cfg):
    """Algorithmic bytes and FLOPs of one decode step over all (b, h): the fp32
    state read and written once, q, k, v, out in bf16, two fp32 gates."""
    heads = cfg.B * cfg.H
    bytes_ = heads * (2 * cfg.dv * cfg.dk * 4 + (2 * cfg.dk + 2 * cfg.dv) * 2 + 8)
    flops = heads * 8 * cfg.dv * cfg.dk
    return flops, bytes_


def run_decode(args):
    """One step = one comba_recurrent_step for every (b, h) of the decode
    workload, state resident in HBM (537 MB, larger than L2)."""
    import chunk_delta_rule_b200 as cdr
    cfg = DECODE
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cdr.library()
    st = make_decode_state(cfg)
    d = st["d"].to(dev)
    S = st["S"].to(dev)
    n_in = 8   # distinct tokens, cycled
    host = [decode_step_inputs(st["gen"], st["decay_scale"], cfg) for _ in range(n_in)]
    host = [{k: v.pin_memory() for k, v in x.items()} for x in host]
    dev_in = [{k: v.to(dev) for k, v in x.items()} for x in host]
    out = torch.empty((cfg.B, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        x = dev_in[i % n_in]
        cdr.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d, S, out=out,
                           stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0).start()
    th0 = time.time()
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    th1 = time.time()
    clocks.wait_after(th0)
    clocks.stop()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    # end to end: this step's token inputs from pinned host memory, out back to host
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    stage = {k: torch.empty_like(v) for k, v in dev_in[0].items()}

    def e2e_step(i):
        for k, v in host[i % n_in].items():
            stage[k].copy_(v, non_blocking=True)
        cdr.recurrent_step(stage["q"], stage["k"], stage["v"], stage["log_alpha"], stage["beta"],
                           d, S, out=out, stream=stream)
        out_h.copy_(out, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = ev0.elapsed_time(ev1) / args.steps
    flops, bytes_ = decode_counts(cfg)
    peaks = load_peaks()
    gbs = bytes_ / (ms_step / 1e3) / 1e9
    line = {
        "metric": "Comba decode-step tokens/s (one token per batch row, all heads), % of HBM roofline",
        "value": cfg.B / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "dk": cfg.dk, "dv": cfg.dv,
                   "l2": "state 537 MB larger than L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic_bytes_per_launch": bytes_},
        "e2e": {"value": cfg.B / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host[0].values()),
                "d2h_bytes_per_step": out_h.numel() * 2, "ms_per_step": ms_e2e},
        "clocks": clocks.summary(th0, th1),
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)


def varlen_counts(cfg, nseq):
    """Algorithmic FLOPs and bytes of one packed varlen forward: the per-head-token
    FLOPs of the chunk workloads over every value head; q and k once per q / k head,
    v and out per value head, two fp32 gates, S0 read and S_final written once per
    (sequence, value head)."""
    C, dk, dv, H = cfg.chunk, cfg.dk, cfg.dv, cfg.H
    flops = cfg.total_T * H * (C * (3 * dk + 2 * dv) + 6 * dk * dv)
    bytes_ = cfg.total_T * ((2 * cfg.Hqk * dk + 2 * H * dv) * 2 + 8 * H) + nseq * H * dv * dk * 4 * 2
    return flops, bytes_


def run_varlen(args):
    """One step = one comba_chunk_fwd_varlen over the packed workload (every
    sequence, every value head), inputs resident in HBM."""
    import chunk_delta_rule_b200 as cdr
    cfg = VARLEN
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cdr.library()
    x = make_varlen_inputs(cfg)
    N = x["cu_seqlens"].numel() - 1
    host = {k: v.pin_memory() for k, v in x.items()}
    d_ = {k: v.to(dev) for k, v in host.items()}
    out = torch.empty((cfg.total_T, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
    S_final = torch.empty((N, cfg.H, cfg.dv, cfg.dk), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cdr.chunk_fwd_varlen(d_["q"], d_["k"], d_["v"], d_["log_alpha"], d_["beta"], d_["d"],
                             d_["cu_seqlens"], S0=d_["S0"], chunk=cfg.chunk, out=out,
                             S_final=S_final, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert cdr.get_last_error(dev) == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0).start()
    th0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    th1 = time.time()
    clocks.wait_after(th0)
    clocks.stop()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    if cdr.get_last_error(dev) != 0:
        raise RuntimeError("device-side error during the timed region")
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    S_h = torch.empty(S_final.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        for k in host:
            d_[k].copy_(host[k], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        S_h.copy_(S_final, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = ev0.elapsed_time(ev1) / args.steps
    flops, bytes_ = varlen_counts(cfg, N)
    peaks = load_peaks()
    gbs = bytes_ / (ms_step / 1e3) / 1e9
    lengths = (x["cu_seqlens"][1:] - x["cu_seqlens"][:-1]).tolist()
    line = {
        "metric": "Comba chunk-fwd tokens/s over packed variable-length sequences, % of HBM roofline",
        "value": cfg.total_T / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "total_T": cfg.total_T, "sequences": N,
                   "length_min": min(lengths), "length_max": max(lengths), "H": cfg.H, "Hqk": cfg.Hqk,
                   "dk": cfg.dk, "dv": cfg.dv, "chunk": cfg.chunk,
                   "l2": "inputs larger than L2 (q,k,v,out %.0f MiB vs 126 MiB L2); no flush"
                         % (cfg.total_T * (2 * cfg.Hqk * cfg.dk + 2 * cfg.H * cfg.dv) * 2 / 2 ** 20)},
        "tflops": flops / (ms_step / 1e3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": peaks["source"] + " hbm_gbs (copy)",
                     "algorithmic_bytes_per_launch": bytes_, "algorithmic_flops_per_launch": flops},
        "e2e": {"value": cfg.total_T / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
                "d2h_bytes_per_step": out_h.numel() * 2 + S_h.numel() * 4, "ms_per_step": ms_e2e},
        "clocks": clocks.summary(th0, th1),
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)


GATED = "layer1p3b_gated_bf16"


def run_gated(args):
    """One step = one comba_chunk_fwd_gated over the 1.3B-layer workload given as raw
    projections (q, k not normalised, raw gate projections): the same algorithmic
    bytes as the plain workload, inputs resident in HBM."""
    import chunk_delta_rule_b200 as cdr
    cfg = CONFIGS["layer1p3b_bf16"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cdr.library()
    x = make_gated_inputs(cfg)
    host = {k: v.pin_memory() for k, v in x.items() if v is not None}
    d_ = {k: v.to(dev) for k, v in host.items()}
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
    S_final = torch.empty((cfg.B, cfg.H, cfg.dv, cfg.dk), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cdr.chunk_fwd_gated(d_["q_raw"], d_["k_raw"], d_["v"], d_["a_raw"], d_["b_raw"], d_["A_log"],
                            d_["dt_bias"], d_["d"], d_.get("S0"), chunk=cfg.chunk, out=out,
                            S_final=S_final, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert cdr.get_last_error(dev) == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0).start()
    th0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    th1 = time.time()
    clocks.wait_after(th0)
    clocks.stop()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    if cdr.get_last_error(dev) != 0:
        raise RuntimeError("device-side error during the timed region")
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    S_h = torch.empty(S_final.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        for k in host:
            d_[k].copy_(host[k], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        S_h.copy_(S_final, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = ev0.elapsed_time(ev1) / args.steps
    flops, bytes_ = algorithmic_counts(cfg)
    peaks = load_peaks()
    gbs = bytes_ / (ms_step / 1e3) / 1e9
    line = {
        "metric": "Comba chunk-fwd tokens/s from raw projections (normalisation and gates in the kernel), % of HBM roofline",
        "value": cfg.B * cfg.T / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_record(cfg), workload=GATED),
        "tflops": flops / (ms_step / 1e3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": peaks["source"] + " hbm_gbs (copy)",
                     "algorithmic_bytes_per_launch": bytes_, "algorithmic_flops_per_launch": flops},
        "e2e": {"value": cfg.B * cfg.T / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
                "d2h_bytes_per_step": out_h.numel() * 2 + S_h.numel() * 4, "ms_per_step": ms_e2e},
        "clocks": clocks.summary(th0, th1),
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)


BWD = "layer1p3b_bwd_bf16"
BWD_CHUNK = 32   # tokens per chunk of the backward kernels


def bwd_algorithmic_flops(cfg):
    """Multiply-add work of one backward over the workload, 2 flops per FMA, per
    32-token chunk of every (b, h) chain.  It counts the products and triangular
    solves the chunk adjoint performs, including recomputing the forward's W, U~,
    X and P.
      prep     K K^T, Q~ K^T, the two-column-block solve, P W, dO^T (Gamma Q~ - P W)
      states   W S^T, X^T diag K
      dstates  dS K^T, Z W
      grads    K S^T, K K^T, K dS'^T, Q~ K^T, two solves, P^T dO, dR X^T, dO X^T,
               dO S, X dS', dZ K, dZ^T Q~, (dY + dY^T) K, dR S"""
    L, dk, dv = BWD_CHUNK, cfg.dk, cfg.dv
    tri = L * (L - 1)                      # flops of one column of a unit-triangular solve
    prep = 3 * 2 * L * L * dk + tri * (dk + dv) + 2 * dv * dk * L
    states = 2 * (2 * L * dk * dv)
    dstates = 2 * (2 * L * dk * dv)
    grads = (5 * 2 * L * dv * dk + 2 * 2 * L * L * dk + 2 * tri * dv + 3 * 2 * L * L * dv
             + 3 * 2 * L * L * dk)
    chunks = cfg.B * cfg.H * ((cfg.T + L - 1) // L)
    return chunks * (prep + states + dstates + grads)


def bwd_algorithmic_bytes(cfg):
    """Bytes one backward must move at the least: every input read once (bf16 q, k,
    v, dout; fp32 gates, d, S0, dS_final) and every gradient written once (fp32 dq,
    dk, dv, dlog_alpha, dbeta, dS0, dd).  The workspace round trips of the staged
    design (per-chunk operand tiles, states and state gradients) are not counted."""
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    tok = B * T * H
    inputs = tok * (2 * dk + 2 * dv) * 2 + tok * 2 * 4 + H * 4 + 2 * B * H * dv * dk * 4
    grads = tok * (2 * dk + dv) * 4 + tok * 2 * 4 + B * H * dv * dk * 4 + H * 4
    return inputs + grads


def cpu_baseline_bwd(cfg, x, cot, target_s: float = 10.0):
    """Times the float64 oracle's gradients (``oracle.recurrence_bwd_np``, as it
    stands) on a bounded sample of the workload's (b, h) chains, stacked as heads of
    one batch row; returns the baseline record in tokens/s of the whole workload."""
    import oracle
    B, H = cfg.B, cfg.H

    def run(chains):
        sl = [(c // H, c % H) for c in chains]
        pick = lambda t: torch.stack([t[b, :, h] for b, h in sl], dim=1)[None]
        pick_s = lambda t: None if t is None else torch.stack([t[b, h] for b, h in sl])[None]
        t0 = time.perf_counter()
        oracle.recurrence_bwd_np(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["log_alpha"]),
                                 pick(x["beta"]), torch.stack([x["d"][h] for _, h in sl]), pick_s(x["S0"]),
                                 pick(cot["dout"]), pick_s(cot["dS_final"]))
        return time.perf_counter() - t0

    probe = run([0])
    n = max(1, min(B * H, int(target_s / max(probe, 1e-6))))
    el = run(list(range(n))) if n > 1 else probe
    tokens = n * cfg.T / H   # a token carries all H heads
    return {"value": tokens / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} of {B * H} (b,h) chains x {cfg.T} tokens of {cfg.name}; float64 NumPy "
                      f"reverse-mode token loop (states recomputed from checkpoints), one thread; {el:.1f} s",
            "seconds": el}


def run_bwd(args):
    """One step = one comba_chunk_bwd over the 1.3B layer (bf16 q, k, v, dout; fp32
    gates, S0 and dS_final), inputs and cotangents resident in HBM.  Under torchrun
    every rank runs its own batch of independent chains (weak scaling, no collective
    in the data path); times are the max over ranks."""
    import chunk_delta_rule_b200 as cdr
    cfg = CONFIGS["layer1p3b_bf16"]
    if args.batch:   # a smaller batch of the same layer, for profiling captures
        cfg = cfg.replace(B=args.batch)
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib = cdr.library()
    x = make_chunk_inputs(cfg, seed=rank_seed(cfg, rank))
    x.update(make_cotangents(cfg, seed=rank_seed(cfg, rank)))
    host = {k: v.pin_memory() for k, v in x.items() if v is not None}
    d_ = {k: v.to(dev) for k, v in host.items()}
    stream = torch.cuda.current_stream(dev)
    need = int(lib.comba_chunk_bwd_workspace_size(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv))
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    res = {}

    def step():
        res.update(cdr.chunk_bwd(d_["q"], d_["k"], d_["v"], d_["log_alpha"], d_["beta"], d_["d"], d_["dout"],
                                 S0=d_.get("S0"), dS_final=d_.get("dS_final"), workspace=ws, stream=stream))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert cdr.get_last_error(dev) == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local).start()
    barrier(world)
    torch.cuda.synchronize(dev)
    th0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    th1 = time.time()
    clocks.wait_after(th0)
    clocks.stop()
    barrier(world)
    ms_step = max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps
    if cdr.get_last_error(dev) != 0:
        raise RuntimeError("device-side error during the timed region")
    outs_h = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in res.items() if v is not None}

    def e2e_step():
        for k in host:
            d_[k].copy_(host[k], non_blocking=True)
        step()
        for k in outs_h:
            outs_h[k].copy_(res[k], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    ev0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps
    flops = bwd_algorithmic_flops(cfg)
    nbytes = bwd_algorithmic_bytes(cfg)
    ck = clocks.summary(th0, th1)
    peaks = load_peaks()
    peak = peaks["hbm_gbs"]
    gbs = nbytes / (ms_step / 1e3) / 1e9
    line = {
        "metric": "Comba chunk-bwd tokens/s (all input gradients) on 1 B200, % of HBM roofline",
        "value": weak_scaling_value(cfg.B * cfg.T, world, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(config_record(cfg), workload=BWD, chunk=BWD_CHUNK, inputs="bf16 q, k, v, dout"),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": None, "peak_source": peaks["source"],
                     "algorithmic_bytes_per_step": nbytes, "algorithmic_flops_per_step": flops,
                     "tflops": flops / (ms_step / 1e3) / 1e12,
                     "scope": "whole backward step (4 launches), against the bytes it must move at the least"},
        "e2e": {"value": weak_scaling_value(cfg.B * cfg.T, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
                "d2h_bytes_per_step": sum(v.numel() * v.element_size() for v in outs_h.values()),
                "ms_per_step": ms_e2e},
        "clocks": ck,
        "gpu_launches": 4 * args.steps,   # prep, both state passes, grads, dd sum
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline_bwd(cfg, x, x).items() if k != "seconds"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="layer1p3b_bf16",
                    choices=sorted(CONFIGS) + [DECODE.name, VARLEN.name, GATED, BWD])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="backward workload only: run the 1.3B layer with this batch instead of 8 "
                         "(for profiling captures; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload == DECODE.name:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the decode workload has no reference arm; the headline workload does"}))
            return
        run_decode(args)
        return
    if args.workload == BWD:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the backward workload has no reference arm; the headline workload does"}))
            return
        run_bwd(args)
        return
    if args.workload == GATED:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the raw-projection workload has no reference arm; the headline workload does"}))
            return
        run_gated(args)
        return
    if args.workload == VARLEN.name:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the packed varlen workload has no reference arm; the headline workload does"}))
            return
        run_varlen(args)
        return
    cfg = CONFIGS[args.workload]
    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import chunk_delta_rule_b200 as cdr
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cdr.library()  # fails loudly if the CUDA library is missing

    # Weak scaling: every rank owns a full batch of independent chains.
    x = make_chunk_inputs(cfg, seed=rank_seed(cfg, rank))
    names = ("q", "k", "v", "log_alpha", "beta", "d", "S0")
    host = {k: x[k].pin_memory() for k in names if x[k] is not None}
    dv_ = {k: host[k].to(dev, non_blocking=True) for k in host}
    S0 = dv_.get("S0")
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=cfg.torch_dtype, device=dev)
    S_final = torch.empty((cfg.B, cfg.H, cfg.dv, cfg.dk), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        cdr.chunk_fwd(dv_["q"], dv_["k"], dv_["v"], dv_["log_alpha"], dv_["beta"], dv_["d"], S0,
                      chunk=cfg.chunk, out=out, S_final=S_final, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert cdr.get_last_error(dev) == 0

    # ---- device-timed region: inputs resident in HBM -------------------------------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local).start()
    barrier(world)
    torch.cuda.synchronize(dev)
    th0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    th1 = time.time()
    clocks.wait_after(th0)
    clocks.stop()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps
    tokens_all = world * cfg.B * cfg.T
    value = weak_scaling_value(cfg.B * cfg.T, world, ms_step)
    if cdr.get_last_error(dev) != 0:
        raise RuntimeError("device-side error during the timed region")

    # ---- end-to-end: pinned host buffers in, the C-ABI host entry point (copies in,
    # kernels and copies out pipelined over groups of batch rows), host results out;
    # fp32 workloads (no host entry) copy around the device call instead ----------------
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    S_h = torch.empty(S_final.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + S_h.numel() * 4

    def e2e_step():
        if cfg.dtype == "bf16" and cfg.B > 1:
            cdr.chunk_fwd_host(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], host["d"],
                               host.get("S0"), chunk=cfg.chunk, out=out_h, S_final=S_h,
                               slices=min(8, cfg.B), device=dev, stream=stream)
            return
        for k in host:
            dv_[k].copy_(host[k], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        S_h.copy_(S_final, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps
    e2e_value = tokens_all / (ms_e2e / 1e3)

    # ---- roofline of the (single) kernel per step ---------------------------------
    flops, bytes_ = algorithmic_counts(cfg)
    peaks = load_peaks()
    achieved_gbs = bytes_ / (ms_step / 1e3) / 1e9
    tflops = flops / (ms_step / 1e3) / 1e12
    traffic = profiled_traffic(cfg.name)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
        "config": config_record(cfg),
        "tflops": tflops,
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                     "traffic": traffic, "peak_source": peaks["source"] + " hbm_gbs (copy)",
                     "algorithmic_bytes_per_launch": bytes_,
                     "algorithmic_flops_per_launch": flops,
                     "tensor_frac_of_bf16_peak": tflops / peaks["bf16_tflops"]},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "clocks": clocks.summary(th0, th1),
        "gpu_launches": args.steps,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(cfg, x).items() if k != "seconds"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

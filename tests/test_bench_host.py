"""Host logic of bench.py on CPU: the multi-rank path (gloo, world size 2), the
weak-scaling arithmetic, the roofline counts and the CPU reference arm."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from comba_workloads import CONFIGS, make_chunk_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports a step time of 1 + r ms: every rank must see the max
        t = bench.max_over_ranks(1.0 + rank, world, "cpu")
        cfg = CONFIGS["tiny_fp32"]
        x = make_chunk_inputs(cfg, seed=bench.rank_seed(cfg, rank))
        digest = float(x["q"].double().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        q.put((rank, t, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, gathered in res:
        assert t == 2.0                    # max over ranks, on every rank
        assert gathered[0] != gathered[1]  # each rank owns its own batch


def test_weak_scaling_value():
    assert bench.weak_scaling_value(32768, 1, 1.0) == pytest.approx(32768e3)
    assert bench.weak_scaling_value(32768, 8, 2.0) == pytest.approx(8 * 32768 / 2e-3)


def test_algorithmic_counts_headline_shape():
    flops, bytes_ = bench.algorithmic_counts(CONFIGS["layer1p3b_bf16"])
    ht = 8 * 4096 * 16
    assert flops == ht * 139264
    assert bytes_ == ht * 1032 + 8 * 16 * 128 * 128 * 4 * 2


def test_reference_arm_prints_one_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_fp32", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=600, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["unit"] == "tokens/s"
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, PYTHONPATH=ROOT, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_fp32", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=600, check=True)
    assert out.stdout.strip() == ""


def test_varlen_workload_is_seeded_and_covers_its_tokens():
    from comba_workloads import VARLEN, make_varlen_inputs, varlen_lengths
    a, b = varlen_lengths(VARLEN), varlen_lengths(VARLEN)
    assert a == b and sum(a) == VARLEN.total_T
    assert all(n >= 1 for n in a) and max(a) <= VARLEN.len_max
    x = make_varlen_inputs(VARLEN)
    cu = x["cu_seqlens"].tolist()
    assert cu[0] == 0 and cu[-1] == VARLEN.total_T and len(cu) == len(a) + 1
    assert tuple(x["q"].shape) == (VARLEN.total_T, VARLEN.Hqk, VARLEN.dk)
    assert tuple(x["v"].shape) == (VARLEN.total_T, VARLEN.H, VARLEN.dv)
    assert tuple(x["S0"].shape) == (len(a), VARLEN.H, VARLEN.dv, VARLEN.dk)
    import bench
    flops, bytes_ = bench.varlen_counts(VARLEN, len(a))
    assert bytes_ < bench.algorithmic_counts(bench.CONFIGS["layer1p3b_bf16"])[1]   # shared q / k heads


def test_backward_flop_and_byte_counts():
    # per 32-token chunk of one chain at dk = dv = 128: prep 2,088,960, states and
    # dstates 2,097,152 each, grads 7,593,984 flops; 16,384 chunks in the 1.3B layer
    per_chunk = 2_088_960 + 2 * 2_097_152 + 7_593_984
    assert bench.bwd_algorithmic_flops(CONFIGS["layer1p3b_bf16"]) == 8 * 16 * 128 * per_chunk
    # a ragged last chunk counts as a whole chunk (the kernels pad it)
    cfg = CONFIGS["layer1p3b_bf16"].replace(B=1, H=1, T=33)
    assert bench.bwd_algorithmic_flops(cfg) == 2 * per_chunk
    # bytes: bf16 q, k, v, dout and fp32 gates read once, fp32 dq, dk, dv, dlog_alpha,
    # dbeta written once, plus d, S0, dS_final, dS0 and dd
    cfg = CONFIGS["layer1p3b_bf16"]
    tok = 8 * 4096 * 16
    want = tok * 512 * 2 + tok * 8 + 16 * 4 + 2 * 128 * 128 * 128 * 4 + tok * 384 * 4 + tok * 8 \
        + 128 * 128 * 128 * 4 + 16 * 4
    assert bench.bwd_algorithmic_bytes(cfg) == want == 1_375_731_840


def test_backward_cpu_baseline_record():
    from comba_workloads import make_cotangents
    cfg = CONFIGS["layer340m_bf16"].replace(B=2, H=2, T=40, dk=16, dv=16, s0_std=0.1)
    x = make_chunk_inputs(cfg, seed=3)
    rec = bench.cpu_baseline_bwd(cfg, x, make_cotangents(cfg, seed=4), target_s=0.05)
    assert rec["kind"] == "oracle" and rec["unit"] == "tokens/s" and rec["cores"] == 1
    assert rec["value"] > 0 and "chains" in rec["sample"]

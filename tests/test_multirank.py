"""The multi-GPU path of bench.py, on CPU with two gloo ranks: every rank gets
its own independent seeded problem (no data-path exchange), the step time is
the max over ranks, and the job throughput counts the work of all ranks."""
from __future__ import annotations

import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from quantized_attention_07_b200 import workloads as W


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.WORKLOADS["small_d64"]
        mine = W.make_inputs(bench.rank_workload(wl, rank))
        # gather a fingerprint of every rank's inputs: problems must differ
        fp = torch.tensor([float(mine.q.float().sum()), float(mine.k.float().sum())])
        allfp = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(allfp, fp)
        local_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        mx = bench.max_over_ranks(local_ms, torch.device("cpu"))
        ops = W.attention_ops(wl)
        q.put((rank, mx, bench.job_throughput(ops, world, 4, mx),
               [t.tolist() for t in allfp]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_independent_problems():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ops = W.attention_ops(W.WORKLOADS["small_d64"])
    for rank, mx, tops, fps in res:
        assert mx == 15.0                                   # max over ranks
        assert tops == pytest.approx(ops * 2 * 4 / 15e-3 / 1e12)
        assert fps[0] != fps[1]                             # independent problems


def test_single_process_defaults():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.rank_workload(W.WORKLOADS["long_32k"], 0) is W.WORKLOADS["long_32k"]


def test_stage1_algorithmic_bytes():
    """Stage 1's roofline numerator: Q and K read at 2 B and coded at 1 B per
    element (6 B per token-channel for the pair), FP8 adds V's 3 B, Q
    smoothing the fp32 per-key mean term; packed batches report none."""
    wl = W.WORKLOADS["long_32k"]
    assert bench.quant_algorithmic_bytes(wl) == 6 * 32 * 32768 * 128
    fp8 = W.WORKLOADS["dit_8k_fp8"]
    el = 24 * 8192 * 64
    assert bench.quant_algorithmic_bytes(fp8) == 9 * el
    sq = W.WORKLOADS["dit_8k_fp8_sq"]
    assert bench.quant_algorithmic_bytes(sq) == 9 * el + 4 * 24 * 64 * 8192
    gqa = W.WORKLOADS["llm_gqa_8k"]
    assert bench.quant_algorithmic_bytes(gqa) == 3 * 8192 * 128 * (32 + 8)
    assert bench.quant_algorithmic_bytes(W.WORKLOADS["varlen_8seq"]) == 0


def test_kernel_hash_ignores_comments_only():
    """The traffic record is keyed by the attention source without comments:
    a comment edit keeps the key, a code edit changes it."""
    src = 'int f(int x) {  // scale\n  /* twice */ return 2 * x;  // "//" stays\n}\nconst char* s = "/*x*/";\n'
    same = 'int f(int x) {\n\n  return 2 * x;   // doubled\n}\nconst char* s = "/*x*/";\n'
    code = 'int f(int x) {  // scale\n  return 3 * x;\n}\nconst char* s = "/*x*/";\n'
    assert bench._code_only(src) == bench._code_only(same)
    assert bench._code_only(src) != bench._code_only(code)
    assert '"/*x*/"' in bench._code_only(src)

"""Benchmark of the SageAttention 8-bit forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic input:
smoothing + quantisation (two HBM-bound kernels) followed by the fused INT8
QK^T / online-softmax / P.V attention kernel, through the library's C ABI.
The metric is 4*B*H*N^2*D / t (halved for causal) in TOPS.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own instance of the
workload (independent problems, no data-path collective: weak scaling); the
time is the max over ranks and `value` counts the work of all ranks.

`--impl reference` times the CPU oracle (the plain restatement of the method)
on the host cores, on a bounded sample of the same workload per step,
extrapolated to the whole step; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_attention_07_b200 import workloads as W  # noqa: E402

METRIC = "SageAttn fwd TOPS (4BHN²D/t) at N=8K–32K, D=64/128; % of INT8/FP8 peak"
DEFAULT_WORKLOAD = "long_32k"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the side workloads timed next to the headline one")
    ap.add_argument("--heads", type=int, default=0,
                    help="override H (smaller cases for profiler captures; not a bench line)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def peaks() -> dict:
    """Roofline denominators from the measured peaks (bf16 GEMM and HBM copy);
    the INT8/FP8 tensor peak is the measured bf16 figure times the nominal
    dense ratio 4.5/2.25 = 2."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    src = "measured"
    try:
        with open(path) as f:
            m = json.load(f)
        bf16, bf16_s, hbm = m["bf16_tflops"], m["bf16_tflops_sustained"], m["hbm_gbs"]
    except (OSError, KeyError, ValueError):
        bf16, bf16_s, hbm, src = 1590.0, 1400.0, 6650.0, "fallback"
    return dict(bf16=bf16, bf16_sustained=bf16_s, int8=2 * bf16, int8_sustained=2 * bf16_s,
                hbm_gbs=hbm, source=src)


def tensor_peak(pk: dict, pv_mode: str, sustained: bool = False) -> float:
    i8 = pk["int8_sustained" if sustained else "int8"]
    b16 = pk["bf16_sustained" if sustained else "bf16"]
    if pv_mode == "fp8":
        return i8                       # INT8 QK^T and FP8 P.V run at the same rate
    return 1.0 / (0.5 / i8 + 0.5 / b16)  # half the ops INT8, half 16-bit


def _code_only(src: str) -> str:
    """C++ source without comments, blank lines and whitespace differences, so
    that an edit of the comments or of the layout does not count as a new
    kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] in "\"'":  # string or character literal, copied as is
            q, j = src[i], i + 1
            while j < n and src[j] != q:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    lines = [" ".join(ln.split()) for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln)


def kernel_hash() -> str:
    """Hash of the attention kernel's code (comments excluded): the key under
    which ncu traffic counters are recorded."""
    h = hashlib.sha256()
    for name in ("attn.cu", "ptx.cuh", "common.cuh", "attn_launch.cuh"):
        with open(os.path.join(ROOT, "quantized_attention_07_b200", "csrc", name),
                  encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, valid only
    while the kernel source is the one the counters were taken on."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("kernel_hash") == kernel_hash():
            return e.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(wl, rank: int):
    """Each rank's independent, seeded instance of the workload (weak scaling)."""
    return wl if rank == 0 else dataclasses.replace(wl, seed=wl.seed + 1000 * rank)


def job_throughput(ops_per_rank: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job TOPS: the work of all ranks over the slowest rank's time."""
    return ops_per_rank * world * steps / (max_ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self) -> dict:
        rows = []
        for line in (self.out or "").splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9:
                rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------- our arm --

def config_of(wl, inp, world: int) -> dict:
    """The `config` object of the JSON line (both arms)."""
    in_bytes = sum(t.numel() * t.element_size() for t in (inp.q, inp.k, inp.v))
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "D": wl.D,
            "Hkv": wl.kv_heads, "qk_gran": wl.qk_gran,
            "in_dtype": wl.dtype, "causal": wl.causal, "pv_mode": wl.pv_mode,
            "seqlens": inp.seqlens if wl.varlen else None,
            "l2": f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB of q,k,v > 126 MiB)"
            if in_bytes > L2_BYTES else "inputs smaller than L2 (no flush)",
            "parallelism": f"replicas x{world}"}


def build_step(wl, inp, dev):
    """The two stages of one step of the workload through the public API, on
    device-resident inputs.  Returns (stage1, stage2, out, ws, launches per
    step, grouped)."""
    import quantized_attention_07_b200 as sage
    from quantized_attention_07_b200 import api

    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    cu = inp.cu_seqlens.to(dev) if inp.cu_seqlens is not None else None
    grouped = not wl.varlen and wl.kv_heads != wl.H
    if grouped:
        # grouped-query attention: the whole public call per step (K, V
        # quantised over the key/value heads, Q over the query heads, then
        # the attention kernel)
        B, H, N, D = q.shape
        out = torch.empty_like(q)
        ws = sage.Workspace(sage.workspace_bytes_gqa(B, H, wl.kv_heads, N, D, wl.pv_mode), dev)

        def stage1():
            pass

        def stage2():
            api.attn_fwd(q, k, v, causal=wl.causal, pv_mode=wl.pv_mode, out=out, workspace=ws)
        launches = 3  # quant_stream_kernel (K, V), quant_stream_kernel (Q), attn_fwd
    elif not wl.varlen:
        B, H, N, D = q.shape
        qz = api.alloc_quantized(B, H, N, D, wl.pv_mode, dev, qk_gran=wl.qk_gran)
        out = torch.empty_like(q)
        ws = sage.Workspace(sage.workspace_bytes(B, H, N, D, wl.pv_mode), dev)

        def stage1():
            api.quantize(q, k, v, wl.pv_mode, qz=qz, workspace=ws, qk_gran=wl.qk_gran,
                         causal=wl.causal)

        def stage2():
            api.attn_quantized(qz, v, causal=wl.causal, out=out, workspace=ws)
        # quant_stream_kernel, attn_fwd_kernel; Q smoothing: Q in its own
        # kernel (quant_q_smooth_kernel) and the mean term (q_smooth_bias_kernel)
        launches = 4 if wl.qk_gran == "block_sq" else 2
    else:
        T, H, D = q.shape
        out = torch.empty_like(q)
        ws = sage.Workspace(sage.workspace_bytes_varlen(T, len(inp.seqlens), H, D, wl.pv_mode), dev)
        maxlen = max(inp.seqlens)

        def stage1():
            pass

        def stage2():
            api.attn_fwd_varlen(q, k, v, cu, maxlen, causal=wl.causal, pv_mode=wl.pv_mode, out=out,
                                workspace=ws)
        launches = 4  # varlen_prep, quant_pass1, quant_pass2, attn_fwd
    return stage1, stage2, out, ws, launches, grouped


def time_steps(stage1, stage2, ws, dev, K: int, warmup: int, local: int, world: int):
    """W untimed steps, then K steps timed with CUDA events on the launching
    stream (bracketed by a barrier and a synchronize), clocks sampled during
    the timed region.  Returns (total ms, per-step stage-2 ms, per-step
    stage-1 ms, clock summary)."""
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(warmup, 3)):
        stage1()
        stage2()
    torch.cuda.synchronize(dev)
    ws.sync_status()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for s in range(K):
            ev[s][0].record(stream)
            stage1()
            ev[s][1].record(stream)
            stage2()
            ev[s][2].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ws.sync_status()
    total_ms = ev[0][0].elapsed_time(ev[K - 1][2])
    attn_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(K)]
    quant_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]
    return total_ms, attn_ms, quant_ms, clk.summary()


# Workloads timed next to the headline one in the same run (1 GPU): the FP8
# P.V configurations (video-DiT D 64, packed causal D 128) and the causal
# LLM block.
SIDE_WORKLOADS = ("dit_8k_fp8", "varlen_8seq", "llm_causal_2k")
SM_COUNT = 148


def mufu_bound_ms(wl, seqlens, sm_mhz: float) -> float:
    """Time of one 2^x per computed score on the special-function units
    (16 per clock per SM): the attention kernel's non-tensor floor."""
    scores = W.attention_ops(wl, seqlens) / (4.0 * wl.D)
    return scores / (16.0 * SM_COUNT * sm_mhz * 1e6) * 1e3


def side_config(name: str, dev, local: int, min_s: float = 0.6) -> dict:
    """One side workload: its step timed like the headline (whole step and the
    attention stage alone), against the tensor peak and the MUFU floor.  The
    timed region lasts at least min_s seconds, so the clock sampler sees it."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    stage1, stage2, _, ws, _, _ = build_step(wl, inp, dev)
    probe_ms, _, _, _ = time_steps(stage1, stage2, ws, dev, 5, 3, local, 1)
    steps = int(min(5000, max(20, min_s * 1e3 / max(probe_ms / 5, 1e-3))))
    total_ms, attn_ms, _, clocks = time_steps(stage1, stage2, ws, dev, steps, 3, local, 1)
    ops = W.attention_ops(wl, inp.seqlens)
    pk = peaks()
    peak = tensor_peak(pk, wl.pv_mode)
    a_ms = statistics.mean(attn_ms)
    achieved = ops / (a_ms * 1e-3) / 1e12
    sm_max = clocks.get("sm_max_mhz") or 1965.0
    mufu = mufu_bound_ms(wl, inp.seqlens, sm_max)
    return {"workload": name, "B": wl.B, "H": wl.H, "N": wl.N, "D": wl.D, "causal": wl.causal,
            "pv_mode": wl.pv_mode, "in_dtype": wl.dtype,
            "seqlens": inp.seqlens if wl.varlen else None,
            "value": round(job_throughput(ops, 1, steps, total_ms), 2),
            "ms_per_step": round(total_ms / steps, 4),
            "attn_ms": round(a_ms, 4), "attn_tops": round(achieved, 2),
            "peak": round(peak, 1), "frac": round(achieved / peak, 4),
            "frac_of_int8_peak": round(achieved / pk["int8"], 4),
            "mufu_bound_ms": round(mufu, 4), "frac_of_mufu_bound": round(mufu / a_ms, 4),
            "mufu_basis": f"one 2^x per computed score, 16/clk/SM x {SM_COUNT} SMs at "
                          f"{sm_max:.0f} MHz",
            "clocks": clocks, "steps": steps}


def run_ours(args, rank, world, local):
    import quantized_attention_07_b200 as sage

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=dev,
                                             timeout=datetime.timedelta(seconds=120))
    wl = W.WORKLOADS[args.workload]
    if args.heads:
        wl = dataclasses.replace(wl, H=args.heads)
    # each rank: its own seeded instance of the workload
    inp = W.make_inputs(rank_workload(wl, rank))
    ops = W.attention_ops(wl, inp.seqlens)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (inp.q, inp.k, inp.v))
    stage1, stage2, out, ws, launches_per_step, grouped = build_step(wl, inp, dev)

    K = args.steps
    total_ms, attn_ms, quant_ms, clocks = time_steps(stage1, stage2, ws, dev, K, args.warmup,
                                                     local, world)
    total_ms = max_over_ranks(total_ms, dev)

    # end to end through the public call with host buffers: pinned H2D of the
    # step's inputs, the forward pass, D2H of the output, every step.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.pin_memory() for x in (inp.q, inp.k, inp.v))
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hcu = inp.cu_seqlens.pin_memory() if inp.cu_seqlens is not None else None

        def e2e_step():
            if wl.varlen:
                # pieces of consecutive sequences: uploads, compute and
                # downloads overlapped
                sage.attn_fwd_varlen_host(hq, hk, hv, hcu, hout, causal=wl.causal,
                                          pv_mode=wl.pv_mode, qk_gran=wl.qk_gran, device=dev)
            else:
                # uploads, compute and downloads of independent head groups overlapped
                sage.attn_fwd_host(hq, hk, hv, hout, causal=wl.causal, pv_mode=wl.pv_mode,
                                   qk_gran=wl.qk_gran, device=dev)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        Ke = max(3, min(K, 10))
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        ws.sync_status()
        h2d = in_bytes + (hcu.numel() * 4 if hcu is not None else 0)
        e2e = {"value": round(job_throughput(ops, world, Ke, ems), 2), "unit": "TOPS",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out.numel() * out.element_size(),
               "steps": Ke}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_throughput(wl, inp, budget_rows=8192, quant_heads=8)
    side = None
    if world == 1 and not args.no_per_config and not args.heads:
        side = {n: side_config(n, dev, local) for n in SIDE_WORKLOADS if n != wl.name}

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    pk = peaks()
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = ops / (attn_avg_ms * 1e-3) / 1e12
    peak = tensor_peak(pk, wl.pv_mode)
    value = job_throughput(ops, world, K, total_ms)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8/fp8" if wl.pv_mode == "fp8" else "int8/fp16",
        "data": "synthetic",
        "config": config_of(wl, inp, world),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(wl.name),
                     "kernel": "attn_fwd_kernel",
                     "peak_basis": f"{pk['source']}: bf16 GEMM burst {pk['bf16']} TF/s; INT8/FP8 = 2x bf16; "
                                   + ("FP8 P.V: INT8/FP8 peak" if wl.pv_mode == "fp8"
                                      else "16-bit P.V: harmonic mix of INT8 (QK^T) and bf16 (P.V) peaks"),
                     "frac_of_int8_peak": round(achieved / pk["int8"], 4),
                     "attn_ms": round(attn_avg_ms, 4), "quant_ms": round(statistics.mean(quant_ms), 4)},
        "clocks": clocks,
        "gpu_launches": launches_per_step * K,
    }
    qb = quant_algorithmic_bytes(wl)
    if qb and not grouped and not wl.varlen:
        # stage 1 (K smoothing + quantisation) against the copy bandwidth
        qms = statistics.mean(quant_ms)
        gbs = qb / (qms * 1e-3) / 1e9
        line["quantisation"] = {"bound": "hbm", "ms": round(qms, 4), "algorithmic_bytes": qb,
                                "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                                "frac": round(gbs / pk["hbm_gbs"], 4),
                                "launches_per_step": launches_per_step - 1}
    if e2e:
        line["e2e"] = e2e
    if cpu:
        line["cpu_baseline"] = cpu
    if side:
        line["per_config"] = side
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- oracle arm --

def quant_algorithmic_bytes(wl) -> int:
    """Bytes stage 1 must move for a dense workload: Q and K read (2 B per
    element) and their int8 codes written (1 B), FP8 P.V: V read and its e4m3
    codes written (3 B); per-token deltas 4 B per row of Q and K; Q smoothing:
    the fp32 per-key mean term written (4 B per query block and key).  The
    second pass over K (its mean first) is overhead, not counted."""
    if wl.varlen:
        return 0
    NB = (wl.N + 127) // 128
    q_el = wl.B * wl.H * wl.N * wl.D
    kv_el = wl.B * wl.kv_heads * wl.N * wl.D
    b = 3 * q_el + 3 * kv_el + (3 * kv_el if wl.pv_mode == "fp8" else 0)
    if wl.qk_gran == "token":
        b += 4 * wl.N * (wl.B * wl.H + wl.B * wl.kv_heads)
    if wl.qk_gran == "block_sq":
        b += 4 * wl.B * wl.H * NB * NB * 128
    return b


def cpu_oracle_throughput(wl, inp, budget_rows: int, quant_heads: int, seed: int = 7) -> dict:
    """Time the CPU oracle (quantisation + emulated attention rows) on a bounded
    sample of the workload and extrapolate to the whole of it."""
    import numpy as np

    import oracle
    from oracle import heads

    oracle.build()
    lens = inp.seqlens
    H = wl.H
    hs = min(quant_heads, H)
    k_in, v_in = inp.k, inp.v
    if not wl.varlen and wl.kv_heads != H:  # grouped-query: the oracle sees repeated K, V
        k_in, v_in = heads.repeat_kv(k_in, H // wl.kv_heads), heads.repeat_kv(v_in, H // wl.kv_heads)
    # quantisation of `hs` heads (all sequences), timed
    sl = lambda x: x[:, :hs].contiguous()
    qh, kh, vh = sl(inp.q), sl(k_in), sl(v_in)
    t0 = time.perf_counter()
    qz = heads.quantize(qh, kh, vh, inp.cu_seqlens, wl.pv_mode, gran=wl.qk_gran)
    t_quant = time.perf_counter() - t0
    # emulated rows, drawn over the quantised heads
    picks = [p for p in W.sample_rows(lens, hs, budget_rows, seed) if p[1] < hs]
    t0 = time.perf_counter()
    heads.emulate_rows(qz, vh, inp.cu_seqlens, picks, wl.D, wl.causal, wl.pv_mode,
                       gran=wl.qk_gran, k=kh if wl.qk_gran == "block_sq" else None)
    t_rows = time.perf_counter() - t0

    def work(i):  # key pairs of row i
        return (i + 1) if wl.causal else None

    if wl.causal:
        total_pairs = H * sum(n * (n + 1) / 2 for n in lens)
        sample_pairs = sum(i + 1 for _, _, i in picks)
    else:
        total_pairs = H * sum(n * n for n in lens)
        sample_pairs = sum(lens[s] for s, _, _ in picks)
    t_total = t_quant * H / hs + t_rows * total_pairs / sample_pairs
    ops = W.attention_ops(wl, lens)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(ops / t_total / 1e12, 6), "unit": "TOPS", "cores": cores,
            "kind": "oracle", "measured_s": round(t_quant + t_rows, 3),
            "projected_s": round(t_total, 1),
            "sample": f"quantisation of {hs}/{H} heads + {len(picks)} emulated query rows, "
                      f"extrapolated by heads and by (query,key) pairs; measured "
                      f"{t_quant + t_rows:.1f} s of CPU time, {t_total:.0f} s projected"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    inp = W.make_inputs(wl)
    K = args.steps
    vals = []
    for s in range(max(args.warmup, 3) + K):
        r = cpu_oracle_throughput(wl, inp, budget_rows=256, quant_heads=1, seed=100 + s)
        if s >= max(args.warmup, 3):
            vals.append(r)
    # value: the whole workload's work over the oracle's projected time for it;
    # ms_per_step: what each (bounded) step took on the host cores
    ops = W.attention_ops(wl, inp.seqlens)
    t_steps = [ops / (r["value"] * 1e12) for r in vals]
    value = ops * K / sum(t_steps) / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(1e3 * sum(r["measured_s"] for r in vals) / K, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8/fp8" if wl.pv_mode == "fp8" else "int8/fp16", "data": "synthetic",
        "config": config_of(wl, inp, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": vals[0]["cores"],
                         "kind": "oracle",
                         "sample": "per step: " + vals[0]["sample"],
                         "projected_ms_per_workload": round(1e3 * sum(t_steps) / K, 1)},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()

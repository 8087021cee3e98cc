"""Helpers shared by the GPU parity tests: run the CUDA library and the CPU
oracle on the same seeded host tensors and compare."""
from __future__ import annotations

import numpy as np
import torch

import quantized_attention_07_b200 as sage
from oracle import heads

# Tolerances on the fp32 output against the oracle's emulation of the plain
# method (max abs): the contract.
TOL = {"fp16": 2e-3, "fp8": 8e-3}

# Agreement of the fp32 output with the oracle's emulation in the library's
# own evaluation order (see `schedule`).  There the two sides take every
# integer decision alike and round every p to P from the same maximum; what
# is left is the special-function unit's 2^x (a few fp32 ulps), the order of
# the sums inside one MMA and of the row sum l, and the reciprocal of l in the
# epilogue, all ~1e-6 relative -- except where a p lies within those few ulps
# of a rounding boundary of its 16- or 8-bit format and the two sides round
# it apart: one such p moves its whole row by up to 2^-8 (bf16) or 2^-4 (e4m3)
# of that p's share of the row, ~1e-3 on short rows.  Such rows are rare
# (measured between two emulations: < 0.5 % of rows above 1e-5).  So the
# check is on the bulk, with room for those rows:
#   median |GPU - E_sched| <= 1e-6, 99th percentile <= 2e-5, and at most 2 % of
#   the rows with a deviation above 1e-4.
# A wrong scale, sub-tile, rescale or flush moves the bulk and fails it.
TIGHT = dict(median=1e-6, q99=2e-5, row=1e-4, row_frac=0.02)


def schedule(pv_mode: str, v_dtype: torch.dtype, qk_gran: str = "block") -> dict:
    """The evaluation order of the CUDA kernels, as oracle emulation options.

    FP8 P.V: the plain running maximum over 128-key blocks, the P scale 448
    applied in the exponent (p = 2^(arg + log2 448)), l summing those scaled p.
    16-bit P.V with bf16 P: the plain method.  16-bit P.V with fp16 P: the
    maximum taken per 64-key sub-tile and moved only when it rises by more
    than 8 (base 2).  Q smoothing: the mean term as fp32 fused multiply-adds
    in channel order."""
    if pv_mode == "fp8":
        opt = dict(kv=128, tau=0.0, p8_exp=True)
    elif v_dtype == torch.bfloat16:
        opt = dict(kv=128, tau=0.0)
    else:
        opt = dict(kv=64, tau=8.0)
    if qk_gran == "block_sq":
        opt["bias_order"] = "fma"
    return opt


def half_ulp(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Half a unit in the last place of |x| in the given 16-bit format."""
    mant, emin = (10, -14) if dtype == torch.float16 else (7, -126)
    a = np.abs(x.astype(np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return 0.5 * np.exp2(e - mant)


def gpu_quantize_dense(q, k, v, pv_mode, qk_gran="block", causal=False, sm_scale=None):
    dev = torch.device("cuda")
    qz = sage.quantize(q.to(dev), k.to(dev), v.to(dev) if v is not None else None, pv_mode,
                       qk_gran=qk_gran, causal=causal, sm_scale=sm_scale)
    torch.cuda.synchronize()
    sage.sync_status()
    return qz


def assert_same(name: str, got: np.ndarray, want: np.ndarray) -> None:
    """Bit-exact equality; on failure, report where and by how much."""
    assert got.shape == want.shape, f"{name}: shape {got.shape} != {want.shape}"
    if np.array_equal(got, want):
        return
    bad = np.argwhere(got != want)
    head = [(tuple(int(i) for i in ix), got[tuple(ix)].item(), want[tuple(ix)].item())
            for ix in bad[:8]]
    raise AssertionError(f"{name}: {len(bad)} of {got.size} differ; first (index, got, want): {head}")


def compare_quant_dense(qz_gpu, qz_ref, pv_mode):
    c = lambda t: t.cpu().numpy()
    assert_same("q deltas", c(qz_gpu.q_scale), qz_ref.q_delta)
    assert_same("q codes", c(qz_gpu.q_codes), qz_ref.q_codes)
    assert_same("k mean", c(qz_gpu.k_mean), qz_ref.k_mean)
    assert_same("k deltas", c(qz_gpu.k_scale), qz_ref.k_delta)
    assert_same("k codes", c(qz_gpu.k_codes), qz_ref.k_codes)
    if pv_mode == "fp8":
        assert_same("v deltas", c(qz_gpu.v_scale), qz_ref.v_delta)
        assert_same("v codes", c(qz_gpu.v_codes), qz_ref.v_codes)


def compare_quant_varlen(qz_gpu, qz_ref, cu, pv_mode):
    """Varlen code arrays are [H, TBmax*128, D]; only the first TB blocks are written."""
    c = lambda t: t.cpu().numpy()
    TB = qz_ref.q_delta.shape[1]
    assert_same("q deltas", c(qz_gpu.q_scale)[:, :TB], qz_ref.q_delta)
    assert_same("q codes", c(qz_gpu.q_codes)[:, :TB * 128], qz_ref.q_codes)
    assert_same("k mean", c(qz_gpu.k_mean), qz_ref.k_mean)
    assert_same("k deltas", c(qz_gpu.k_scale)[:, :TB], qz_ref.k_delta)
    assert_same("k codes", c(qz_gpu.k_codes)[:, :TB * 128], qz_ref.k_codes)
    if pv_mode == "fp8":
        assert_same("v deltas", c(qz_gpu.v_scale), qz_ref.v_delta)
        assert_same("v codes", c(qz_gpu.v_codes), qz_ref.v_codes)


def run_dense(q, k, v, causal, pv_mode, out_dtype=torch.float32, sm_scale=None,
              qk_gran="block"):
    dev = torch.device("cuda")
    out = sage.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, sm_scale=sm_scale,
                        pv_mode=pv_mode, out_dtype=out_dtype, qk_gran=qk_gran)
    torch.cuda.synchronize()
    sage.sync_status()
    return out.cpu()


def run_varlen(q, k, v, cu, causal, pv_mode, out_dtype=torch.float32, sm_scale=None,
               qk_gran="block"):
    dev = torch.device("cuda")
    lens = (cu[1:] - cu[:-1]).tolist()
    out = sage.attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), max(lens) if lens else 0,
                               causal=causal, sm_scale=sm_scale, pv_mode=pv_mode,
                               out_dtype=out_dtype, qk_gran=qk_gran)
    torch.cuda.synchronize()
    sage.sync_status()
    return out.cpu()


def gather(out: torch.Tensor, picks, cu=None) -> np.ndarray:
    o = out.float().numpy()
    if cu is None:
        return np.stack([o[s, h, i] for s, h, i in picks])
    c = cu.tolist()
    return np.stack([o[c[s] + i, h] for s, h, i in picks])


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    a = a.astype(np.float64).ravel(); b = b.astype(np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def check_against_oracle(q, k, v, cu, causal, pv_mode, picks, sm_scale=None,
                         ref_cos_bar=0.999, qk_gran="block", tight=TIGHT):
    """GPU fp32 output vs the oracle's emulation of the plain method (max-abs
    tolerance TOL, the contract), vs the emulation in the library's evaluation
    order (the bulk statistics of `tight`), and vs the fp64 reference
    (cosine).  Also checks a
    16-bit output run against the plain emulation.  Returns a stats dict.
    Dense k, v with fewer heads than q run grouped-query attention on the GPU;
    the oracle sees them repeated (its repeat_kv)."""
    D = q.shape[-1]
    if cu is None:
        out32 = run_dense(q, k, v, causal, pv_mode, torch.float32, sm_scale, qk_gran)
        out16 = run_dense(q, k, v, causal, pv_mode, q.dtype, sm_scale, qk_gran)
        if k.shape[1] != q.shape[1]:
            g = q.shape[1] // k.shape[1]
            k, v = heads.repeat_kv(k, g), heads.repeat_kv(v, g)
    else:
        out32 = run_varlen(q, k, v, cu, causal, pv_mode, torch.float32, sm_scale, qk_gran)
        out16 = run_varlen(q, k, v, cu, causal, pv_mode, q.dtype, sm_scale, qk_gran)
        if k.shape[1] != q.shape[1]:
            g = q.shape[1] // k.shape[1]
            k, v = heads.repeat_kv_packed(k, g), heads.repeat_kv_packed(v, g)
    qz = heads.quantize(q, k, v, cu, pv_mode, gran=qk_gran)
    kk = k if qk_gran == "block_sq" else None
    emu = heads.emulate_rows(qz, v, cu, picks, D, causal, pv_mode, sm_scale, gran=qk_gran, k=kk)
    sched = schedule(pv_mode, v.dtype, qk_gran)
    emu_s = heads.emulate_rows(qz, v, cu, picks, D, causal, pv_mode, sm_scale, gran=qk_gran, k=kk,
                               **sched)
    ref = heads.reference_rows(q, k, v, cu, picks, causal, sm_scale)
    E = np.stack([emu[p] for p in picks])
    Es = np.stack([emu_s[p] for p in picks])
    R = np.stack([ref[p] for p in picks])
    G = gather(out32, picks, cu)
    G16 = gather(out16, picks, cu)
    tol = TOL[pv_mode]
    err = np.abs(G - E)
    err_s = np.abs(G - Es)
    err16 = np.abs(G16 - E) - half_ulp(E, q.dtype)
    row_s = err_s.max(axis=1)
    stats = dict(max_abs=float(err.max()), max_abs16=float(err16.max()),
                 sched_median=float(np.median(err_s)), sched_q99=float(np.quantile(err_s, 0.99)),
                 sched_rows_over=float((row_s > tight["row"]).mean()),
                 max_abs_sched=float(err_s.max()), plain_vs_sched=float(np.abs(E - Es).max()),
                 cos_gpu_ref=cosine(G, R), cos_emu_ref=cosine(E, R))
    assert np.isfinite(G).all()
    assert err.max() <= tol, stats
    assert err16.max() <= tol, stats
    assert err_s.max() <= tol, stats
    assert stats["sched_median"] <= tight["median"], stats
    assert stats["sched_q99"] <= tight["q99"], stats
    assert stats["sched_rows_over"] <= tight["row_frac"], stats
    bar = min(ref_cos_bar, stats["cos_emu_ref"] - 1e-4)
    assert stats["cos_gpu_ref"] >= bar, stats
    return stats

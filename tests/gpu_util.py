"""Helpers shared by the GPU parity tests: run the CUDA library and the CPU
oracle on the same seeded host tensors and compare."""
from __future__ import annotations

import numpy as np
import torch

import quantized_attention_07_b200 as sage
from oracle import heads

# Tolerances on the fp32 output against the oracle's emulation (max abs).
TOL = {"fp16": 2e-3, "fp8": 8e-3}


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
                         ref_cos_bar=0.999, qk_gran="block"):
    """GPU fp32 output vs the oracle's emulation (max-abs tolerance) and the fp64
    reference (cosine).  Also checks a 16-bit output run.  Returns a stats dict.
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
    emu = heads.emulate_rows(qz, v, cu, picks, D, causal, pv_mode, sm_scale, gran=qk_gran,
                             k=k if qk_gran == "block_sq" else None)
    ref = heads.reference_rows(q, k, v, cu, picks, causal, sm_scale)
    E = np.stack([emu[p] for p in picks])
    R = np.stack([ref[p] for p in picks])
    G = gather(out32, picks, cu)
    G16 = gather(out16, picks, cu)
    tol = TOL[pv_mode]
    err = np.abs(G - E)
    err16 = np.abs(G16 - E) - half_ulp(E, q.dtype)
    stats = dict(max_abs=float(err.max()), max_abs16=float(err16.max()),
                 cos_gpu_ref=cosine(G, R), cos_emu_ref=cosine(E, R))
    assert np.isfinite(G).all()
    assert err.max() <= tol, stats
    assert err16.max() <= tol, stats
    bar = min(ref_cos_bar, stats["cos_emu_ref"] - 1e-4)
    assert stats["cos_gpu_ref"] >= bar, stats
    return stats

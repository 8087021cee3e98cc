"""GPU parity: the CUDA library against the CPU oracle on the same seeded inputs.

  * quantisation outputs (codes, deltas, K mean, FP8 V codes/scales): bit-exact,
  * the int32 QK^T scores of the fused attention kernel itself: bit-exact,
  * attention output: within the stated max-abs tolerance of the oracle's
    emulation of the plain method (fp32 output, and 16-bit output with half an
    ulp of slack), within 1e-4 of the emulation in the library's evaluation
    order, and cosine >= 0.999 against the fp64 reference (or, where the
    method's own accuracy is lower, no worse than the emulation's cosine).
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_07_b200 as sage
from oracle import heads
from quantized_attention_07_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_07_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


# ----------------------------------------------------------- quantisation --

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("N", [1, 127, 300, 1000])
@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
def test_quantize_bit_exact_small(D, dtype, N, pv_mode):
    q, k, v = W.make_dense(2, 3, N, D, dtype, bias_sigma=3.0, outlier_p=0.01, outlier_scale=20.0,
                           seed=1000 + N + D)
    qz = U.gpu_quantize_dense(q, k, v, pv_mode)
    U.compare_quant_dense(qz, heads.quantize(q, k, v, None, pv_mode), pv_mode)


@pytest.mark.parametrize("name", [n for n, w in W.WORKLOADS.items() if w.kv_heads == w.H])
def test_quantize_bit_exact_full_workloads(name):
    """(The grouped-query workload's quantisation runs inside attn_fwd; its codes
    are checked through the attention tests in test_gpu_gqa.py.)"""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    ref = heads.quantize(inp.q, inp.k, inp.v, inp.cu_seqlens, wl.pv_mode, gran=wl.qk_gran)
    if wl.varlen:
        dev = torch.device("cuda")
        qz = sage.quantize_varlen(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev),
                                  inp.cu_seqlens.to(dev), max(inp.seqlens), wl.pv_mode)
        torch.cuda.synchronize()
        sage.sync_status()
        U.compare_quant_varlen(qz, ref, inp.cu_seqlens, wl.pv_mode)
    else:
        qz = U.gpu_quantize_dense(inp.q, inp.k, inp.v, wl.pv_mode, wl.qk_gran)
        U.compare_quant_dense(qz, ref, wl.pv_mode)


@pytest.mark.parametrize("D,dtype,pv_mode", [(64, "bf16", "fp8"), (128, "fp16", "fp16")])
def test_quantize_bit_exact_many_heads_ragged(D, dtype, pv_mode):
    """Many heads of a long ragged sequence: the dense quantiser interleaves the
    pass-1 blocks of later heads with the pass-2 blocks of earlier ones."""
    q, k, v = W.make_dense(2, 20, 8000, D, dtype, bias_sigma=3.0, outlier_p=0.01,
                           outlier_scale=20.0, seed=4242 + D)
    qz = U.gpu_quantize_dense(q, k, v, pv_mode)
    U.compare_quant_dense(qz, heads.quantize(q, k, v, None, pv_mode), pv_mode)


def test_constant_k_channels_give_zero_codes():
    """K constant over tokens: the smoothed K is exactly zero (mean is exact)."""
    q, k, v = W.make_dense(1, 2, 333, 128, "fp16", bias_sigma=5.0, seed=7, k_const_over_tokens=True)
    qz = U.gpu_quantize_dense(q, k, v, "fp16")
    assert not qz.k_codes.any().item() and not qz.k_scale.any().item()
    assert torch.equal(qz.k_mean.cpu(), k[:, :, 0, :].float())


def test_quant_qk_bit_exact_and_equal_to_quantize():
    """sage_quant_qk (Q and K only) against the oracle, and equal to the Q/K
    outputs of sage_quantize."""
    q, k, v = W.make_dense(2, 3, 777, 128, "bf16", bias_sigma=3.0, seed=91)
    dev = torch.device("cuda")
    qz = sage.quant_qk(q.to(dev), k.to(dev))
    torch.cuda.synchronize()
    sage.sync_status()
    U.compare_quant_dense(qz, heads.quantize(q, k, v, None, "fp16"), "fp16")
    full = U.gpu_quantize_dense(q, k, v, "fp16")
    for a in ("q_codes", "q_scale", "k_codes", "k_scale", "k_mean"):
        assert torch.equal(getattr(qz, a), getattr(full, a)), a


# ----------------------------------------------------------- INT8 QK^T --

def _random_codes(B, H, N, D, seed):
    """int8 codes in [-127, 127] with padding rows 0, and rows of +-127 for the
    extreme products (|S| up to 127^2 D)."""
    rng = np.random.default_rng(seed)
    NP = (N + 127) // 128 * 128
    qc = rng.integers(-127, 128, size=(B, H, NP, D)).astype(np.int8)
    kc = rng.integers(-127, 128, size=(B, H, NP, D)).astype(np.int8)
    qc[:, :, N:] = 0
    kc[:, :, N:] = 0
    qc[:, :, 5] = 127
    qc[:, :, N - 1] = -127
    kc[:, :, 9] = -127
    kc[:, :, 70] = 127      # second 64-key half of the first block
    kc[:, :, N - 1] = 127
    return qc, kc


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 777])
def test_attention_kernel_s_bit_exact(D, pv_mode, causal, N):
    """The int32 S = Q^ K^T of the fused attention kernel itself, stored as it
    reads each 64-key sub-tile from tensor memory, equals the oracle's exact
    integer product on every (row, key) the kernel visits: first, last,
    diagonal and ragged-tail blocks, both 64-key halves of each block, the
    extremes +-127^2 D; nothing outside the visited sub-tiles is written.  The
    diagnostic build's output equals the product build's bit for bit."""
    B, H = 1, 2
    qc, kc = _random_codes(B, H, N, D, seed=N + D)
    NP = qc.shape[2]
    rng = np.random.default_rng(7)
    dev = torch.device("cuda")
    fp8 = pv_mode == "fp8"
    qz = sage.alloc_quantized(B, H, N, D, pv_mode, dev)
    qz.q_codes.copy_(torch.from_numpy(qc))
    qz.k_codes.copy_(torch.from_numpy(kc))
    qz.q_scale.copy_(torch.from_numpy(rng.uniform(0.5e-3, 2e-3, qz.q_scale.shape).astype(np.float32)))
    qz.k_scale.copy_(torch.from_numpy(rng.uniform(0.5e-3, 2e-3, qz.k_scale.shape).astype(np.float32)))
    v = torch.randn(B, H, N, D, generator=torch.Generator().manual_seed(3)).half().to(dev)
    if fp8:
        codes = rng.integers(0, 0x7E, size=qz.v_codes.shape) | (rng.integers(0, 2, size=qz.v_codes.shape) << 7)
        qz.v_codes.copy_(torch.from_numpy(codes.astype(np.uint8)))
        qz.v_scale.copy_(torch.from_numpy(rng.uniform(0.001, 0.01, qz.v_scale.shape).astype(np.float32)))
    out_d, S = sage.attn_quantized_dump_s(qz, v, causal=causal)
    out = sage.attn_quantized(qz, v, causal=causal, out_dtype=torch.float32)
    torch.cuda.synchronize()
    sage.sync_status()
    assert torch.equal(out_d, out)
    S = S.cpu().numpy().reshape(B * H, NP, NP)
    ns = (N + 63) // 64
    rows = np.arange(NP)[:, None]
    keys = np.arange(NP)[None, :]
    visited = (rows < N) & (keys < ns * 64)
    if causal:
        visited &= keys < (rows // 128 + 1) * 128
    for bh in range(B * H):
        want = oracle.qk_int(qc[0, bh], kc[0, bh], 0, NP, 0, NP)
        U.assert_same(f"S head {bh}", S[bh][visited], want[visited])
        assert np.all(S[bh][~visited] == -2 ** 31), "the kernel wrote outside its sub-tiles"
    assert np.abs(S[:, :N, :N]).max() == 127 * 127 * D


def test_attention_kernel_s_of_a_quantised_workload():
    """The same dump on the codes of a quantised causal LLM-shaped input."""
    q, k, v = W.make_dense(1, 2, 1000, 128, "fp16", 3.0, seed=20260002)
    dev = torch.device("cuda")
    qz = sage.quantize(q.to(dev), k.to(dev), v.to(dev), "fp8")
    _, S = sage.attn_quantized_dump_s(qz, v.to(dev), causal=True)
    torch.cuda.synchronize()
    sage.sync_status()
    qc, kc = qz.q_codes.cpu().numpy(), qz.k_codes.cpu().numpy()
    S = S.cpu().numpy()
    NP = qc.shape[2]
    rows, keys = np.arange(NP)[:, None], np.arange(NP)[None, :]
    visited = (rows < 1000) & (keys < (rows // 128 + 1) * 128) & (keys < 1024)
    for bh in range(2):
        want = qc[0, bh].astype(np.int64) @ kc[0, bh].astype(np.int64).T
        assert np.array_equal(S[bh][visited].astype(np.int64), want[visited])


@pytest.mark.parametrize("D", [64, 128])
def test_qk_int8_tiles_bit_exact(D):
    rng = np.random.default_rng(D)
    B, H, NP = 1, 3, 512
    qc = torch.from_numpy(rng.integers(-127, 128, size=(B, H, NP, D)).astype(np.int8))
    kc = torch.from_numpy(rng.integers(-127, 128, size=(B, H, NP, D)).astype(np.int8))
    qc[0, 1, 5, :] = 127
    kc[0, 1, 9, :] = -127                       # extreme products
    tiles = [(0, 0, 0), (1, 0, 0), (1, 3, 2), (2, 1, 3), (2, 3, 3)]
    S = sage.qk_int8_tiles(qc.cuda(), kc.cuda(), tiles).cpu().numpy()
    sage.sync_status()
    for t, (bh, I, J) in enumerate(tiles):
        ref = oracle.qk_int(qc[0, bh].numpy(), kc[0, bh].numpy(), I * 128, 128, J * 128, 128)
        assert np.array_equal(S[t], ref), (bh, I, J)


def test_qk_int8_tiles_of_quantised_workload():
    wl = W.WORKLOADS["llm_causal_2k"]
    q, k, v = W.make_dense(1, 2, 2048, 128, "bf16", 3.0, seed=wl.seed)
    qz = U.gpu_quantize_dense(q, k, v, "fp16")
    tiles = [(0, 0, 0), (0, 15, 15), (1, 15, 0), (1, 7, 8), (0, 3, 12)]
    S = sage.qk_int8_tiles(qz.q_codes, qz.k_codes, tiles).cpu().numpy()
    qc, kc = qz.q_codes.cpu().numpy(), qz.k_codes.cpu().numpy()
    for t, (bh, I, J) in enumerate(tiles):
        ref = qc[0, bh, I * 128:(I + 1) * 128].astype(np.int64) @ \
            kc[0, bh, J * 128:(J + 1) * 128].astype(np.int64).T
        assert np.array_equal(S[t].astype(np.int64), ref)


# ------------------------------------------------------------- attention --

SMALL = [
    # (B, H, N, D, dtype, causal, pv_mode)
    (1, 2, 256, 64, "fp16", False, "fp16"),
    (1, 2, 256, 128, "fp16", False, "fp16"),
    (2, 1, 300, 128, "bf16", True, "fp16"),
    (1, 2, 777, 64, "bf16", False, "fp16"),
    (1, 2, 777, 64, "fp16", True, "fp16"),
    (1, 1, 1, 128, "fp16", False, "fp16"),
    (1, 1, 1, 64, "bf16", True, "fp8"),
    (1, 2, 127, 128, "fp16", True, "fp8"),
    (1, 2, 640, 64, "fp16", False, "fp8"),
    (2, 2, 513, 128, "bf16", False, "fp8"),
    (1, 2, 1000, 128, "bf16", True, "fp8"),
    (1, 3, 129, 64, "fp16", True, "fp16"),
]


@pytest.mark.parametrize("B,H,N,D,dtype,causal,pv_mode", SMALL)
def test_attention_small_all_rows(B, H, N, D, dtype, causal, pv_mode):
    q, k, v = W.make_dense(B, H, N, D, dtype, bias_sigma=3.0, seed=N * 7 + D)
    picks = [(b * H + h, h, i) for b in range(B) for h in range(H) for i in range(N)]
    # dense picks index [B, H] as (b, h); emulate/reference take (seq=b, head=h)
    picks = [(b, h, i) for b in range(B) for h in range(H) for i in range(N)]
    U.check_against_oracle(q, k, v, None, causal, pv_mode, picks)


def test_attention_custom_scale():
    q, k, v = W.make_dense(1, 2, 384, 64, "fp16", 2.0, seed=5)
    picks = [(0, h, i) for h in range(2) for i in range(0, 384, 5)]
    U.check_against_oracle(q, k, v, None, False, "fp16", picks, sm_scale=0.05)


def test_attention_varlen_small():
    lens = [1, 129, 300, 0, 511, 64]
    for causal, pv_mode, dt in ((True, "fp8", "bf16"), (False, "fp16", "fp16"),
                                (True, "fp16", "bf16"), (False, "fp8", "fp16")):
        q, k, v, cu = W.make_varlen(lens, 2, 128 if pv_mode == "fp8" else 64, dt, seed=11)
        picks = [(s, h, i) for s, n in enumerate(lens) for h in range(2) for i in range(n)]
        U.check_against_oracle(q, k, v, cu, causal, pv_mode, picks)


# The method's own accuracy on each workload (oracle emulation vs fp64 on the
# sampled rows), written by tests/golden/make_accuracy_ceiling.py.
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                       "accuracy_ceiling.json")) as _f:
    CEILING = json.load(_f)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_attention_full_workloads_sampled_rows(name):
    """Each workload at full size, in the launch configuration the benchmark
    times; the oracle checks 512 seeded rows (all rows for the small one).
    The cosine bar against fp64 is 0.999, or the method's recorded ceiling
    minus 1e-4 where that is lower (the outlier workloads)."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    lens = inp.seqlens
    if wl.varlen:
        picks = W.sample_rows(lens, wl.H, 512, seed=wl.seed)
    elif wl.B * wl.H * wl.N <= 4096:
        picks = [(b, h, i) for b in range(wl.B) for h in range(wl.H) for i in range(wl.N)]
    else:
        flat = W.sample_rows([wl.N] * wl.B, wl.H, 512, seed=wl.seed)
        picks = flat
    rec = CEILING[name]["cosine_emulation_vs_fp64"]
    stats = U.check_against_oracle(inp.q, inp.k, inp.v, inp.cu_seqlens, wl.causal, wl.pv_mode,
                                   picks, qk_gran=wl.qk_gran, ref_cos_bar=min(0.999, rec - 1e-4))
    print(name, stats)
    assert abs(stats["cos_emu_ref"] - rec) <= 1e-6   # the recorded ceiling is this run's

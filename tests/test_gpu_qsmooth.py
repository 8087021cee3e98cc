"""Q smoothing (SageAttention2's smoothing of Q: "SageAttention v1/v2/v2++/v3
overview", SageAttention2 bullet 2): the GPU block means, codes and deltas of
the smoothed Q equal the oracle's bit for bit, the per-key mean term lies
within the fp32 error bound of the plain fp64 term (and equals the fixed-order
fp32 form bit for bit), the attention output matches the oracle's smoothed
emulation, and on queries with a channel offset smoothing is more accurate
than plain per-block deltas."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_07_b200 as sage
from quantized_attention_07_b200 import workloads as W
from oracle import heads

from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_07_b200 import build
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _inputs(B, H, Hkv, N, D, dtype, seed, q_off=3.0):
    q, k, v = W.make_dense(B, H, N, D, dtype, bias_sigma=3.0, seed=seed, q_bias_sigma=q_off)
    return q, k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()


def _check_bias(qz, ref, k_rep, H, N, causal, sm_scale):
    """GPU q_bias against the oracle's term.

    Contract: the plain term fp32(kappa * qmean . k~) (fp64 dot product,
    rounded once), within the error bound of an fp32 evaluation: D fused
    multiply-adds and one multiplication by kappa, each rounded once, give
    |got - want| <= (D + 2) * 2^-24 * kappa * sum_d |qmean_d k~_d| (the standard
    bound of recursive summation, gamma_D <= (D + 1) u for D u < 2^-10, plus
    the final rounding of the fp64 side).
    Evaluation order: the term as fp32 fused multiply-adds in channel order,
    bit for bit.
    k_rep: K with the key/value heads repeated to the query heads (ref
    quantised from it)."""
    got = qz.q_bias.cpu().numpy()
    NB = (N + 127) // 128
    kf = k_rep.float().numpy()
    B, D = k_rep.shape[0], k_rep.shape[-1]
    kap = float(oracle.kappa(sm_scale))
    for b in range(B):
        for h in range(H):
            want = oracle.q_smooth_bias(ref.q_mean[b, h], kf[b, h], ref.k_mean[b, h], sm_scale,
                                        ldo=NB * 128)
            want_fma = oracle.q_smooth_bias(ref.q_mean[b, h], kf[b, h], ref.k_mean[b, h], sm_scale,
                                            ldo=NB * 128, order="fma")
            ks = (kf[b, h] - ref.k_mean[b, h][None, :]).astype(np.float32).astype(np.float64)
            absdot = np.abs(ref.q_mean[b, h].astype(np.float64)) @ np.abs(ks).T  # [NB, N]
            bound = (D + 2) * 2.0 ** -24 * kap * absdot + 2.0 ** -149
            g = got[b, h][:, :N]
            if causal:  # blocks I < J are not written (the mask hides them)
                J = np.arange(N) // 128
                keep = np.arange(NB)[:, None] >= J[None, :]
            else:
                keep = np.ones_like(g, dtype=bool)
            err = np.abs(g.astype(np.float64) - want[:, :N].astype(np.float64))
            assert np.all(err[keep] <= bound[keep]), (b, h, float((err - bound)[keep].max()))
            U.assert_same(f"mean term b{b} h{h}", g[keep], want_fma[:, :N][keep])
            if not causal:
                assert np.all(got[b, h][:, N:] == 0)  # keys past N


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal,pv_mode", [
    (1, 2, 2, 300, 64, "fp16", False, "fp16"),
    (2, 2, 1, 1000, 128, "bf16", True, "fp8"),
    (1, 4, 2, 128, 128, "fp16", False, "fp8"),
    (1, 1, 1, 1, 64, "bf16", True, "fp16"),
])
def test_smoothed_quantisation_and_term(B, H, Hkv, N, D, dtype, causal, pv_mode):
    q, k, v = _inputs(B, H, Hkv, N, D, dtype, seed=91 + N + D)
    sm = oracle.default_sm_scale(D)
    qz = U.gpu_quantize_dense(q, k, v, pv_mode, qk_gran="block_sq", causal=causal, sm_scale=sm)
    g = H // Hkv
    k_rep, v_rep = heads.repeat_kv(k, g), heads.repeat_kv(v, g)
    ref = heads.quantize(q, k_rep, v_rep, None, pv_mode, gran="block_sq")
    c = lambda t: t.cpu().numpy()
    U.assert_same("q means", c(qz.q_mean), ref.q_mean)
    U.assert_same("q deltas", c(qz.q_scale), ref.q_delta)
    U.assert_same("q codes", c(qz.q_codes), ref.q_codes)
    # K and V per key/value head: the oracle's repeated heads h*g
    U.assert_same("k mean", c(qz.k_mean), ref.k_mean[:, ::g])
    U.assert_same("k deltas", c(qz.k_scale), ref.k_delta[:, ::g])
    U.assert_same("k codes", c(qz.k_codes), ref.k_codes[:, ::g])
    if pv_mode == "fp8":
        U.assert_same("v deltas", c(qz.v_scale), ref.v_delta[:, ::g])
        U.assert_same("v codes", c(qz.v_codes), ref.v_codes[:, ::g])
    _check_bias(qz, ref, k_rep, H, N, causal, sm)


CASES = [
    # (B, H, Hkv, N, D, dtype, causal, pv_mode)
    (1, 2, 2, 333, 64, "fp16", False, "fp16"),
    (1, 2, 2, 520, 128, "bf16", True, "fp16"),
    (2, 2, 1, 257, 128, "fp16", False, "fp8"),
    (1, 4, 2, 700, 64, "bf16", True, "fp8"),
    (1, 2, 2, 1024, 64, "fp16", True, "fp16"),
]


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal,pv_mode", CASES)
def test_smoothed_attention_against_oracle(B, H, Hkv, N, D, dtype, causal, pv_mode):
    q, k, v = _inputs(B, H, Hkv, N, D, dtype, seed=N * 7 + D)
    picks = [(b, h, i) for b in range(B) for h in range(H) for i in range(0, N, 2)]
    U.check_against_oracle(q, k, v, None, causal, pv_mode, picks, qk_gran="block_sq")


def test_full_size_sampled_rows():
    """The video-DiT shape of the bench (24 heads x 8192 tokens, D 64, FP8 P.V)
    in the bench's launch configuration, on sampled rows."""
    wl = W.WORKLOADS["dit_8k_fp8_sq"]
    inp = W.make_inputs(wl)
    rows = sage.api.sample_query_rows(wl.B, wl.H, wl.N, 96, seed=5)
    picks = [tuple(r) for r in rows]
    U.check_against_oracle(inp.q, inp.k, inp.v, None, wl.causal, wl.pv_mode, picks,
                           qk_gran="block_sq")


def test_split_stages_equal_fused_call():
    q, k, v = (t.cuda() for t in _inputs(1, 4, 2, 900, 128, "bf16", seed=3))
    for causal in (False, True):
        fused = sage.attn_fwd(q, k, v, causal=causal, pv_mode="fp16", out_dtype=torch.float32,
                              qk_gran="block_sq")
        qz = sage.quantize(q, k, v, "fp16", qk_gran="block_sq", causal=causal)
        split = sage.attn_quantized(qz, v, causal=causal, out_dtype=torch.float32)
        torch.cuda.synchronize()
        sage.sync_status()
        assert torch.equal(fused, split)
        with pytest.raises(ValueError):  # the mean term was built for the other mask
            sage.attn_quantized(qz, v, causal=not causal)


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,pv_mode,chunks", [
    (1, 4, 2, 1000, 128, "bf16", "fp16", (2, 4, 6)),      # NB 8
    (2, 3, 3, 700, 64, "fp16", "fp8", (2, 4)),            # NB 6, ragged tail
    (1, 2, 1, 1290, 64, "bf16", "fp8", (2, 8, 10)),       # NB 11: odd, last chunk one block
    (1, 2, 2, 129, 128, "fp16", "fp16", (2,)),            # NB 2: one chunk of both
])
def test_chunked_mean_term_equals_one_pass(B, H, Hkv, N, D, dtype, pv_mode, chunks):
    """With a workspace that holds the mean term of R query blocks at a time,
    the fused call runs R blocks' term and attention per chunk; every value
    is that of the single pass, so the outputs are equal bit for bit."""
    q, k, v = (t.cuda() for t in _inputs(B, H, Hkv, N, D, dtype, seed=N + H))
    for causal in (False, True):
        one = sage.attn_fwd(q, k, v, causal=causal, pv_mode=pv_mode, out_dtype=torch.float32,
                            qk_gran="block_sq")
        for r in chunks:
            got = sage.attn_fwd(q, k, v, causal=causal, pv_mode=pv_mode,
                                out_dtype=torch.float32, qk_gran="block_sq", sq_chunk_blocks=r)
            torch.cuda.synchronize()
            sage.sync_status()
            assert torch.equal(got, one), (causal, r)
    with pytest.raises(ValueError):
        sage.attn_fwd(q, k, v, qk_gran="block_sq", sq_chunk_blocks=3 if N > 500 else -1)


def test_smoothing_helps_with_a_query_offset():
    """A channel offset in Q (sigma 3, as K's) eats most of the int8 range of the
    unsmoothed codes; with smoothing the result is closer to fp64 attention."""
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in _inputs(1, 4, 4, 2048, 64, "fp16", seed=17, q_off=6.0))
    rows = sage.api.sample_query_rows(1, 4, 2048, 512, seed=2)
    ref = sage.attn_ref_rows(q, k, v, rows)
    idx = torch.tensor(rows, dtype=torch.long, device=dev)
    cos = {}
    for gran in ("block", "block_sq"):
        o = sage.attn_fwd(q, k, v, pv_mode="fp16", out_dtype=torch.float32, qk_gran=gran)
        cos[gran] = sage.cosine_similarity(o[idx[:, 0], idx[:, 1], idx[:, 2]], ref)
    print(cos)
    assert cos["block_sq"] > cos["block"] and cos["block_sq"] > 0.99


VARLEN = [
    # (seqlens, H, Hkv, D, dtype, causal, pv_mode)
    ([300, 1, 130, 700], 2, 2, 64, "fp16", True, "fp16"),
    ([520, 257], 4, 2, 128, "bf16", False, "fp8"),
    ([0, 200, 0, 129], 2, 1, 128, "fp16", True, "fp8"),
]


@pytest.mark.parametrize("seqlens,H,Hkv,D,dtype,causal,pv_mode", VARLEN)
def test_smoothed_varlen_against_oracle(seqlens, H, Hkv, D, dtype, causal, pv_mode):
    """Packed batches: every sequence's Q blocks take their own means and the
    mean term covers that sequence's keys (empty sequences included)."""
    q, k, v, cu = W.make_varlen(seqlens, H, D, dtype, seed=sum(seqlens) + D, q_bias_sigma=3.0)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    picks = [(si, h, i) for si, n in enumerate(seqlens) for h in range(H) for i in range(0, n, 3)]
    U.check_against_oracle(q, k, v, cu, causal, pv_mode, picks, qk_gran="block_sq")

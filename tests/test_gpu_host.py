"""attn_fwd_host (pinned host inputs and output; uploads, compute and
downloads of independent head groups overlapped, each slot with its own
compute stream and workspace) returns exactly what one attn_fwd over the
device copies returns."""
from __future__ import annotations

import pytest
import torch

import quantized_attention_07_b200 as sage
from quantized_attention_07_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal,pv_mode,gran,chunks,slots", [
    (2, 4, 4, 300, 64, "fp16", False, "fp16", "block", 8, 3),
    (1, 8, 2, 513, 128, "bf16", True, "fp8", "block", 3, 2),
    (1, 6, 6, 257, 128, "fp16", True, "fp16", "token", 64, 4),
    (3, 2, 1, 129, 64, "bf16", False, "fp8", "token", 1, 3),
    (2, 8, 8, 640, 128, "fp16", False, "fp16", "block_sq", 16, 3),
])
def test_host_pipeline_equals_device_call(B, H, Hkv, N, D, dtype, causal, pv_mode, gran, chunks,
                                          slots):
    q, k, v = W.make_dense(B, H, N, D, dtype, bias_sigma=3.0, seed=N + H)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    hout = torch.empty((B, H, N, D), dtype=torch.float32).pin_memory()
    for _ in range(2):  # the second call reuses the cached buffers and streams
        sage.attn_fwd_host(hq, hk, hv, hout, causal=causal, pv_mode=pv_mode, qk_gran=gran,
                           chunks=chunks, slots=slots)
        torch.cuda.synchronize()
        dev = torch.device("cuda")
        want = sage.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, pv_mode=pv_mode,
                             out_dtype=torch.float32, qk_gran=gran)
        torch.cuda.synchronize()
        sage.sync_status()
        assert torch.equal(hout, want.cpu())


@pytest.mark.parametrize("lens,H,Hkv,D,dtype,causal,pv_mode,gran,chunks,slots", [
    ([300, 129, 0, 700, 1, 512], 4, 4, 64, "fp16", True, "fp16", "block", 3, 2),
    ([1000, 20, 640, 333], 4, 2, 128, "bf16", True, "fp8", "block", 4, 3),
    ([257, 0, 0, 129], 2, 2, 128, "fp16", False, "fp16", "token", 8, 3),
    ([640, 700, 90], 4, 4, 64, "bf16", False, "fp8", "block_sq", 2, 2),
    ([5], 2, 1, 64, "fp16", True, "fp16", "block", 4, 3),
])
def test_varlen_host_pipeline_equals_device_call(lens, H, Hkv, D, dtype, causal, pv_mode, gran,
                                                 chunks, slots):
    """attn_fwd_varlen_host (pieces of consecutive sequences, each its own
    packed problem) returns exactly what one attn_fwd_varlen returns, with
    empty sequences, more pieces asked for than sequences, grouped heads."""
    q, k, v, cu = W.make_varlen(lens, H, D, dtype, seed=sum(lens) + H, q_bias_sigma=2.0)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    hout = torch.empty((q.shape[0], H, D), dtype=torch.float32).pin_memory()
    dev = torch.device("cuda")
    for _ in range(2):  # the second call reuses the cached buffers and streams
        sage.attn_fwd_varlen_host(hq, hk, hv, cu, hout, causal=causal, pv_mode=pv_mode,
                                  qk_gran=gran, chunks=chunks, slots=slots)
        torch.cuda.synchronize()
        want = sage.attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), max(lens),
                                    causal=causal, pv_mode=pv_mode, out_dtype=torch.float32,
                                    qk_gran=gran)
        torch.cuda.synchronize()
        sage.sync_status()
        assert torch.equal(hout, want.cpu())


def test_guide_entry_points_equal_the_core_calls():
    """The guide's API names run the same kernels as attn_fwd / attn_fwd_varlen."""
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in W.make_dense(1, 4, 700, 128, "bf16", seed=8))
    a = sage.sageattn_qk_int8_pv_fp16_cuda(q, k, v, is_causal=True)
    b = sage.attn_fwd(q, k, v, causal=True, pv_mode="fp16")
    assert torch.equal(a, b)
    a = sage.sageattn_qk_int8_pv_fp8_cuda(q, k, v, pv_accum_dtype="fp32+fp32")
    b = sage.attn_fwd(q, k, v, pv_mode="fp8")
    assert torch.equal(a, b)
    qp, kp, vp, cu = (t.to(dev) for t in W.make_varlen([300, 129], 4, 64, "fp16", seed=9))
    a = sage.sageattn_varlen(qp, kp, vp, cu, 300, is_causal=True)
    b = sage.attn_fwd_varlen(qp, kp, vp, cu, 300, causal=True)
    torch.cuda.synchronize()
    sage.sync_status()
    assert torch.equal(a, b)

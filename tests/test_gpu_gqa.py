"""Grouped-query attention (query head h reads key/value head h // (H/Hkv)):
the GPU result must equal, bit for bit, the same library on repeat_kv'd K and
V -- K means, deltas and V scales are per key/value head, so repeating changes
no code -- and must match the oracle's emulation on the repeated inputs."""
from __future__ import annotations

import pytest
import torch

import quantized_attention_07_b200 as sage
from quantized_attention_07_b200 import workloads as W
from oracle import heads

from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_07_b200 import build
    import oracle
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _grouped(B, H, Hkv, N, D, dtype, seed):
    q, k, v = W.make_dense(B, H, N, D, dtype, bias_sigma=3.0, outlier_p=0.01,
                           outlier_scale=10.0, seed=seed)
    return q, k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()


CASES = [
    # (B, H, Hkv, N, D, dtype, causal, pv_mode)
    (1, 8, 2, 700, 128, "fp16", False, "fp16"),
    (2, 4, 1, 333, 64, "bf16", True, "fp16"),
    (1, 8, 4, 1000, 64, "fp16", False, "fp8"),
    (1, 6, 3, 257, 128, "bf16", True, "fp8"),
    (1, 4, 2, 1, 128, "fp16", True, "fp16"),
]


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal,pv_mode", CASES)
def test_gqa_equals_repeated_kv_bit_for_bit(B, H, Hkv, N, D, dtype, causal, pv_mode):
    q, k, v = _grouped(B, H, Hkv, N, D, dtype, seed=N + H + D)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    g = H // Hkv
    kr, vr = heads.repeat_kv(k, g).to(dev), heads.repeat_kv(v, g).to(dev)
    for od in (torch.float32, q.dtype):
        a = sage.attn_fwd(qd, kd, vd, causal=causal, pv_mode=pv_mode, out_dtype=od)
        b = sage.attn_fwd(qd, kr, vr, causal=causal, pv_mode=pv_mode, out_dtype=od)
        torch.cuda.synchronize()
        sage.sync_status()
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal,pv_mode", CASES[:4])
def test_gqa_against_oracle(B, H, Hkv, N, D, dtype, causal, pv_mode):
    q, k, v = _grouped(B, H, Hkv, N, D, dtype, seed=N * 3 + H)
    picks = [(b, h, i) for b in range(B) for h in range(H) for i in range(0, N, 3)]
    U.check_against_oracle(q, k, v, None, causal, pv_mode, picks)


def test_gqa_sageattn_shim_needs_no_repeat():
    q, k, v = _grouped(1, 8, 2, 512, 128, "bf16", seed=9)
    dev = torch.device("cuda")
    out = sage.sageattn(q.to(dev), k.to(dev), v.to(dev), is_causal=True)
    ref = sage.sageattn(q.to(dev), heads.repeat_kv(k, 4).to(dev), heads.repeat_kv(v, 4).to(dev),
                        is_causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("causal,pv_mode,dtype,H,Hkv", [(True, "fp16", "bf16", 8, 2),
                                                       (False, "fp8", "fp16", 4, 1),
                                                       (True, "fp8", "bf16", 6, 3)])
def test_varlen_gqa_equals_repeated_and_oracle(causal, pv_mode, dtype, H, Hkv):
    lens = [1, 300, 129, 0, 517]
    D = 128 if pv_mode == "fp8" else 64
    q, k, v, cu = W.make_varlen(lens, H, D, dtype, seed=H * 7 + Hkv)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    dev = torch.device("cuda")
    g = H // Hkv
    kr, vr = heads.repeat_kv_packed(k, g), heads.repeat_kv_packed(v, g)
    a = sage.attn_fwd_varlen(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), max(lens), causal=causal,
                             pv_mode=pv_mode, out_dtype=torch.float32)
    b = sage.attn_fwd_varlen(q.to(dev), kr.to(dev), vr.to(dev), cu.to(dev), max(lens),
                             causal=causal, pv_mode=pv_mode, out_dtype=torch.float32)
    torch.cuda.synchronize()
    sage.sync_status()
    assert torch.equal(a, b)
    picks = [(s, h, i) for s, n in enumerate(lens) for h in range(H) for i in range(0, n, 3)]
    U.check_against_oracle(q, k, v, cu, causal, pv_mode, picks)

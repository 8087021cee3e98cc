"""Per-token Q/K deltas ("SageAttention v1/v2/v2++/v3 overview", SageAttention
v1 item (1): per-block or per-token quantisation): the GPU codes and deltas
equal the oracle's bit for bit, the attention output matches the oracle's
per-token emulation, and on inputs with channel outliers the finer deltas are
more accurate than per-block ones."""
from __future__ import annotations

import numpy as np
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


@pytest.mark.parametrize("N,D,dtype,pv_mode", [(300, 64, "fp16", "fp16"), (1000, 128, "bf16", "fp8"),
                                               (128, 128, "fp16", "fp8"), (1, 64, "bf16", "fp16")])
def test_per_token_quantisation_bit_exact(N, D, dtype, pv_mode):
    q, k, v = W.make_dense(2, 3, N, D, dtype, bias_sigma=3.0, outlier_p=0.01, outlier_scale=20.0,
                           seed=77 + N + D)
    dev = torch.device("cuda")
    qz = sage.quantize(q.to(dev), k.to(dev), v.to(dev), pv_mode, qk_gran="token")
    torch.cuda.synchronize()
    sage.sync_status()
    ref = heads.quantize(q, k, v, None, pv_mode, gran="token")
    U.compare_quant_dense(qz, ref, pv_mode)


CASES = [
    # (B, H, Hkv, N, D, dtype, causal, pv_mode)
    (1, 2, 2, 333, 64, "fp16", False, "fp16"),
    (1, 2, 2, 520, 128, "bf16", True, "fp16"),
    (2, 2, 1, 257, 128, "fp16", False, "fp8"),
    (1, 4, 2, 700, 64, "bf16", True, "fp8"),
]


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal,pv_mode", CASES)
def test_per_token_attention_against_oracle(B, H, Hkv, N, D, dtype, causal, pv_mode):
    q, k, v = W.make_dense(B, H, N, D, dtype, bias_sigma=3.0, outlier_p=0.01, outlier_scale=10.0,
                           seed=N * 5 + D)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    picks = [(b, h, i) for b in range(B) for h in range(H) for i in range(0, N, 2)]
    U.check_against_oracle(q, k, v, None, causal, pv_mode, picks, qk_gran="token")


def test_per_token_deltas_help_with_outliers():
    """Video-DiT-like channel outliers (1 % of entries x20): per-token deltas
    keep the other rows' codes fine-grained, so the result is closer to
    full-precision attention than with one delta per 128 tokens."""
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in W.make_dense(1, 4, 2048, 64, "fp16", bias_sigma=3.0,
                                               outlier_p=0.01, outlier_scale=20.0, seed=11))
    rows = sage.api.sample_query_rows(1, 4, 2048, 512, seed=2)
    ref = sage.attn_ref_rows(q, k, v, rows)
    idx = torch.tensor(rows, dtype=torch.long, device=dev)
    cos = {}
    for gran in ("block", "token"):
        o = sage.attn_fwd(q, k, v, pv_mode="fp16", out_dtype=torch.float32, qk_gran=gran)
        cos[gran] = sage.cosine_similarity(o[idx[:, 0], idx[:, 1], idx[:, 2]], ref)
    print(cos)
    assert cos["token"] > cos["block"] + 0.01 and cos["token"] > 0.98


@pytest.mark.parametrize("causal,pv_mode,dtype,H,Hkv", [(True, "fp16", "bf16", 4, 2),
                                                       (False, "fp8", "fp16", 2, 2)])
def test_per_token_varlen_against_oracle(causal, pv_mode, dtype, H, Hkv):
    lens = [1, 300, 0, 129, 517]
    D = 128 if pv_mode == "fp8" else 64
    q, k, v, cu = W.make_varlen(lens, H, D, dtype, seed=31 + H)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    picks = [(s, h, i) for s, n in enumerate(lens) for h in range(H) for i in range(0, n, 2)]
    U.check_against_oracle(q, k, v, cu, causal, pv_mode, picks, qk_gran="token")

"""GPU side of the accuracy-driven P.V mode choice: the full-precision
reference rows against the oracle's fp64 definition, and the choice itself on
inputs where FP8 P.V is and is not accurate enough."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import quantized_attention_07_b200 as sage
from quantized_attention_07_b200 import api
from quantized_attention_07_b200 import workloads as W
from oracle import heads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_07_b200 import build
    import oracle
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("B,H,Hkv,N,D,dtype,causal", [
    (1, 2, 2, 300, 64, "fp16", False),
    (2, 4, 2, 513, 128, "bf16", True),
    (1, 8, 1, 129, 128, "fp16", True),
])
def test_reference_rows_match_oracle_definition(B, H, Hkv, N, D, dtype, causal):
    q, k, v = W.make_dense(B, H, N, D, dtype, bias_sigma=3.0, outlier_p=0.01, outlier_scale=10.0,
                           seed=N + D)
    k, v = k[:, :Hkv].contiguous(), v[:, :Hkv].contiguous()
    rows = api.sample_query_rows(B, H, N, 64, seed=3)
    dev = torch.device("cuda")
    got = sage.attn_ref_rows(q.to(dev), k.to(dev), v.to(dev), rows, causal).cpu().numpy()
    kr, vr = heads.repeat_kv(k, H // Hkv), heads.repeat_kv(v, H // Hkv)
    want = heads.reference_rows(q, kr, vr, None, rows, causal)
    W_ = np.stack([want[r] for r in rows])
    assert np.abs(got - W_).max() <= 3e-5 * max(1.0, np.abs(W_).max())


def test_choice_keeps_16bit_where_fp8_is_not_accurate_enough():
    dev = torch.device("cuda")
    # channel outliers in Q and K (as in the video-DiT workload): FP8 P.V loses accuracy
    qo, ko, vo = (t.to(dev) for t in W.make_dense(1, 4, 2048, 64, "fp16", bias_sigma=3.0,
                                                  outlier_p=0.01, outlier_scale=20.0, seed=11))
    # plain Gaussian inputs: FP8 P.V is as accurate as the threshold asks
    qg, kg, vg = (t.to(dev) for t in W.make_dense(1, 4, 2048, 128, "bf16", bias_sigma=3.0,
                                                  seed=12))
    got = sage.calibrate_pv_modes({"outliers": [(qo, ko, vo, False)],
                                   "gaussian": [(qg, kg, vg, True)]})
    print(got)
    assert got["outliers"][0] == "fp16" and got["outliers"][1] <= api.PV_COSINE_THRESHOLD
    assert got["gaussian"][0] == "fp8" and got["gaussian"][1] > api.PV_COSINE_THRESHOLD
    for mode, lo8, lo16 in got.values():
        assert lo16 >= lo8 - 1e-4   # the 16-bit mode is never the less accurate one

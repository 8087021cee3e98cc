"""Host logic of the accuracy-driven P.V mode choice ("SageAttention
v1/v2/v2++/v3 overview", SageAttention v1: a layer takes the faster variant
only where its cosine similarity to full precision is above 99.8 %)."""
from __future__ import annotations

import pytest

from quantized_attention_07_b200 import _lib, api, build


def test_threshold_is_strict():
    assert api.choose_pv_mode(0.9981) == "fp8"
    assert api.choose_pv_mode(0.998) == "fp16"      # "above" 99.8 %, not at it
    assert api.choose_pv_mode(0.95) == "fp16"
    assert api.choose_pv_mode(0.96, threshold=0.95) == "fp8"


def test_calibration_takes_each_layers_worst_input():
    sims = {"a": [0.9995, 0.9990], "b": [0.9995, 0.9970], "c": [0.998]}
    layers = {name: [(name, j, None, False) for j in range(len(v))] for name, v in sims.items()}

    def fake_measure(q, k, v, causal):  # q = layer name, k = input index
        return {"fp8": sims[q][k], "fp16": 0.9999}

    got = api.calibrate_pv_modes(layers, measure=fake_measure)
    assert got["a"] == ("fp8", 0.9990, 0.9999)
    assert got["b"][0] == "fp16" and got["b"][1] == 0.9970
    assert got["c"][0] == "fp16"


def test_sampled_rows_cover_first_and_last_rows():
    rows = api.sample_query_rows(2, 3, 50, 40, seed=1)
    assert rows == api.sample_query_rows(2, 3, 50, 40, seed=1)
    assert len(rows) == 40 and len(set(rows)) == 40
    for b in range(2):
        for h in range(3):
            assert (b, h, 0) in rows and (b, h, 49) in rows
    assert all(0 <= b < 2 and 0 <= h < 3 and 0 <= i < 50 for b, h, i in rows)
    assert len(api.sample_query_rows(1, 1, 3, 100)) == 3   # capped by the input


def test_reference_rows_validation_on_host():
    build.build()
    f = _lib.load().sage_attn_ref_rows
    F = 0x10000
    assert f(F, F, F, 0, 1, 8, 3, 64, 64, 0, 0.0, F, 4, F, None) == 1   # Hkv must divide H
    assert f(F, F, F, 0, 1, 8, 2, 64, 96, 0, 0.0, F, 4, F, None) == 1   # D
    assert f(F, F, F, 2, 1, 8, 2, 64, 64, 0, 0.0, F, 4, F, None) == 1   # dtype
    assert f(F, F, F, 0, 1, 8, 2, 64, 64, 0, float("nan"), F, 4, F, None) == 1
    assert f(F, F, F, 0, 1, 8, 2, 64, 64, 0, 0.0, F, 0, F, None) == 0   # nothing to do


def test_fp8_entry_point_refuses_other_accumulation_types():
    import torch

    import quantized_attention_07_b200 as sage
    x = torch.zeros((1, 1, 128, 64), dtype=torch.float16)
    with pytest.raises(sage.SageError):
        sage.sageattn_qk_int8_pv_fp8_cuda(x, x, x, pv_accum_dtype="fp16")

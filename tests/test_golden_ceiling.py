"""The recorded accuracy ceiling of the method (tests/golden/accuracy_ceiling.json,
written by tests/golden/make_accuracy_ceiling.py from the oracle alone) covers
every workload, and its entry for the small workload is what the oracle
computes now."""
from __future__ import annotations

import json
import os
import sys

from quantized_attention_07_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def _load():
    with open(os.path.join(HERE, "golden", "accuracy_ceiling.json")) as f:
        return json.load(f)


def test_ceiling_covers_every_workload():
    data = _load()
    assert set(data) == set(W.WORKLOADS)
    for name, e in data.items():
        assert 0.9 < e["cosine_emulation_vs_fp64"] <= 1.0, name
        assert e["pv_mode"] == W.WORKLOADS[name].pv_mode
    # the outlier workload is the one below the 0.999 bar, and per-token
    # deltas and Q smoothing raise it
    assert data["dit_8k_fp8"]["cosine_emulation_vs_fp64"] < 0.999
    assert data["dit_8k_fp8_tok"]["cosine_emulation_vs_fp64"] > \
        data["dit_8k_fp8"]["cosine_emulation_vs_fp64"]


def test_small_workload_ceiling_reproduces():
    sys.path.insert(0, os.path.join(HERE, "golden"))
    import make_accuracy_ceiling as mk
    got = mk.ceiling("small_d64")
    assert got == _load()["small_d64"]

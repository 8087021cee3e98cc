"""Writes accuracy_ceiling.json: the accuracy of the quantised method itself on
each workload, measured on the CPU oracle alone.

For every workload, at full size, the oracle quantises all heads and
computes, on the same 512 seeded query rows the GPU parity test samples (all
rows of the small one), both its emulation E of the plain method and the fp64
reference R = softmax(QK^T * sm_scale) V; the recorded figure is the cosine
similarity of E and R over those rows (flattened), and the largest |E - R|.
This is the ceiling a correct implementation reaches: the per-block INT8
method cannot be more accurate than its own exact emulation.  The GPU parity
test of a workload whose ceiling is below 0.999 (channel outliers) gates on
this recorded value.

    python tests/golden/make_accuracy_ceiling.py

Calls only the oracle and the seeded input generators.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import heads  # noqa: E402
from quantized_attention_07_b200 import workloads as W  # noqa: E402

OUT = os.path.join(HERE, "accuracy_ceiling.json")


def picks_of(wl, inp):
    if wl.varlen:
        return W.sample_rows(inp.seqlens, wl.H, 512, seed=wl.seed)
    if wl.B * wl.H * wl.N <= 4096:
        return [(b, h, i) for b in range(wl.B) for h in range(wl.H) for i in range(wl.N)]
    return W.sample_rows([wl.N] * wl.B, wl.H, 512, seed=wl.seed)


def ceiling(name: str) -> dict:
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    k, v = inp.k, inp.v
    if not wl.varlen and wl.kv_heads != wl.H:
        g = wl.H // wl.kv_heads
        k, v = heads.repeat_kv(k, g), heads.repeat_kv(v, g)
    picks = picks_of(wl, inp)
    qz = heads.quantize(inp.q, k, v, inp.cu_seqlens, wl.pv_mode, gran=wl.qk_gran)
    emu = heads.emulate_rows(qz, v, inp.cu_seqlens, picks, wl.D, wl.causal, wl.pv_mode,
                             gran=wl.qk_gran, k=k if wl.qk_gran == "block_sq" else None)
    ref = heads.reference_rows(inp.q, k, v, inp.cu_seqlens, picks, wl.causal)
    E = np.stack([emu[p] for p in picks]).astype(np.float64).ravel()
    R = np.stack([ref[p] for p in picks]).ravel()
    cos = float(E @ R / (np.linalg.norm(E) * np.linalg.norm(R)))
    return {"cosine_emulation_vs_fp64": round(cos, 6), "max_abs_emulation_vs_fp64":
            round(float(np.abs(E - R).max()), 6), "rows": len(picks),
            "pv_mode": wl.pv_mode, "qk_gran": wl.qk_gran}


def main():
    names = sys.argv[1:] or list(W.WORKLOADS)
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    for n in names:
        data[n] = ceiling(n)
        print(n, data[n], flush=True)
    with open(OUT, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main()

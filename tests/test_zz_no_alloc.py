"""sage_quantize_noalloc: the quantisation stage without a caller workspace.

Some callers may not allocate device memory and have no workspace to give the
library -- an extension living inside a host application that owns every
device allocation, or a path where cudaMalloc's implicit synchronisation is
not allowed.  For them the library keeps the stage's reduction scratch in a
fixed device array.  These tests call that entry point through the C ABI and
check that its outputs are identical to those of sage_quantize (the
workspace-taking entry point) on two calls in a row with different inputs, so
that nothing left in the shared array by one call leaks into the next.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import quantized_attention_07_b200 as sage
from quantized_attention_07_b200 import _lib, api
from quantized_attention_07_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc(q, k, v, pv_mode, status=None):
    B, H, N, D = q.shape
    qz = api.alloc_quantized(B, H, N, D, pv_mode, q.device)
    p = lambda t: None if t is None else t.data_ptr()
    rc = _lib.load().sage_quantize_noalloc(
        p(q), p(k), p(v) if pv_mode == "fp8" else None, api._dtype_code(q.dtype), B, H, N, D,
        api.PV_MODES[pv_mode], p(qz.q_codes), p(qz.q_scale), p(qz.k_codes), p(qz.k_scale),
        p(qz.k_mean), p(qz.v_codes), p(qz.v_scale), p(status),
        torch.cuda.current_stream().cuda_stream)
    return rc, qz


def _same(a: api.Quantized, b: api.Quantized):
    for name in ("q_codes", "q_scale", "k_codes", "k_scale", "k_mean", "v_codes", "v_scale"):
        x, y = getattr(a, name), getattr(b, name)
        if x is None:
            assert y is None
            continue
        assert torch.equal(x, y), name


@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
def test_noalloc_matches_workspace_entry_point_twice(pv_mode):
    cases = [(2, 4, 1000, 128, "fp16", 11), (1, 8, 777, 64, "bf16", 12)]
    for B, H, N, D, dt, seed in cases:   # two calls in a row, different shapes/data
        q, k, v = (t.cuda() for t in W.make_dense(B, H, N, D, dt, 3.0, 0.01, 20.0, seed=seed))
        status = torch.full((1,), 123, dtype=torch.int32, device="cuda")
        rc, got = _noalloc(q, k, v, pv_mode, status)
        assert rc == 0
        ref = sage.quantize(q, k, v, pv_mode)
        torch.cuda.synchronize()
        sage.sync_status()
        assert status.item() == 0
        _same(got, ref)


def test_noalloc_reports_range_error_and_recovers():
    q, k, v = (t.cuda() for t in W.make_dense(1, 2, 256, 64, "bf16", seed=13))
    k[0, 1, 5, 9] = 70000.0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc, _ = _noalloc(q, k, v, "fp16", status)
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == 4
    k[0, 1, 5, 9] = 1.0
    rc, got = _noalloc(q, k, v, "fp16", status)
    ref = sage.quantize(q, k, v, "fp16")
    torch.cuda.synchronize()
    assert rc == 0 and status.item() == 0
    _same(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib.load()
    FAKE = 0x10000
    # B*H*D = 4*129*128 > 65536: rejected on the host before anything runs
    rc = lib.sage_quantize_noalloc(FAKE, FAKE, None, 0, 4, 129, 256, 128, 0, FAKE, FAKE, FAKE,
                                   FAKE, FAKE, None, None, None, None)
    assert rc == 3
    rc = lib.sage_quantize_noalloc(FAKE, FAKE, None, 0, 1, 1, 256, 96, 0, FAKE, FAKE, FAKE,
                                   FAKE, FAKE, None, None, None, None)
    assert rc == 1

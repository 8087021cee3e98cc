"""Device-side failure reporting, exercised without faulting the GPU: a wait
that runs out (in a one-barrier stand-in and in the fused attention kernel
itself, on a barrier that nothing completes), inconsistent cu_seqlens and
out-of-range K values are recorded in the workspace status word, reported by
sync_status, and the next call on the same workspace succeeds."""
from __future__ import annotations

import pytest
import torch

import quantized_attention_07_b200 as sage
from quantized_attention_07_b200 import _lib
from quantized_attention_07_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _ok_call(ws=None):
    q, k, v = (t.cuda() for t in W.make_dense(1, 2, 300, 64, "fp16", seed=3))
    out = sage.attn_fwd(q, k, v, workspace=ws)
    sage.sync_status(ws)
    assert torch.isfinite(out).all()


def test_wait_timeout_is_reported_and_recovers():
    ws = sage.Workspace(1 << 20)
    rc = _lib.load().sage_selftest_wait_timeout(200000, ws.ptr, ws.nbytes,
                                                torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    with pytest.raises(sage.SageError) as e:
        ws.sync_status()
    assert e.value.code == 5
    ws.sync_status()          # cleared by the read
    _ok_call(ws)


@pytest.mark.parametrize("cu", [[0, 100, 50, 300], [0, 100, 200, 301], [1, 100, 200, 300]])
def test_bad_cu_seqlens(cu):
    T = 300
    q, k, v, _ = W.make_varlen([100, 100, 100], 2, 64, "bf16", seed=4)
    ws = sage.Workspace(sage.workspace_bytes_varlen(T, 3, 2, 64))
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    sage.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_t, 300, workspace=ws)
    with pytest.raises(sage.SageError) as e:
        ws.sync_status()
    assert e.value.code == 6
    _ok_call(ws)


def test_seqlen_above_max_seqlen():
    q, k, v, cu = W.make_varlen([100, 200], 2, 64, "fp16", seed=4)
    ws = sage.Workspace(sage.workspace_bytes_varlen(300, 2, 2, 64))
    sage.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), 150, workspace=ws)
    with pytest.raises(sage.SageError) as e:
        ws.sync_status()
    assert e.value.code == 6


def test_k_out_of_exact_mean_range():
    q, k, v = W.make_dense(1, 1, 256, 64, "bf16", seed=5)
    k[0, 0, 17, 3] = 70000.0
    ws = sage.Workspace(sage.workspace_bytes(1, 1, 256, 64))
    sage.attn_fwd(q.cuda(), k.cuda(), v.cuda(), workspace=ws)
    with pytest.raises(sage.SageError) as e:
        ws.sync_status()
    assert e.value.code == 7
    _ok_call(ws)


def test_unsupported_mask_and_dropout():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.sageattn(q, q, q, attn_mask=torch.ones(8, 8, dtype=torch.bool, device="cuda"))
    assert e.value.code == 2
    with pytest.raises(sage.SageError):
        sage.sageattn(q, q, q, dropout_p=0.1)


def test_sageattn_shim_matches_attn_fwd():
    q, k, v = (t.cuda() for t in W.make_dense(1, 4, 300, 128, "bf16", seed=6))
    a = sage.sageattn(q.transpose(1, 2).contiguous().transpose(1, 2), k, v, is_causal=True)
    b = sage.attn_fwd(q, k, v, causal=True)
    assert torch.equal(a, b)


def _attn_selftest(qz, v, out, wait_cycles, skip, ws):
    B, H, NP, D = qz.q_codes.shape
    p = lambda t: None if t is None else t.data_ptr()
    return _lib.load().sage_selftest_attn_timeout(
        p(qz.q_codes), p(qz.q_scale), p(qz.k_codes), p(qz.k_scale), p(v), p(qz.v_codes),
        p(qz.v_scale), p(out), 0, 2, B, H, v.shape[2], D, 0, 0.0,
        1 if qz.pv_mode == "fp8" else 0, wait_cycles, skip, ws.ptr, ws.nbytes,
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
@pytest.mark.parametrize("H,skip", [(1, 1), (1, 3), (4, 2)])
def test_attention_kernel_wait_timeout_is_reported_and_recovers(pv_mode, H, skip):
    """The fused attention kernel's own bounded waits: with one K tile left
    unloaded its barrier never completes; the MMA role gives up after the
    (shortened) limit, records a timeout, and every role reaches the teardown,
    which frees tensor memory and resets the work counter -- the next call on
    the same workspace returns the normal result bit for bit."""
    q, k, v = (t.cuda() for t in W.make_dense(1, H, 512, 128, "fp16", seed=8))
    ws = sage.Workspace(1 << 20)
    qz = sage.quantize(q, k, v, pv_mode, workspace=ws)
    ref = sage.attn_quantized(qz, v, out_dtype=torch.float32, workspace=ws)
    ws.sync_status()
    out = torch.empty_like(ref)
    limit = 1 << 24  # ~8 ms of SM clock: far above any legitimate wait here
    assert _attn_selftest(qz, v, out, limit, 0, ws) == 0     # shorter limit, no fault
    ws.sync_status()
    assert torch.equal(out, ref)
    assert _attn_selftest(qz, v, out, limit, skip, ws) == 0
    with pytest.raises(sage.SageError) as e:
        ws.sync_status()
    assert e.value.code == 5
    again = sage.attn_quantized(qz, v, out_dtype=torch.float32, workspace=ws)
    ws.sync_status()
    assert torch.equal(again, ref)

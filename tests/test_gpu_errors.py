"""Device-side failure reporting, exercised without faulting the GPU: a wait
that runs out, inconsistent cu_seqlens and out-of-range K values are recorded
in the workspace status word, reported by sync_status, and the next call on
the same workspace succeeds."""
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


def test_software_exp2_error_bound():
    """The FMA-pipe 2^x used for a share of the softmax exponentials stays within
    2.2e-7 relative error of the exact value over its range (and is exact-ish at
    integers), checked against fp64."""
    import numpy as np
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125, 8, 2_000_000), np.arange(-125, 9, dtype=np.float64),
                        rng.uniform(-0.5, 0.5, 200_000), [0.0, -0.0, 8.0, -125.0]]).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    yt = torch.empty_like(xt)
    rc = _lib.load().sage_selftest_exp2(xt.data_ptr(), yt.data_ptr(), x.size,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    y = yt.cpu().numpy().astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y - exact) / exact
    assert rel.max() <= 2.2e-7, rel.max()

"""Pins of the oracle's Q smoothing (SageAttention2's smoothing of Q: the
dtcms.com page, v2 bullet 2; the postsniper.ru post, SageAttention2 bullet 1).

The smoothed method is q = q~ + qmean_I per 128-token query block I, q~
quantised per block, and the per-key term qmean_I . k~_j added back to the
scaled logit.  The pins below fix it from outside the oracle:

- exactly quantisable inputs: when q~ and k~ are integer multiples of 2^-7
  whose block maxima are 127 * 2^-7, every code and delta is exact, so the
  emulated output must equal fp64 attention up to the rounding of P to 16 bits
  (2^-11 relative), whatever the block means are.  A dropped, transposed or
  mis-signed mean term, a mean taken over the wrong block, or codes of the
  unsmoothed q all miss by orders of magnitude;
- zero block means: smoothing is then the identity, and the emulation must be
  bit-identical to the plain per-block one;
- a packed batch of one sequence is the dense problem: bit-identical.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import heads

BLK = 128


def _pair_rows(rng, rows, D, scale_bits=7):
    """[rows, D] integer multiples of 2^-scale_bits in [-127, 127] * 2^-7,
    rows in +/- pairs (column sums exactly 0), one entry 127 per pair set."""
    assert rows % 2 == 0
    half = rng.integers(-100, 101, size=(rows // 2, D))
    half[0, 0] = 127
    z = np.empty((rows, D), np.int64)
    z[0::2] = half
    z[1::2] = -half
    return z * 2.0 ** -scale_bits


def _exact_inputs(N, D, seed, causal_len=None):
    rng = np.random.default_rng(seed)
    nb = (N + BLK - 1) // BLK
    q = np.empty((N, D))
    for I in range(nb):
        r0, r1 = I * BLK, min(N, (I + 1) * BLK)
        mu = rng.integers(-64, 65, size=D) * 2.0 ** -4      # block mean, |mu| <= 4
        q[r0:r1] = mu + _pair_rows(rng, r1 - r0, D)
    # K: global mean m0 plus pairs; each 128-key block holds its own +/-127 pair
    m0 = rng.integers(-32, 33, size=D) * 2.0 ** -4
    w = np.concatenate([_pair_rows(rng, min(N, (I + 1) * BLK) - I * BLK, D) for I in range(nb)])
    k = m0 + w
    v = rng.standard_normal((N, D))
    t = lambda a: torch.from_numpy(a).half()[None, None]
    qh, kh, vh = t(q), t(k), t(v)
    # exactly representable in fp16
    assert np.array_equal(qh[0, 0].double().numpy(), q)
    assert np.array_equal(kh[0, 0].double().numpy(), k)
    return qh, kh, vh


@pytest.mark.parametrize("N,D,causal", [(256, 64, False), (200, 64, True), (330, 128, False)])
def test_exact_inputs_reach_fp64_attention(N, D, causal):
    q, k, v = _exact_inputs(N, D, seed=N + D)
    qz = heads.quantize(q, k, v, gran="block_sq")
    assert qz.status == 0
    # the smoothing reached exact codes: q~ = z, deltas 2^-7
    assert np.all(qz.q_delta == np.float32(2.0 ** -7))
    assert np.all(qz.k_delta == np.float32(2.0 ** -7))
    rows = sorted({0, 1, 77, BLK - 1, min(N - 1, BLK), N // 2, N - 1})
    picks = [(0, 0, i) for i in rows]
    e = heads.emulate_rows(qz, v, None, picks, D, causal, "fp16", gran="block_sq", k=k)
    sm = oracle.default_sm_scale(D)
    ref = oracle.attn_ref_rows(q[0, 0].float().numpy(), k[0, 0].float().numpy(),
                               v[0, 0].float().numpy(), sm, causal, rows)
    vmax = float(v.abs().max())
    # P rounded to fp16 (2^-11 relative) dominates; fp32 steps add ~1e-6
    bound = 2.0 ** -11 * vmax + 1e-5
    for r, i in enumerate(rows):
        err = np.abs(e[(0, 0, i)] - ref[r]).max()
        assert err <= bound, (i, err, bound)

    # the same inputs without the per-key mean term are far off: the pin
    # separates a dropped term from rounding
    qc, qd, kc, kd, _, _ = heads._head_view(qz, None, 0, 0)
    no_bias = oracle.attn_emul_rows(qc, qd, kc, kd, N, D, sm, causal, "fp16", rows,
                                    v=v[0, 0].float().numpy())
    worst = max(np.abs(no_bias[r] - ref[r]).max() for r in range(len(rows)))
    assert worst > 50 * bound


def test_bias_is_per_block_and_per_key():
    """q_smooth_bias against its definition on dyadic values, where every fp32
    partial sum is exact (so the fp64 matrix product gives the same sum):
    out[I, j] = fp32(kappa * qmean_I . (k_j - kmean))."""
    rng = np.random.default_rng(5)
    nb, n, D = 3, 70, 64
    qm = (rng.integers(-64, 65, size=(nb, D)) * 2.0 ** -4).astype(np.float32)
    k = (rng.integers(-512, 513, size=(n, D)) * 2.0 ** -8).astype(np.float32)
    km = (rng.integers(-16, 17, size=D) * 2.0 ** -4).astype(np.float32)
    sm = 0.125
    out = oracle.q_smooth_bias(qm, k, km, sm, ldo=80)
    kappa = float(oracle.kappa(sm))
    exact = (qm.astype(np.float64) @ (k.astype(np.float64) - km).T) * kappa
    np.testing.assert_array_equal(out[:, :n], exact.astype(np.float32))
    assert np.all(out[:, n:] == 0)
    # rows follow the block, columns the key
    assert not np.array_equal(out[0, :n], out[1, :n])


def test_zero_block_means_reduce_to_plain_per_block():
    rng = np.random.default_rng(11)
    N, D = 256, 64
    z = np.concatenate([rng.standard_normal((BLK // 2, D)) for _ in range(N // BLK)])
    q = np.empty((N, D))
    q[0::2], q[1::2] = z, -z           # every 128-row block has channel sums exactly 0
    q = torch.from_numpy(q).half()[None, None]
    k = torch.randn(1, 1, N, D, generator=torch.Generator().manual_seed(3)).half()
    v = torch.randn(1, 1, N, D, generator=torch.Generator().manual_seed(4)).half()
    sq = heads.quantize(q, k, v, gran="block_sq")
    pb = heads.quantize(q, k, v, gran="block")
    assert np.all(sq.q_mean == 0)
    np.testing.assert_array_equal(sq.q_codes, pb.q_codes)
    np.testing.assert_array_equal(sq.q_delta, pb.q_delta)
    picks = [(0, 0, i) for i in (0, 100, 200, 255)]
    a = heads.emulate_rows(sq, v, None, picks, D, True, "fp16", gran="block_sq", k=k)
    b = heads.emulate_rows(pb, v, None, picks, D, True, "fp16")
    for p in picks:
        np.testing.assert_array_equal(a[p], b[p])


def test_smoothing_helps_on_biased_queries():
    """The point of the method: with a large shared offset in Q, the smoothed
    emulation is closer to fp64 attention than the unsmoothed one."""
    g = torch.Generator().manual_seed(21)
    N, D = 256, 64
    q = (torch.randn(1, 1, N, D, generator=g) + 4.0 * torch.randn(1, 1, 1, D, generator=g)).half()
    k = torch.randn(1, 1, N, D, generator=g).half()
    v = torch.randn(1, 1, N, D, generator=g).half()
    rows = list(range(0, N, 9))
    picks = [(0, 0, i) for i in rows]
    sq = heads.emulate_rows(heads.quantize(q, k, v, gran="block_sq"), v, None, picks, D, False,
                            "fp16", gran="block_sq", k=k)
    pb = heads.emulate_rows(heads.quantize(q, k, v), v, None, picks, D, False, "fp16")
    ref = oracle.attn_ref_rows(q[0, 0].float().numpy(), k[0, 0].float().numpy(),
                               v[0, 0].float().numpy(), oracle.default_sm_scale(D), False, rows)
    e_sq = np.mean([np.abs(sq[p] - ref[r]).mean() for r, p in enumerate(picks)])
    e_pb = np.mean([np.abs(pb[p] - ref[r]).mean() for r, p in enumerate(picks)])
    assert e_sq < 0.7 * e_pb, (e_sq, e_pb)


def test_packed_single_sequence_equals_dense():
    """A packed batch of one sequence is the dense problem with B = 1: the
    smoothed codes, means and emulated rows agree bit for bit, and a second
    sequence after it does not change the first one's rows."""
    g = torch.Generator().manual_seed(31)
    n, H, D = 300, 2, 64
    qd_, kd_, vd_ = (torch.randn(1, H, n, D, generator=g).half() for _ in range(3))
    qd_ = (qd_.float() + 3.0 * torch.randn(1, H, 1, D, generator=g)).half()
    dense = heads.quantize(qd_, kd_, vd_, gran="block_sq")
    pk = lambda t: t[0].transpose(0, 1).contiguous()              # [n, H, D]
    extra = lambda t: torch.randn(200, H, D, generator=g).half()
    qp = torch.cat([pk(qd_), extra(qd_)]); kp = torch.cat([pk(kd_), extra(kd_)])
    vp = torch.cat([pk(vd_), extra(vd_)])
    cu = torch.tensor([0, n, n + 200], dtype=torch.int32)
    packed = heads.quantize(qp, kp, vp, cu, gran="block_sq")
    nb = (n + BLK - 1) // BLK
    for h in range(H):
        np.testing.assert_array_equal(packed.q_mean[h, :nb], dense.q_mean[0, h])
        np.testing.assert_array_equal(packed.q_codes[h, :nb * BLK], dense.q_codes[0, h])
        np.testing.assert_array_equal(packed.q_delta[h, :nb], dense.q_delta[0, h])
    rows = [0, 1, 127, 128, 299]
    for causal in (False, True):
        a = heads.emulate_rows(dense, vd_, None, [(0, h, i) for h in range(H) for i in rows], D,
                               causal, "fp16", gran="block_sq", k=kd_)
        b = heads.emulate_rows(packed, vp, cu, [(0, h, i) for h in range(H) for i in rows], D,
                               causal, "fp16", gran="block_sq", k=kp)
        for h in range(H):
            for i in rows:
                np.testing.assert_array_equal(a[(0, h, i)], b[(0, h, i)])

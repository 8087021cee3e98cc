"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print, exact rational arithmetic, library routines (torch casts, SDPA,
numpy integer matmul), closed forms and invariants.  They are chosen so that a
plausible slip in the oracle (a wrong rounding mode, a dropped rescale factor,
a transposed operand, a wrong block index or mask boundary) fails at least one.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import heads
from tests.exact import all_finite_fp16, fp32, quantize_exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            out[k.strip()] = [float(t) for t in v.split()]
    return out


# --- quantiser -------------------------------------------------------------------

def test_worked_outlier_example():
    """The page's worked example: [0.1, 0.2, 0.15, 1000] -> delta ~ 7.87, codes [0,0,0,127]."""
    g = _golden("p5_outlier_example.txt")
    A = np.array(g["A"], dtype=np.float32).reshape(1, -1)
    codes, delta = oracle.quant_block(A)
    assert codes.ravel().tolist() == [int(c) for c in g["codes"]]
    assert round(float(delta), int(g["delta_printed_digits"][0])) == g["delta_printed"][0]
    assert float(delta) == fp32(Fraction(1000) / 127)


def test_quantiser_exhaustive_fp16_against_exact_rationals():
    """Every finite fp16 value, quantised in a block with a seeded max |.|, equals
    the exact-rational evaluation of the quantiser's binary32 steps."""
    rng = np.random.default_rng(1)
    xs = all_finite_fp16().astype(np.float32)
    ratio = rng.uniform(1.0, 6.0, size=xs.shape).astype(np.float32)
    for x, r in zip(xs, ratio):
        ax = abs(float(x))
        amax = float(np.float16(min(65504.0, ax * float(r)))) if ax > 0 else 1.0
        amax = max(amax, ax)
        block = np.array([[x, amax]], dtype=np.float32)
        codes, delta = oracle.quant_block(block)
        c_exact, d_exact = quantize_exact(float(x), amax)
        assert int(codes[0, 0]) == c_exact, (x, amax)
        assert float(delta) == d_exact


def test_quantiser_error_bound_and_page_formula():
    """|x - code*delta| <= delta*(1/2 + 2^-15), the max element maps to +-127, and
    codes differ from the page's literal round(x/delta) by at most 1 (rarely)."""
    rng = np.random.default_rng(2)
    total = differ = 0
    for scale in (1e-3, 1.0, 37.0, 3e3):
        x = (rng.standard_normal((128, 64)) * scale).astype(np.float16).astype(np.float32)
        codes, delta = oracle.quant_block(x)
        d = float(delta)
        err = np.abs(x.astype(np.float64) - codes.astype(np.float64) * d)
        assert err.max() <= d * (0.5 + 2.0 ** -15)
        i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
        assert abs(int(codes[i])) == 127
        literal = np.rint(x.astype(np.float64) / d)
        assert np.abs(literal - codes).max() <= 1
        total += x.size
        differ += int((literal != codes).sum())
    assert differ / total < 1e-3


def test_integer_block_is_identity():
    """Integer values with max |.| = 127 give delta = 1 and codes equal to the values."""
    rng = np.random.default_rng(3)
    x = rng.integers(-127, 128, size=(128, 128)).astype(np.float32)
    x[5, 7] = -127.0
    codes, delta = oracle.quant_block(x)
    assert float(delta) == 1.0
    assert np.array_equal(codes.astype(np.float32), x)


def test_all_zero_block():
    codes, delta = oracle.quant_block(np.zeros((128, 64), np.float32))
    assert float(delta) == 0.0 and not codes.any()


def test_quant_head_padding_and_blocks():
    """Blocks are 128 consecutive tokens; the ragged last block is quantised on its
    own rows only and the padding rows are zero."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((300, 64)).astype(np.float32)
    x[270, 3] = 50.0                 # outlier only in the last block (rows 256..299)
    codes, delta = oracle.quant_head(x)
    assert codes.shape == (384, 64) and delta.shape == (3,)
    assert not codes[300:].any()
    for b in range(3):
        rows = x[b * 128:min(300, (b + 1) * 128)]
        c, d = oracle.quant_block(rows)
        assert float(d) == float(delta[b])
        assert np.array_equal(c, codes[b * 128:b * 128 + rows.shape[0]])
    assert float(delta[2]) == fp32(Fraction(50) / 127)


# --- K mean (smoothing) -------------------------------------------------------------

def test_k_mean_closed_form():
    """K = c_d + integer noise with zero per-channel sum  =>  mean is exactly c_d."""
    rng = np.random.default_rng(5)
    n, D = 1000, 64
    c = (rng.integers(-200, 200, size=D) / 8.0).astype(np.float32)
    half = rng.integers(-50, 51, size=(n // 2, D))
    noise = np.concatenate([half, -half], axis=0)
    rng.shuffle(noise, axis=0)
    k = (c[None, :] + noise).astype(np.float16).astype(np.float32)
    s, m, st = oracle.k_mean(k)
    assert st == 0
    assert np.array_equal(m, c)
    assert np.array_equal(s, (c.astype(np.float64) * n * 2 ** 24).astype(np.int64))


def test_k_mean_is_the_mean():
    """Against the exact rational mean: within one binary32 ulp (fp16 and bf16 data)."""
    rng = np.random.default_rng(6)
    for dt in (torch.float16, torch.bfloat16):
        k = torch.from_numpy(rng.standard_normal((37, 8)).astype(np.float32) * 3 + 1).to(dt)
        kf = k.float().numpy()
        _, m, st = oracle.k_mean(kf)
        assert st == 0
        for d in range(8):
            exact = sum(Fraction(float(v)) for v in kf[:, d]) / 37
            ulp = float(np.spacing(np.float32(float(exact))))
            assert abs(Fraction(float(m[d])) - exact) <= Fraction(ulp)


def test_k_mean_range_flag():
    k = np.ones((4, 8), np.float32)
    k[2, 3] = 70000.0
    _, _, st = oracle.k_mean(k)
    assert st == oracle.ORACLE_ERR_RANGE


# --- number formats ---------------------------------------------------------------

def test_e4m3_against_torch_cast():
    """Dense sweep of binary32 values in the finite range vs torch.float8_e4m3fn."""
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-464.0, 464.0, 40001, endpoint=False),
        rng.uniform(-1, 1, 20000) * 2.0 ** rng.integers(-12, 9, 20000),
        [0.0, -0.0, 2 ** -10, 2 ** -9, 1.5 * 2 ** -9, 2 ** -6, 448.0, -448.0, 464.0 - 2 ** -5],
    ]).astype(np.float32)
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_roundtrip_and_saturation():
    codes = [c for c in range(256) if (c & 0x7F) != 0x7F]
    dec = oracle.e4m3_decode(codes)
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(dec, ref)
    assert np.array_equal(oracle.e4m3_encode(dec.astype(np.float32)), np.array(codes, np.uint8))
    assert oracle.e4m3_encode([1e6, -500.0]).tolist() == [0x7E, 0xFE]


def test_fp16_bf16_rounding_against_torch():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.uniform(0, 1, 5000), 2.0 ** rng.uniform(-30, 0, 5000),
                        [2 ** -24, 2 ** -25, 3 * 2 ** -26, 1.0]]).astype(np.float32)
    for fn, dt in ((oracle.round_fp16, torch.float16), (oracle.round_bf16, torch.bfloat16)):
        ours = np.array([fn(float(v)) for v in x])
        ref = torch.from_numpy(x).to(dt).double().numpy()
        assert np.array_equal(ours, ref)


# --- QK^T ----------------------------------------------------------------------------

def test_qk_int_against_numpy_matmul():
    rng = np.random.default_rng(9)
    qc = rng.integers(-127, 128, size=(256, 128)).astype(np.int8)
    kc = rng.integers(-127, 128, size=(256, 128)).astype(np.int8)
    S = oracle.qk_int(qc, kc, 128, 128, 0, 256)
    ref = qc[128:256].astype(np.int64) @ kc[0:256].astype(np.int64).T
    assert np.array_equal(S.astype(np.int64), ref)


# --- R: fp64 reference ---------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_reference_against_sdpa(causal):
    rng = np.random.default_rng(10)
    n, D = 19, 8
    q, k, v = (rng.standard_normal((n, D)).astype(np.float32) for _ in range(3))
    rows = np.arange(n)
    out = oracle.attn_ref_rows(q, k, v, 0.3, causal, rows)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None], torch.from_numpy(k).double()[None],
        torch.from_numpy(v).double()[None], is_causal=causal, scale=0.3)[0].numpy()
    assert np.abs(out - ref).max() < 1e-12


def test_reference_smoothing_invariance():
    """softmax is unchanged by subtracting a per-channel constant from K."""
    rng = np.random.default_rng(11)
    n, D = 64, 16
    q, k, v = (rng.standard_normal((n, D)).astype(np.float64) for _ in range(3))
    k = k + rng.standard_normal(D) * 5
    kbar = k.mean(axis=0)
    k32 = k.astype(np.float32)
    ks = (k32.astype(np.float64) - kbar).astype(np.float32)
    a = oracle.attn_ref_rows(q, k32, v, 0.25, False, np.arange(n))
    b = oracle.attn_ref_rows(q, ks, v, 0.25, False, np.arange(n))
    # the only difference is the fp32 rounding of k - kbar (|k| ~ 5, ulp ~ 5e-7)
    assert np.abs(a - b).max() < 1e-5


# --- E: the quantised method ---------------------------------------------------------

def _emulate(q, k, v, causal, pv_mode, sm_scale=None, rows=None):
    """Run the oracle's own steps over a single-head [1,1,n,D] input."""
    n, D = q.shape[-2:]
    qz = heads.quantize(q, k, v, None, pv_mode)
    rows = list(range(n)) if rows is None else rows
    picks = [(0, 0, i) for i in rows]
    out = heads.emulate_rows(qz, v, None, picks, D, causal, pv_mode, sm_scale)
    return np.stack([out[p] for p in picks]), qz


@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
@pytest.mark.parametrize("causal", [False, True])
def test_emulation_constant_keys_gives_mean_of_values(causal, pv_mode):
    """K constant over tokens: smoothing makes K zero, every logit equal, so each
    output row is the (prefix) mean of the values actually multiplied."""
    n, D = 333, 64
    q, k, v = [t[None, None] for t in (torch.randn(n, D), torch.zeros(n, D), torch.randn(n, D))]
    k = (k + torch.randn(1, 1, 1, D) * 3).half()
    q, v = q.half(), v.half()
    out, qz = _emulate(q, k, v, causal, pv_mode)
    assert not qz.k_codes.any() and not qz.k_delta.any()
    if pv_mode == "fp16":
        vals = v[0, 0].double().numpy()
    else:
        vals = oracle.e4m3_decode(qz.v_codes[0, 0]).reshape(n, D) * qz.v_delta[0, 0][None, :]
    if causal:
        ref = np.cumsum(vals, axis=0) / np.arange(1, n + 1)[:, None]
    else:
        ref = np.broadcast_to(vals.mean(axis=0), (n, D))
    assert np.abs(out - ref).max() < 2e-6 * max(1.0, np.abs(vals).max())


@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
def test_emulation_constant_values(pv_mode):
    """V equal to c_d on every token: every row's output is c_d, up to the P rounding
    (relative 2^-11 for fp16 P; 2^-4 for e4m3 P; V codes are exact here)."""
    torch.manual_seed(12)
    n, D = 300, 64
    q = torch.randn(1, 1, n, D).half()
    k = (torch.randn(1, 1, n, D) + 2).half()
    c = torch.tensor([(-1) ** d * (1 + d / 16) for d in range(D)])
    v = c.expand(1, 1, n, D).half().contiguous()
    out, _ = _emulate(q, k, v, False, pv_mode)
    cd = v[0, 0, 0].double().numpy()
    tol = 2.0 ** -10 if pv_mode == "fp16" else 2.0 ** -3
    assert np.abs(out - cd).max() <= tol * np.abs(cd).max()


@pytest.mark.parametrize("pv_mode", ["fp16", "fp8"])
def test_emulation_causal_first_row_is_first_value(pv_mode):
    torch.manual_seed(13)
    n, D = 200, 128
    q, k, v = (torch.randn(1, 1, n, D).half() for _ in range(3))
    out, qz = _emulate(q, k, v, True, pv_mode, rows=[0])
    if pv_mode == "fp16":
        ref = v[0, 0, 0].double().numpy()
    else:
        ref = oracle.e4m3_decode(qz.v_codes[0, 0, 0]) * qz.v_delta[0, 0]
    assert np.abs(out[0] - ref).max() <= 1e-6 * np.abs(ref).max()


def _lossless_inputs(n, D, seed, q_exp=(0,), k_exp=(0,)):
    """q, k whose 128-token blocks are integer codes times a power of two 2^e_b, each
    block containing the code 127, and whose K blocks have zero channel sums; so
    deltaQ_b = 2^eq_b, deltaK_b = 2^ek_b exactly, the K mean is 0 and quantisation
    reproduces the values exactly."""
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(n, D)).astype(np.int64)
    k = rng.integers(-126, 127, size=(n, D)).astype(np.int64)
    for bi, b in enumerate(range(0, n, 128)):
        rows = slice(b, min(n, b + 128))
        q[b, 0] = 127
        k[b, 0] = 127
        kb = k[rows]
        for d in range(D):
            s = int(kb[:, d].sum())
            for r in range(kb.shape[0]):
                if s == 0:
                    break
                if r == 0 and d == 0:
                    continue
                step = max(-126 - kb[r, d], min(126 - kb[r, d], -s))
                kb[r, d] += step
                s += step
            assert s == 0
    qs = np.ones((n, 1)); ks = np.ones((n, 1))
    for bi, b in enumerate(range(0, n, 128)):
        qs[b:b + 128] = 2.0 ** q_exp[bi % len(q_exp)]
        ks[b:b + 128] = 2.0 ** k_exp[bi % len(k_exp)]
    v = rng.standard_normal((n, D)).astype(np.float16).astype(np.float32)
    return (q * qs).astype(np.float32), (k * ks).astype(np.float32), v


@pytest.mark.parametrize("causal", [False, True])
def test_emulation_lossless_quantisation_matches_reference(causal):
    """With exactly representable codes the only approximation left in E (16-bit
    P.V) is rounding P to fp16: |E - R| <= 2^-10 * max|v| (plus fp32 noise).
    Per-block power-of-two deltas make a wrong block index visible; a transposed
    operand, missing rescale or mask slip fails as well."""
    n, D = 300, 16
    q, k, v = _lossless_inputs(n, D, 14, q_exp=(0, -1, 1), k_exp=(-1, 0, 1))
    sm = 1.0 / 12000.0
    qt, kt, vt = (torch.from_numpy(x)[None, None].half() for x in (q, k, v))
    assert torch.equal(kt.float()[0, 0], torch.from_numpy(k))
    assert torch.equal(qt.float()[0, 0], torch.from_numpy(q))
    out, qz = _emulate(qt, kt, vt, causal, "fp16", sm_scale=sm)
    assert qz.q_delta[0, 0].tolist() == [1.0, 0.5, 2.0]
    assert qz.k_delta[0, 0].tolist() == [0.5, 1.0, 2.0]
    assert not qz.k_mean.any()
    ref = oracle.attn_ref_rows(q, k, v, float(np.float32(sm)), causal, np.arange(n))
    assert np.abs(out - ref).max() <= 2.0 ** -10 * np.abs(v).max() + 1e-5
    # the running maximum moves after the first key block for many rows, so the
    # rescale factor alpha is exercised
    logits = q.astype(np.float64) @ k.T.astype(np.float64) * sm
    if not causal:
        moved = logits[:, :128].max(axis=1) < logits.max(axis=1) - 0.5
        assert moved.mean() > 0.2


def test_v_fp8_quant_against_torch_cast():
    """Per-channel V scale: delta_d = max_t|v_td|/448 and codes = e4m3(v * 448/max|v|),
    checked against numpy's per-channel max and torch's float8_e4m3fn cast."""
    rng = np.random.default_rng(16)
    v = (rng.standard_normal((333, 64)) * rng.uniform(0.1, 10, 64)).astype(np.float16)
    v = v.astype(np.float32)
    v[:, 5] = 0.0
    codes, delta = oracle.quant_v_fp8(v)
    amax = np.abs(v).max(axis=0)
    assert np.array_equal(delta, (amax / np.float32(448)).astype(np.float32))
    s = np.where(amax > 0, np.float32(448) / np.where(amax > 0, amax, 1), 0).astype(np.float32)
    ref = torch.from_numpy((v * s[None, :]).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(codes, ref.view(torch.uint8).numpy())


def test_emulation_close_to_reference_on_gaussian_data():
    """On the smoothing workload recipe, E agrees with R to cosine > 0.9999 (fp16 P)
    and > 0.999 (fp8 P), and K smoothing is what makes the first one hold."""
    torch.manual_seed(15)
    n, D = 384, 64
    q = torch.randn(1, 1, n, D).half()
    k = (torch.randn(1, 1, n, D) + torch.randn(1, 1, 1, D) * 4).half()
    v = torch.randn(1, 1, n, D).half()
    rows = list(range(0, n, 7))
    ref = oracle.attn_ref_rows(q[0, 0].float().numpy(), k[0, 0].float().numpy(),
                               v[0, 0].float().numpy(), 0.125, False, rows)
    def cos(a):
        return (a.ravel() @ ref.ravel()) / np.linalg.norm(a) / np.linalg.norm(ref)
    for mode, bar in (("fp16", 0.9999), ("fp8", 0.999)):
        out, _ = _emulate(q, k, v, False, mode, rows=rows)
        assert cos(out) > bar, (mode, cos(out))
    # the same steps with the smoothing left out fall below the bar
    qz = heads.quantize(q, k, v, None, "fp16")
    qz.k_codes[0, 0], qz.k_delta[0, 0] = oracle.quant_head(k[0, 0].float().numpy(), None)
    picks = [(0, 0, i) for i in rows]
    o = heads.emulate_rows(qz, v, None, picks, D, False, "fp16")
    unsmoothed = np.stack([o[p] for p in picks])
    assert cos(unsmoothed) < 0.9999


@pytest.mark.parametrize("causal", [False, True])
def test_emulation_rescale_threshold_changes_rounding_only(causal):
    """The threshold tau of the running maximum cancels in O / l: tau = 8 and
    tau = 0 differ only through the rounding of P (|diff| <= 2^-10 max|v|), and
    both stay within that bound of the fp64 reference on lossless inputs."""
    n, D = 300, 16
    q, k, v = _lossless_inputs(n, D, 17, q_exp=(0, -1, 1), k_exp=(-1, 0, 1))
    sm = 1.0 / 12000.0
    qt, kt, vt = (torch.from_numpy(x)[None, None].half() for x in (q, k, v))
    qz = heads.quantize(qt, kt, vt, None, "fp16")
    outs = {}
    for tau in (0.0, 8.0):
        outs[tau] = oracle.attn_emul_rows(qz.q_codes[0, 0], qz.q_delta[0, 0], qz.k_codes[0, 0],
                                          qz.k_delta[0, 0], n, D, sm, causal, "fp16",
                                          np.arange(n), v=v, tau=tau)
    bound = 2.0 ** -10 * np.abs(v).max() + 1e-5
    assert np.abs(outs[0.0] - outs[8.0]).max() <= bound
    ref = oracle.attn_ref_rows(q, k, v, float(np.float32(sm)), causal, np.arange(n))
    assert np.abs(outs[8.0] - ref).max() <= bound
    assert not np.array_equal(outs[0.0], outs[8.0])   # the threshold is in effect


# ------------------------------------------------------ grouped-query heads --

def test_repeat_kv_matches_repeat_interleave():
    """The oracle's head mapping equals the library routine it restates."""
    x = torch.randn(2, 3, 5, 4, generator=torch.Generator().manual_seed(3))
    for g in (1, 2, 4):
        assert torch.equal(heads.repeat_kv(x, g), torch.repeat_interleave(x, g, dim=1))


def test_grouped_reference_uses_the_kv_head_of_each_group():
    """Brute force: with each key/value head filled with its own constant value
    vector, every query head's output is the value of key/value head h // g."""
    B, Hkv, g, N, D = 1, 3, 2, 7, 4
    gen = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hkv * g, N, D, generator=gen)
    k = torch.randn(B, Hkv, N, D, generator=gen)
    v = torch.zeros(B, Hkv, N, D)
    for h in range(Hkv):
        v[:, h] = float(h + 1)  # softmax weights sum to 1: output = h + 1
    kr, vr = heads.repeat_kv(k, g), heads.repeat_kv(v, g)
    for hq in range(Hkv * g):
        out = oracle.attn_ref_rows(q[0, hq].numpy(), kr[0, hq].numpy(), vr[0, hq].numpy(),
                                   oracle.default_sm_scale(D), False, np.arange(N))
        assert np.allclose(out, hq // g + 1.0, atol=1e-12)


# ------------------------------------------------------- per-token deltas --

def test_per_token_quantiser_is_the_block_quantiser_on_each_row():
    """Per-token granularity = the quantiser with one-row blocks: every row's
    delta and codes match the exact rational quantiser of that row alone."""
    gen = torch.Generator().manual_seed(21)
    x = (torch.randn(37, 16, generator=gen) * 3).half().float().numpy()
    x[5] = 0.0                                     # an all-zero row: delta 0, codes 0
    codes, delta = oracle.quant_head(x, None, 1)
    assert codes.shape == (37, 16) and delta.shape == (37,)
    for r in range(37):
        amax = float(np.abs(x[r]).max())
        for d in range(16):
            c, dl = quantize_exact(float(x[r, d]), amax)
            assert codes[r, d] == c
        assert delta[r] == (dl if amax > 0 else 0.0)


def _per_token_lossless(n, D, seed):
    """Rows of integer codes with a +-127 in channel 0 (so each row's delta is
    its power-of-two scale exactly); K rows in pairs (r, r+1) with opposite
    codes and equal scales, so every channel of K sums to zero (mean 0)."""
    rng = np.random.default_rng(seed)
    q = rng.integers(-126, 127, size=(n, D)).astype(np.float64)
    q[:, 0] = 127
    qs = np.array([2.0 ** ((r % 3) - 1) for r in range(n)])
    k = np.zeros((n, D))
    ks = np.zeros(n)
    for r in range(0, n, 2):
        row = rng.integers(-126, 127, size=D).astype(np.float64)
        row[0] = 127
        k[r], k[r + 1] = row, -row
        ks[r] = ks[r + 1] = 2.0 ** ((r // 2) % 3 - 1)
    return (q * qs[:, None]).astype(np.float32), (k * ks[:, None]).astype(np.float32), qs, ks


@pytest.mark.parametrize("causal", [False, True])
def test_per_token_emulation_lossless_matches_reference(causal):
    """Exact per-token codes: the only approximation left (16-bit P.V) is P's
    fp16 rounding; per-row and per-key deltas that differ by powers of two make
    a wrong index visible."""
    n, D = 200, 16
    q, k, qs, ks = _per_token_lossless(n, D, 4)
    v = np.random.default_rng(5).standard_normal((n, D)).astype(np.float32)
    qt, kt, vt = (torch.from_numpy(a)[None, None].half() for a in (q, k, v))
    assert torch.equal(qt.float()[0, 0], torch.from_numpy(q))
    assert torch.equal(kt.float()[0, 0], torch.from_numpy(k))
    qz = heads.quantize(qt, kt, vt, None, "fp16", gran="token")
    assert np.array_equal(qz.q_delta[0, 0, :n], qs.astype(np.float32))
    assert np.array_equal(qz.k_delta[0, 0, :n], ks.astype(np.float32))
    assert not qz.k_mean.any() and not qz.q_delta[0, 0, n:].any()
    sm = 1.0 / 12000.0
    picks = [(0, 0, i) for i in range(n)]
    emu = heads.emulate_rows(qz, vt, None, picks, D, causal, "fp16", sm, gran="token")
    out = np.stack([emu[p] for p in picks])
    ref = oracle.attn_ref_rows(q, k, vt[0, 0].float().numpy(), float(np.float32(sm)), causal,
                               np.arange(n))
    assert np.abs(out - ref).max() <= 2.0 ** -10 * np.abs(v).max() + 1e-5


def test_per_token_emulation_follows_its_rounding_sequence():
    """One query row over three keys in one tile, computed with exact rationals
    along the documented steps (y = fp32(S dK_j), c = fp32(dQ kappa),
    mb = fp32(max y * c), arg = fp32(y c - mb), p = fp32(2^arg), P = fp16(p),
    out = fp32(fp32(sum P v) / fp32(sum p))): the C emulation agrees exactly."""
    from fractions import Fraction as Fr
    import math
    qc = np.array([[3, -7, 11, 2]], np.int8)
    kc = np.array([[5, 1, -2, 9], [-4, 8, 3, 1], [7, 7, -7, 0]], np.int8)
    qd = np.array([0.0123], np.float32)
    kd = np.array([0.031, 0.0207, 0.0444], np.float32)
    v = np.array([[1.5, -2.0, 0.25, 3.0], [0.5, 1.0, -1.0, 2.0], [-0.75, 0.125, 2.5, -1.5]],
                 np.float32)
    sm = 0.5
    kap = oracle.kappa(sm)
    got = oracle.attn_emul_rows(qc, qd, kc, kd, 3, 4, sm, False, "fp16", [0], v=v,
                                per_token=True, tau=8.0)[0]
    S = [int(np.dot(qc[0].astype(np.int64), kc[j].astype(np.int64))) for j in range(3)]
    y = [fp32(Fr(S[j]) * Fr(float(kd[j]))) for j in range(3)]
    c = fp32(Fr(float(qd[0])) * Fr(float(kap)))
    mb = fp32(Fr(max(y)) * Fr(c))
    args = [fp32(Fr(y[j]) * Fr(c) - Fr(mb)) for j in range(3)]
    p = [float(np.float32(math.pow(2.0, a))) for a in args]
    P = [float(np.float16(x)) for x in p]
    l = fp32(sum(Fr(x) for x in p))
    want = [fp32(fp32(sum(Fr(P[j]) * Fr(float(v[j, d])) for j in range(3))) / Fr(l))
            for d in range(4)]
    assert got.tolist() == want


def test_per_token_varlen_layout_matches_dense_per_sequence():
    """Packed per-token quantisation = the dense per-token quantisation of each
    sequence, placed at the sequence's code rows (deltas one per code row)."""
    lens = [5, 130, 0, 3]
    gen = torch.Generator().manual_seed(8)
    T, H, D = sum(lens), 2, 16
    q = (torch.randn(T, H, D, generator=gen) * 2).half()
    k = (torch.randn(T, H, D, generator=gen) + 1).half()
    cu = torch.tensor([0, 5, 135, 135, 138], dtype=torch.int32)
    qz = heads.quantize(q, k, None, cu, "fp16", gran="token")
    r0 = 0
    for s, n in enumerate(lens):
        if n == 0:
            continue
        qs, ks = q[cu[s]:cu[s + 1]], k[cu[s]:cu[s + 1]]
        dz = heads.quantize(qs.permute(1, 0, 2)[None].contiguous(),
                            ks.permute(1, 0, 2)[None].contiguous(), None, None, "fp16",
                            gran="token")
        for h in range(H):
            assert np.array_equal(qz.q_codes[h, r0:r0 + n], dz.q_codes[0, h, :n])
            assert np.array_equal(qz.q_delta[h, r0:r0 + n], dz.q_delta[0, h, :n])
            assert np.array_equal(qz.k_codes[h, r0:r0 + n], dz.k_codes[0, h, :n])
            assert np.array_equal(qz.k_delta[h, r0:r0 + n], dz.k_delta[0, h, :n])
        r0 += ((n + 127) // 128) * 128


# --------------------------------------------- E exact: powers-of-two inputs --

def _kappa_one_scale() -> float:
    """An fp32 sm_scale with kappa = fp32(sm_scale * log2 e) = 1 exactly, so the
    base-2 logits are the dequantised scores themselves."""
    sm = float(np.float32(math.log(2.0)))
    assert float(oracle.kappa(sm)) == 1.0
    return sm


def _exact_inputs(n, D, seed, eq=(0, 1), ek=(-1, 0, -1), nz=(1, 2, 2), ev=(-8, -7, -6)):
    """q, k, v for which every step of E is exact and every p is a power of two.

    Codes: Q row r of block I has three entries +-1 in channels 2..D-1
    (times 2^eq_I); K rows nz_J entries +-1 (+-2 in blocks with ek_J = -1) with
    zero channel sums per block (times 2^ek_J; the first block's logits are
    smaller, so the running maximum moves later); each Q block holds the code 127
    in channel 0 and each K block 127 and -127 in channel 1, channels no other
    operand touches, so the deltas are exactly 2^eq_I, 2^ek_J and the K mean is
    0.  With kappa = 1 the base-2 logit t_ij = S_ij 2^(eq_I + ek_J) is an
    integer in [-8, 8] (eq in {0, 1}, ek in {-1, 0}).
    V: e4m3 values times 2^ev_d per channel, each channel holding +-448, so V's
    FP8 codes and scales reproduce it exactly (and it is exact in fp16)."""
    rng = np.random.default_rng(seed)
    q = np.zeros((n, D), np.int64)
    k = np.zeros((n, D), np.int64)
    for i in range(n):
        for d in rng.choice(np.arange(2, D), size=3, replace=False):
            q[i, d] = rng.choice([-1, 1])
    for b in range(0, n, 128):
        rows = np.arange(b, min(n, b + 128))
        half = len(rows) // 2
        mag = 2 if ek[(b // 128) % len(ek)] == -1 else 1
        for r in rows[:half]:  # pairs of opposite rows: zero channel sums
            for d in rng.choice(np.arange(2, D), size=nz[(b // 128) % len(nz)], replace=False):
                k[r, d] = mag * rng.choice([-1, 1])
        k[rows[half:2 * half]] = -k[rows[:half]]
        q[b, 0] = 127
        k[b, 1], k[rows[-1] if len(rows) > 1 else b, 1] = 127, -127
    qs = np.array([2.0 ** eq[(i // 128) % len(eq)] for i in range(n)])[:, None]
    ks = np.array([2.0 ** ek[(i // 128) % len(ek)] for i in range(n)])[:, None]
    codes = rng.integers(0, 126, size=(n, D))          # e4m3 magnitudes below 448
    vmag = oracle.e4m3_decode(codes.astype(np.uint8)).reshape(n, D)
    vmag[rng.integers(0, n, size=D), np.arange(D)] = 448.0
    vsign = rng.choice([-1.0, 1.0], size=(n, D))
    v = vmag * vsign * np.array([2.0 ** ev[d % len(ev)] for d in range(D)])[None, :]
    return (q * qs).astype(np.float32), (k * ks).astype(np.float32), v.astype(np.float32)


EXACT_VARIANTS = [
    ("fp16", {}),
    ("fp8", {}),
    ("fp16", dict(kv=64, tau=8.0)),
    ("fp8", dict(p8_exp=True)),
]


@pytest.mark.parametrize("pv_mode,opts", EXACT_VARIANTS)
@pytest.mark.parametrize("causal", [False, True])
def test_emulation_exact_on_power_of_two_probabilities(pv_mode, opts, causal):
    """Every p is 2^-a with a <= 15: P is exact in fp16, 448 p is exact in e4m3,
    the rescale factors are powers of two, and the row sums are exact in fp32.
    So E equals the fp64 reference up to the fp32 rounding of the partial sums
    and of the final division (|E - R| <= 1e-5 max|v|), in either P.V mode and
    in the other evaluation orders.  A rescale applied one block late or
    never, a partial flushed twice or not at all, the delta of a wrong block,
    a transposed operand or a mask slip each move rows by O(|v|)."""
    n, D = 300, 16
    q, k, v = _exact_inputs(n, D, seed=41 + causal)
    sm = _kappa_one_scale()
    qt, kt, vt = (torch.from_numpy(x)[None, None].half() for x in (q, k, v))
    for a, b in ((qt, q), (kt, k), (vt, v)):
        assert np.array_equal(a[0, 0].float().numpy(), b)
    qz = heads.quantize(qt, kt, vt, None, pv_mode)
    assert qz.q_delta[0, 0].tolist() == [1.0, 2.0, 1.0]
    assert qz.k_delta[0, 0].tolist() == [0.5, 1.0, 0.5]
    assert not qz.k_mean.any()
    if pv_mode == "fp8":
        dec = oracle.e4m3_decode(qz.v_codes[0, 0]).reshape(n, D) * qz.v_delta[0, 0][None, :]
        assert np.array_equal(dec, v.astype(np.float64))
    # preconditions: integer logits with a spread of at most 15 per row, and a
    # running maximum that moves after the first block for many rows
    t = (q.astype(np.float64) @ k.T.astype(np.float64))
    assert np.array_equal(t, np.round(t))
    mask = np.tril(np.ones((n, n), bool)) if causal else np.ones((n, n), bool)
    tm = np.where(mask, t, np.nan)
    assert (np.nanmax(tm, axis=1) - np.nanmin(tm, axis=1)).max() <= 15
    first = np.nanmax(np.where(mask[:, :128], t[:, :128], np.nan), axis=1)
    assert (first[128:] < np.nanmax(tm, axis=1)[128:]).mean() > 0.3
    picks = [(0, 0, i) for i in range(n)]
    out = heads.emulate_rows(qz, vt, None, picks, D, causal, pv_mode, sm, **opts)
    E = np.stack([out[p] for p in picks])
    R = oracle.attn_ref_rows(q, k, v, sm, causal, np.arange(n))
    assert np.abs(E - R).max() <= 1e-5 * np.abs(v).max()


@pytest.mark.parametrize("causal", [False, True])
def test_emulation_fp8_within_the_rounding_of_p(causal):
    """FP8 P.V on exactly quantisable Q, K (power-of-two block deltas, so the
    running maximum moves between blocks) and exactly e4m3-representable V:
    the only approximation left in E is P^ = e4m3(448 p), whose error is at most
    2^-4 p (normal range) or 2^-10 / 448 (subnormal), so for every row i and
    channel d
        |E_id - R_id| <= sum_j max(2^-4 p_ij, 2^-10/448) |v_jd| / sum_j p_ij
    with p_ij = exp(logit_ij - max_j logit_ij) from the fp64 reference."""
    n, D = 300, 16
    q, k, _ = _lossless_inputs(n, D, 18, q_exp=(0, -1, 1), k_exp=(-1, 0, 1))
    _, _, v = _exact_inputs(n, D, seed=19)
    sm = 1.0 / 12000.0
    qt, kt, vt = (torch.from_numpy(x)[None, None].half() for x in (q, k, v))
    qz = heads.quantize(qt, kt, vt, None, "fp8")
    assert qz.q_delta[0, 0].tolist() == [1.0, 0.5, 2.0] and not qz.k_mean.any()
    picks = [(0, 0, i) for i in range(n)]
    out = heads.emulate_rows(qz, vt, None, picks, D, causal, "fp8", float(np.float32(sm)))
    E = np.stack([out[p] for p in picks]).astype(np.float64)
    R = oracle.attn_ref_rows(q, k, v, float(np.float32(sm)), causal, np.arange(n))
    logit = q.astype(np.float64) @ k.T.astype(np.float64) * float(np.float32(sm))
    if causal:
        logit = np.where(np.tril(np.ones((n, n), bool)), logit, -np.inf)
    p = np.exp(logit - logit.max(axis=1, keepdims=True))
    perr = np.maximum(2.0 ** -4 * p, np.where(p > 0, 2.0 ** -10 / 448, 0.0))
    bound = perr @ np.abs(v.astype(np.float64)) / p.sum(axis=1, keepdims=True)
    slack = 1e-5 * np.abs(v).max()
    assert np.all(np.abs(E - R) <= bound + slack)
    # the bound is not vacuous: P^'s rounding shows, well inside it
    assert 1e-4 * bound.max() < np.abs(E - R).max() < 0.5 * bound.max()

"""The C-ABI library loads, exports every function include/sage.h declares, and
its host-side logic (sizes, argument validation) behaves as documented.  No
call here reaches the GPU: every call either computes sizes or is rejected by
host-side validation before anything is launched."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from quantized_attention_07_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage.h")

FAKE = 0x10000  # a 16-byte aligned non-null "device pointer" never dereferenced


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions() -> list[str]:
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    """The entry points of the hot path's C ABI: smoothing + quantisation of Q
    and K (sage_quant_qk), the whole forward pass over [B, H, N, D]
    (sage_attn_fwd: q, k, v, out, B, H, N, D, causal, sm_scale, pv_mode) and
    its variable-length variant taking cu_seqlens; plus the split stages, the
    status word and the kernel's own int32 QK^T dump."""
    names = declared_functions()
    for required in ("sage_quant_qk", "sage_attn_fwd", "sage_attn_fwd_varlen", "sage_quantize",
                     "sage_attn_quantized", "sage_quantize_varlen", "sage_sync_status",
                     "sage_attn_quantized_dump_s"):
        assert required in names
    text = open(HEADER).read()
    sig = re.search(r"sage_status_t sage_attn_fwd\((.*?)\);", text, flags=re.S).group(1)
    params = [p.split()[-1].strip("*") for p in sig.split(",")]
    for p in ("q", "k", "v", "out", "B", "H", "N", "D", "causal", "sm_scale", "pv_mode"):
        assert p in params, p
    sig = re.search(r"sage_status_t sage_attn_fwd_varlen\((.*?)\);", text, flags=re.S).group(1)
    assert "cu_seqlens" in sig
    sig = re.search(r"sage_status_t sage_quant_qk\((.*?)\);", text, flags=re.S).group(1)
    params = [p.split()[-1].strip("*") for p in sig.split(",")]
    for p in ("q", "k", "B", "H", "N", "D", "q_codes", "q_scale", "k_codes", "k_scale",
              "k_mean", "ws"):
        assert p in params, p


def test_quant_qk_and_dump_reject_bad_arguments(lib):
    """Host-side validation of the two newer entry points (nothing launches)."""
    qa = dict(q=FAKE, k=FAKE, in_dt=0, B=1, H=2, N=256, D=64, qc=FAKE, qs=FAKE, kc=FAKE, ks=FAKE,
              km=FAKE, ws=FAKE, wsb=1 << 30, st=None)
    for bad in (dict(D=96), dict(N=0), dict(in_dt=2), dict(q=None), dict(kc=FAKE + 4),
                dict(ws=None)):
        a = dict(qa, **bad)
        assert lib.sage_quant_qk(*a.values()) == 1, bad
    a = dict(qa, wsb=16)
    assert lib.sage_quant_qk(*a.values()) == 3
    da = dict(qc=FAKE, qs=FAKE, kc=FAKE, ks=FAKE, v=FAKE, vc=FAKE, vs=FAKE, out=FAKE, v_dt=0,
              out_dt=2, B=1, H=2, N=256, D=64, causal=0, sm=0.0, pv=0, s=FAKE, ws=FAKE,
              wsb=1 << 30, st=None)
    for bad in (dict(D=96), dict(s=None), dict(s=FAKE + 4), dict(out_dt=5), dict(pv=3)):
        a = dict(da, **bad)
        assert lib.sage_attn_quantized_dump_s(*a.values()) == 1, bad
    a = dict(da, v_dt=1)  # bf16 V with 16-bit P.V: no diagnostic instance
    assert lib.sage_attn_quantized_dump_s(*a.values()) == 2


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # and the binding attaches a signature to each of them
    assert set(declared_functions()) == set(_lib.SIGNATURES)


def test_workspace_sizes(lib):
    B, H, N, D = 1, 32, 32768, 128
    NP = N
    fp16 = lib.sage_workspace_bytes(B, H, N, D, 0)
    fp8 = lib.sage_workspace_bytes(B, H, N, D, 1)
    codes = 2 * B * H * NP * D
    assert codes < fp16 < codes + (1 << 20)
    assert fp8 - fp16 >= B * H * N * D            # FP8 V codes
    assert lib.sage_workspace_bytes(1, 1, 100, 96, 0) == 0   # rejected shapes -> 0
    assert lib.sage_workspace_bytes(1, 1, 0, 64, 0) == 0
    assert lib.sage_workspace_bytes(1, 1, 1 << 23, 64, 0) == 0
    v = lib.sage_workspace_bytes_varlen(34000, 8, 32, 128, 1)
    assert v > 2 * 32 * 34000 * 128
    assert lib.sage_scratch_bytes(2, 16, 128) >= 256 + 2 * 16 * 128 * 12


def test_status_strings(lib):
    for code, name in ((0, b"SAGE_OK"), (1, b"SAGE_ERR_INVALID_ARG"), (5, b"SAGE_ERR_TIMEOUT"),
                       (6, b"SAGE_ERR_BAD_SEQLENS"), (7, b"SAGE_ERR_RANGE")):
        assert lib.sage_status_string(code) == name


def _fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, in_dt=0, out_dt=0, B=1, H=2, N=256, D=64,
             causal=0, sm_scale=0.0, pv_mode=0, ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.sage_attn_fwd(*a.values())


@pytest.mark.parametrize("bad", [dict(D=96), dict(D=0), dict(N=0), dict(B=0), dict(H=-1),
                                 dict(pv_mode=2), dict(in_dt=2), dict(out_dt=7),
                                 dict(q=None), dict(v=FAKE + 8), dict(out=FAKE + 2),
                                 dict(ws=None), dict(sm_scale=float("nan")),
                                 dict(N=(1 << 22) + 1), dict(B=300, H=300)])
def test_invalid_arguments_rejected_on_host(lib, bad):
    assert _fwd(lib, **bad) == 1


def test_small_workspace_rejected_on_host(lib):
    need = lib.sage_workspace_bytes(1, 2, 256, 64, 0)
    assert _fwd(lib, ws_bytes=need - 1) == 3


def test_varlen_and_stage_validation(lib):
    f = lib.sage_attn_fwd_varlen
    # batch 0, D=96, null cu_seqlens
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 0, 100, 100, 2, 64, 0, 0.0, 0, FAKE, 1 << 40, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 100, 100, 2, 96, 0, 0.0, 0, FAKE, 1 << 40, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 0, None, 1, 100, 100, 2, 64, 0, 0.0, 0, FAKE, 1 << 40, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 1, 100, 100, 2, 64, 0, 0.0, 0, FAKE, 1000, None) == 3
    q = lib.sage_quantize
    # FP8 mode without V codes
    assert q(FAKE, FAKE, FAKE, 0, 1, 2, 256, 64, 1, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
             FAKE, 1 << 30, None) == 1
    assert q(FAKE, FAKE, None, 0, 1, 2, 256, 64, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
             FAKE, 16, None) == 3
    t = (ctypes.c_int32 * 3)(0, 5, 0)   # tile row out of range for NP = 256
    assert lib.sage_qk_int8_tiles(FAKE, FAKE, 1, 256, 64, ctypes.cast(t, ctypes.c_void_p), 1,
                                  FAKE, FAKE, 1 << 20, None) == 1


def test_grouped_query_sizes_and_validation(lib):
    B, H, N, D = 1, 8, 1024, 128
    full = lib.sage_workspace_bytes(B, H, N, D, 1)
    assert lib.sage_workspace_bytes_gqa(B, H, H, N, D, 1) == full   # Hkv = H: the plain layout
    g4 = lib.sage_workspace_bytes_gqa(B, H, 2, N, D, 1)
    # K codes and FP8 V codes shrink with the key/value heads; Q codes do not
    assert full - g4 >= (H - 2) * N * D * 2 and g4 > B * H * N * D
    for hkv in (0, 3, 16, -1):                                    # must divide H, 1 <= Hkv <= H
        assert lib.sage_workspace_bytes_gqa(B, H, hkv, N, D, 0) == 0
    f = lib.sage_attn_fwd_gqa
    args = [FAKE, FAKE, FAKE, FAKE, 0, 0, 1, 8, 2, 256, 64, 0, 0.0, 0, FAKE, 1 << 40, None]
    bad = list(args); bad[8] = 3
    assert f(*bad) == 1
    bad = list(args); bad[10] = 96
    assert f(*bad) == 1
    small = list(args); small[15] = lib.sage_workspace_bytes_gqa(1, 8, 2, 256, 64, 0) - 1
    assert f(*small) == 3


def test_grouped_varlen_sizes_and_validation(lib):
    full = lib.sage_workspace_bytes_varlen(5000, 4, 8, 128, 1)
    assert lib.sage_workspace_bytes_varlen_gqa(5000, 4, 8, 8, 128, 1) == full
    assert 0 < lib.sage_workspace_bytes_varlen_gqa(5000, 4, 8, 2, 128, 1) < full
    assert lib.sage_workspace_bytes_varlen_gqa(5000, 4, 8, 3, 128, 1) == 0
    f = lib.sage_attn_fwd_varlen_gqa
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 0, FAKE, 4, 100, 300, 8, 3, 64, 0, 0.0, 0, FAKE, 1 << 40,
             None) == 1


def test_q_smoothing_sizes_and_validation(lib):
    """Q smoothing's workspace adds the block means and the fp32 per-key mean
    term; packed batches size the term from max_seqlen; the plain split-stage
    entry points refuse the smoothing granularity."""
    B, H, N, D = 1, 4, 1000, 64
    NB = (N + 127) // 128
    al = lambda x: (x + 255) // 256 * 256
    plain = lib.sage_workspace_bytes_ex(B, H, H, N, D, 1, 0)
    sq = lib.sage_workspace_bytes_ex(B, H, H, N, D, 1, 2)
    assert sq == plain + al(B * H * NB * D * 4) + al(B * H * NB * NB * 128 * 4)
    assert lib.sage_workspace_bytes_ex(B, H, H, N, D, 1, 3) == 0        # unknown granularity
    # the mean term of R query blocks at a time: R even below NB, clamped to NB
    sqr = lambda r: lib.sage_workspace_bytes_sq(B, H, H, N, D, 1, r)
    assert sqr(NB) == sqr(NB + 5) == sq
    assert sqr(2) == plain + al(B * H * NB * D * 4) + al(B * H * 2 * NB * 128 * 4)
    assert sqr(4) - sqr(2) == B * H * 2 * NB * 128 * 4
    assert sqr(3) == sqr(0) == sqr(-2) == 0
    assert lib.sage_workspace_bytes_sq(B, H, H, N, 96, 1, 2) == 0      # D
    # by default the term holds as many query blocks as fit 256 MiB (at least 2)
    Bl, Hl, Nl, Dl = 1, 32, 32768, 128
    NBl = Nl // 128
    row = Bl * Hl * NBl * 128 * 4                                      # 4 MiB per query block
    base = lib.sage_workspace_bytes_ex(Bl, Hl, Hl, Nl, Dl, 0, 0)
    assert lib.sage_workspace_bytes_ex(Bl, Hl, Hl, Nl, Dl, 0, 2) == (
        base + al(Bl * Hl * NBl * Dl * 4) + (256 << 20) // row * row)
    huge = lib.sage_workspace_bytes_ex(1, 1024, 1024, 1 << 20, 64, 0, 2)
    assert huge == lib.sage_workspace_bytes_sq(1, 1024, 1024, 1 << 20, 64, 0, 2)
    # packed: 0 through the _ex query (no max_seqlen), sized by the _sq query
    assert lib.sage_workspace_bytes_varlen_ex(5000, 4, 8, 8, 128, 1, 2) == 0
    short = lib.sage_workspace_bytes_varlen_sq(5000, 4, 1000, 8, 8, 128, 1)
    long_ = lib.sage_workspace_bytes_varlen_sq(5000, 4, 4000, 8, 8, 128, 1)
    base = lib.sage_workspace_bytes_varlen_ex(5000, 4, 8, 8, 128, 1, 0)
    assert base < short < long_
    assert lib.sage_workspace_bytes_varlen_sq(5000, 4, -1, 8, 8, 128, 1) == 0
    # the plain split stages refuse qk_gran 2 before touching anything
    q = lib.sage_quantize_ex
    assert q(FAKE, FAKE, FAKE, 0, B, H, H, N, D, 0, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
             FAKE, 1 << 40, None) == 1
    a = lib.sage_attn_quantized_ex
    assert a(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, B, H, H, N, D, 0, 0.0, 0, 2,
             FAKE, 1 << 40, None) == 1
    # the smoothing stages validate like the others (D = 96 rejected)
    qs = lib.sage_quantize_sq
    assert qs(FAKE, FAKE, FAKE, 0, B, H, H, N, 96, 0, 0, 0.0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
              FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == 1
    aq = lib.sage_attn_quantized_sq
    assert aq(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0, B, H, H, N, 96, 0, 0.0,
              0, FAKE, 1 << 40, None) == 1

"""CPU oracle for the SageAttention 8-bit forward pass -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and the
two share no code: the arithmetic lives in ``sage_oracle.c`` (plain C, one
IEEE operation per stated step), this file only marshals numpy arrays.

Entry points work on one (sequence, head) at a time, on fp32 arrays holding the
exact values of the 16-bit inputs; ``heads.py`` runs them over whole
workloads.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-Wall", "-Wextra"]

ORACLE_OK = 0
ORACLE_ERR_RANGE = 1

# The plain form of the method (see sage_oracle.c): the online softmax and
# the FP8 two-level flush run over the 128-token key blocks of the quantised K,
# with the plain running maximum.  Other evaluation orders (shorter key tiles,
# a threshold on moving the maximum, the FP8 P scale applied in the exponent,
# a fixed-order fp32 Q-smoothing term) are parameters of the calls below.
BLOCK = 128


def build(force: bool = False) -> str:
    """Compile sage_oracle.c into liboracle.so (gcc, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.oracle_round_fp16.argtypes = [f64]; L.oracle_round_fp16.restype = f64
        L.oracle_round_bf16.argtypes = [f64]; L.oracle_round_bf16.restype = f64
        L.oracle_e4m3_encode.argtypes = [f32]; L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]; L.oracle_e4m3_decode.restype = f64
        L.oracle_k_mean.argtypes = [P, i64, i32, i64, P, P]; L.oracle_k_mean.restype = i32
        L.oracle_quant_block.argtypes = [P, i32, i32, i64, P, P]; L.oracle_quant_block.restype = f32
        L.oracle_quant_head.argtypes = [P, i64, i32, i64, P, i32, P, P]; L.oracle_quant_head.restype = None
        L.oracle_quant_v_fp8.argtypes = [P, i64, i32, i64, P, P]; L.oracle_quant_v_fp8.restype = None
        L.oracle_qk_int.argtypes = [P, P, i32, i64, i32, i64, i32, P]; L.oracle_qk_int.restype = None
        L.oracle_attn_ref_rows.argtypes = [P, P, P, i64, i32, i64, i64, i64, f64, i32, P, i64, P]
        L.oracle_attn_ref_rows.restype = None
        L.oracle_attn_emul_rows.argtypes = [P, P, P, P, P, i64, P, P, i64, i32, i32, i32, f32, f32,
                                            i32, i32, i32, P, i64, P, i32, P, i64, i32]
        L.oracle_attn_emul_rows.restype = None
        for name in ("oracle_q_smooth_bias", "oracle_q_smooth_bias_fma"):
            getattr(L, name).argtypes = [P, i64, P, i64, i32, i64, P, f32, P, i64]
            getattr(L, name).restype = None
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


# --- number formats ---------------------------------------------------------

def round_fp16(x: float) -> float:
    return lib().oracle_round_fp16(float(x))


def round_bf16(x: float) -> float:
    return lib().oracle_round_bf16(float(x))


def e4m3_encode(x) -> np.ndarray:
    x = _f32(x).ravel()
    f = lib().oracle_e4m3_encode
    return np.array([f(float(v)) for v in x], dtype=np.uint8)


def e4m3_decode(c) -> np.ndarray:
    c = np.asarray(c, dtype=np.uint8).ravel()
    f = lib().oracle_e4m3_decode
    return np.array([f(int(v)) for v in c], dtype=np.float64)


def kappa(sm_scale: float) -> np.float32:
    """Softmax scale in base 2: fp32(sm_scale * log2(e)), sm_scale an fp32 value."""
    return np.float32(float(np.float32(sm_scale)) * math.log2(math.e))


def default_sm_scale(D: int) -> float:
    return float(np.float32(1.0 / math.sqrt(D)))


# --- steps --------------------------------------------------------------------

def k_mean(k: np.ndarray) -> tuple[np.ndarray, np.ndarray, int]:
    """k: [n, D] fp32 view of one head.  Returns (int64 sums, fp32 mean, status)."""
    k = _f32(k)
    n, D = k.shape
    s = np.zeros(D, dtype=np.int64)
    m = np.zeros(D, dtype=np.float32)
    st = lib().oracle_k_mean(_p(k), n, D, D, _p(s), _p(m))
    return s, m, st


def quant_block(x: np.ndarray, mean: Optional[np.ndarray] = None) -> tuple[np.ndarray, np.float32]:
    x = _f32(x)
    rows, D = x.shape
    codes = np.zeros((rows, D), dtype=np.int8)
    mean = None if mean is None else _f32(mean)
    d = lib().oracle_quant_block(_p(x), rows, D, D, _p(mean), _p(codes))
    return codes, np.float32(d)


def quant_head(x: np.ndarray, mean: Optional[np.ndarray] = None, blk: int = 128):
    """x: [n, D].  Returns codes [nblk*blk, D] (padding rows 0) and deltas [nblk]."""
    x = _f32(x)
    n, D = x.shape
    nblk = (n + blk - 1) // blk
    codes = np.zeros((nblk * blk, D), dtype=np.int8)
    delta = np.zeros(nblk, dtype=np.float32)
    mean = None if mean is None else _f32(mean)
    lib().oracle_quant_head(_p(x), n, D, D, _p(mean), blk, _p(codes), _p(delta))
    return codes, delta


def quant_v_fp8(v: np.ndarray):
    """v: [n, D].  Returns E4M3 codes [n, D] (uint8) and per-channel deltas [D]."""
    v = _f32(v)
    n, D = v.shape
    codes = np.zeros((n, D), dtype=np.uint8)
    delta = np.zeros(D, dtype=np.float32)
    lib().oracle_quant_v_fp8(_p(v), n, D, D, _p(codes), _p(delta))
    return codes, delta


def qk_int(qc: np.ndarray, kc: np.ndarray, i0: int, mi: int, j0: int, nj: int) -> np.ndarray:
    qc = np.ascontiguousarray(qc, dtype=np.int8)
    kc = np.ascontiguousarray(kc, dtype=np.int8)
    D = qc.shape[1]
    S = np.zeros((mi, nj), dtype=np.int32)
    lib().oracle_qk_int(_p(qc), _p(kc), D, i0, mi, j0, nj, _p(S))
    return S


def attn_ref_rows(q, k, v, sm_scale: float, causal: bool, rows) -> np.ndarray:
    """fp64 softmax(q k^T sm_scale) v for the listed rows of one head."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    n, D = q.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((len(rows), D), dtype=np.float64)
    lib().oracle_attn_ref_rows(_p(q), _p(k), _p(v), n, D, D, D, D, float(sm_scale), int(causal),
                               _p(rows), len(rows), _p(out))
    return out


def q_smooth_bias(qmean: np.ndarray, k: np.ndarray, kmean: np.ndarray, sm_scale: float,
                  ldo: Optional[int] = None, order: str = "fp64") -> np.ndarray:
    """Per-key term of Q smoothing for one head: [nb, ldo] fp32 with
    out[I, j] = kappa * qmean[I] . (k[j] - kmean) for j < n (0 beyond).
    order "fp64": the dot product in fp64, rounded once (the plain form);
    "fma": fp32 fused multiply-adds in channel order, then times kappa.
    qmean: [nb, D] block means of Q; k: [n, D]; kmean: [D]."""
    qmean, k, kmean = _f32(qmean), _f32(k), _f32(kmean)
    nb, D = qmean.shape
    n = k.shape[0]
    ldo = n if ldo is None else ldo
    out = np.zeros((nb, ldo), dtype=np.float32)
    fn = {"fp64": lib().oracle_q_smooth_bias, "fma": lib().oracle_q_smooth_bias_fma}[order]
    fn(_p(qmean), nb, _p(k), n, D, D, _p(kmean), float(kappa(sm_scale)), _p(out), ldo)
    return out


def attn_emul_rows(qc, qdelta, kc, kdelta, n: int, D: int, sm_scale: float, causal: bool,
                   pv_mode: str, rows, v=None, p16: str = "fp16", vc=None, vdelta=None,
                   blk: int = BLOCK, kv: int = BLOCK, tau: float = 0.0, p8_exp: bool = False,
                   per_token: bool = False, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """The quantised method's output rows (fp32) for one head; see sage_oracle.c.
    blk: quantisation block (tokens); per_token: qdelta / kdelta hold one delta
    per token (blk is then unused); bias: Q smoothing's per-key term
    [nb, >= n] (q_smooth_bias), per-block deltas only.
    The defaults are the plain method.  Other evaluation orders: kv (key tile
    of the online softmax and of the FP8 flush, a divisor of the block), tau
    (threshold on moving the maximum) and p8_exp (FP8 P scale applied in the
    exponent)."""
    if not per_token and blk % kv:
        raise ValueError("the key tile must divide the quantisation block")
    if bias is not None and per_token:
        raise ValueError("Q smoothing is defined with per-block deltas")
    qc = np.ascontiguousarray(qc, dtype=np.int8)
    kc = np.ascontiguousarray(kc, dtype=np.int8)
    qdelta, kdelta = _f32(qdelta), _f32(kdelta)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((len(rows), D), dtype=np.float32)
    if bias is not None:
        bias = _f32(bias)
    if pv_mode == "fp16":
        v = _f32(v)
        vc_p, vd_p, v_p, ldv, mode = None, None, _p(v), D, 0
    else:
        vc = np.ascontiguousarray(vc, dtype=np.uint8)
        vdelta = _f32(vdelta)
        vc_p, vd_p, v_p, ldv, mode = _p(vc), _p(vdelta), None, D, 1
    lib().oracle_attn_emul_rows(_p(qc), _p(qdelta), _p(kc), _p(kdelta), v_p, ldv, vc_p, vd_p, n,
                                D, blk, kv, float(kappa(sm_scale)),
                                float(tau), int(causal), mode,
                                1 if p16 == "bf16" else 0, _p(rows), len(rows), _p(out),
                                int(bool(per_token)), _p(bias),
                                0 if bias is None else bias.shape[1], int(bool(p8_exp)))
    return out

"""Workload-level driver of the CPU oracle -- TEST INFRASTRUCTURE.

Runs the per-head oracle steps over every (sequence, head) of a dense
[B,H,N,D] or packed varlen [T,H,D] input and lays the results out the way the
CUDA library's quantisation outputs are laid out, so tests can compare them
element by element:

  dense   q/k codes [B,H,NP,D] int8 (NP = ceil(N/128)*128, padding rows 0),
          q/k deltas [B,H,NB], k mean [B,H,D], v codes [B,H,N,D] e4m3,
          v deltas [B,H,D]
  varlen  q/k codes [H, sum_s ceil(n_s/128)*128, D], deltas [H, total blocks],
          k mean [n_seqs,H,D], v codes [T,H,D], v deltas [n_seqs,H,D]
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import (attn_emul_rows, attn_ref_rows, default_sm_scale, k_mean, q_smooth_bias, quant_block,
               quant_head, quant_v_fp8)

BLK = 128


@dataclasses.dataclass
class Quantized:
    q_codes: np.ndarray
    q_delta: np.ndarray
    k_codes: np.ndarray
    k_delta: np.ndarray
    k_sum: np.ndarray
    k_mean: np.ndarray
    v_codes: Optional[np.ndarray]
    v_delta: Optional[np.ndarray]
    status: int
    q_mean: Optional[np.ndarray] = None   # gran "block_sq": Q block means [B,H,NB,D]


def _heads(x: torch.Tensor, cu: Optional[list[int]]):
    """Yield (seq, head, [n, D] fp32 numpy view) over a dense or packed tensor."""
    if cu is None:
        B, H = x.shape[0], x.shape[1]
        xf = x.float().numpy()
        for b in range(B):
            for h in range(H):
                yield b, h, xf[b, h]
    else:
        H = x.shape[1]
        xf = x.float().numpy()
        for s in range(len(cu) - 1):
            for h in range(H):
                yield s, h, np.ascontiguousarray(xf[cu[s]:cu[s + 1], h])


def repeat_kv(x: torch.Tensor, groups: int) -> torch.Tensor:
    """Grouped-query attention's head mapping, written out: [B, Hkv, N, D] ->
    [B, Hkv*groups, N, D], query head h reading key/value head h // groups.

    Follows the attention code on the "sageattention in DeepSeek-VL2" page,
    which repeats every key/value head for `num_key_value_groups` consecutive
    query heads (repeat_kv) before calling attention.
    """
    B, Hkv, N, D = x.shape
    out = torch.empty((B, Hkv * groups, N, D), dtype=x.dtype)
    for h in range(Hkv * groups):
        out[:, h] = x[:, h // groups]
    return out


def repeat_kv_packed(x: torch.Tensor, groups: int) -> torch.Tensor:
    """repeat_kv for packed [T, Hkv, D] tensors: head h of the result is key/value
    head h // groups."""
    T, Hkv, D = x.shape
    out = torch.empty((T, Hkv * groups, D), dtype=x.dtype)
    for h in range(Hkv * groups):
        out[:, h] = x[:, h // groups]
    return out


def quantize(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor] = None,
             cu_seqlens: Optional[torch.Tensor] = None, pv_mode: str = "fp16",
             gran: str = "block") -> Quantized:
    """gran "block": one delta per 128-token block (deltas [B,H,NB] dense,
    [H, TB] varlen); "token": one delta per token, the quantiser applied to
    one-row blocks, stored like the code rows (deltas [B,H,NP] dense,
    [H, TB*128] varlen; padding rows 0); "block_sq": per-block deltas of Q
    smoothed by its block mean (SageAttention2's smoothing of Q), the means in
    q_mean ([B,H,NB,D] dense, [H,TB,D] varlen)."""
    cu = None if cu_seqlens is None else [int(c) for c in cu_seqlens.tolist()]
    status = 0
    tok = gran == "token"
    if gran == "block_sq" and cu is not None:
        # per sequence: Q blocks smoothed by their own means (q_mean [H, TB, D],
        # indexed like the deltas); K and V as for "block"
        qz = quantize(q, k, v, cu_seqlens, pv_mode, "block")
        T, H, D = q.shape
        S = len(cu) - 1
        nblk = [(cu[s + 1] - cu[s] + BLK - 1) // BLK for s in range(S)]
        boff = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
        TB = int(boff[-1])
        qc = np.zeros((H, TB * BLK, D), np.int8)
        qd = np.zeros((H, TB), np.float32)
        qm = np.zeros((H, TB, D), np.float32)
        for s, h, x in _heads(q, cu):
            for I in range(nblk[s]):
                xb = np.ascontiguousarray(x[I * BLK:(I + 1) * BLK])
                g = int(boff[s]) + I
                _, qm[h, g], st = k_mean(xb)
                status |= st
                qc[h, g * BLK:g * BLK + xb.shape[0]], qd[h, g] = quant_block(xb, qm[h, g])
        return Quantized(qc, qd, qz.k_codes, qz.k_delta, qz.k_sum, qz.k_mean, qz.v_codes,
                         qz.v_delta, status | qz.status, qm)
    if gran == "block_sq":
        qz = quantize(q, k, v, None, pv_mode, "block")  # K and V as for "block"
        B, H, N, D = q.shape
        NB = (N + BLK - 1) // BLK
        qc = np.zeros((B, H, NB * BLK, D), np.int8)
        qd = np.zeros((B, H, NB), np.float32)
        qm = np.zeros((B, H, NB, D), np.float32)
        for b, h, x in _heads(q, None):
            for I in range(NB):
                xb = np.ascontiguousarray(x[I * BLK:(I + 1) * BLK])
                _, qm[b, h, I], st = k_mean(xb)  # the exact row mean, over this block's rows
                status |= st
                qc[b, h, I * BLK:I * BLK + xb.shape[0]], qd[b, h, I] = quant_block(xb, qm[b, h, I])
        return Quantized(qc, qd, qz.k_codes, qz.k_delta, qz.k_sum, qz.k_mean, qz.v_codes,
                         qz.v_delta, status | qz.status, qm)
    if cu is None:
        B, H, N, D = q.shape
        NB = (N + BLK - 1) // BLK
        qc = np.zeros((B, H, NB * BLK, D), np.int8)
        qd = np.zeros((B, H, NB * BLK if tok else NB), np.float32)
        kc = np.zeros_like(qc); kd = np.zeros_like(qd)
        ks = np.zeros((B, H, D), np.int64); km = np.zeros((B, H, D), np.float32)
        for b, h, x in _heads(q, None):
            if tok:
                c, d = quant_head(x, None, 1)
                qc[b, h, :N], qd[b, h, :N] = c, d
            else:
                qc[b, h], qd[b, h] = quant_head(x, None, BLK)
        for b, h, x in _heads(k, None):
            ks[b, h], km[b, h], st = k_mean(x)
            status |= st
            if tok:
                c, d = quant_head(x, km[b, h], 1)
                kc[b, h, :N], kd[b, h, :N] = c, d
            else:
                kc[b, h], kd[b, h] = quant_head(x, km[b, h], BLK)
        vc = vd = None
        if pv_mode == "fp8":
            vc = np.zeros((B, H, N, D), np.uint8); vd = np.zeros((B, H, D), np.float32)
            for b, h, x in _heads(v, None):
                vc[b, h], vd[b, h] = quant_v_fp8(x)
        return Quantized(qc, qd, kc, kd, ks, km, vc, vd, status)
    T, H, D = q.shape
    S = len(cu) - 1
    nblk = [(cu[s + 1] - cu[s] + BLK - 1) // BLK for s in range(S)]
    boff = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
    TB = int(boff[-1])
    qc = np.zeros((H, TB * BLK, D), np.int8)
    qd = np.zeros((H, TB * BLK if tok else TB), np.float32)
    kc = np.zeros_like(qc); kd = np.zeros_like(qd)
    ks = np.zeros((S, H, D), np.int64); km = np.zeros((S, H, D), np.float32)
    for s, h, x in _heads(q, cu):
        r0 = boff[s] * BLK
        if tok:
            c, d = quant_head(x, None, 1)
            qc[h, r0:r0 + c.shape[0]] = c; qd[h, r0:r0 + d.shape[0]] = d
        else:
            c, d = quant_head(x, None, BLK)
            qc[h, r0:r0 + c.shape[0]] = c; qd[h, boff[s]:boff[s + 1]] = d
    for s, h, x in _heads(k, cu):
        ks[s, h], km[s, h], st = k_mean(x)
        status |= st
        r0 = boff[s] * BLK
        if tok:
            c, d = quant_head(x, km[s, h], 1)
            kc[h, r0:r0 + c.shape[0]] = c; kd[h, r0:r0 + d.shape[0]] = d
        else:
            c, d = quant_head(x, km[s, h], BLK)
            kc[h, r0:r0 + c.shape[0]] = c; kd[h, boff[s]:boff[s + 1]] = d
    vc = vd = None
    if pv_mode == "fp8":
        vc = np.zeros((T, H, D), np.uint8); vd = np.zeros((S, H, D), np.float32)
        for s, h, x in _heads(v, cu):
            vc[cu[s]:cu[s + 1], h], vd[s, h] = quant_v_fp8(x)
    return Quantized(qc, qd, kc, kd, ks, km, vc, vd, status)


def _head_view(qz: Quantized, cu, s: int, h: int, tok: bool = False):
    """Per-head slices of the quantised tensors for sequence s, head h (tok:
    deltas stored per code row)."""
    if cu is None:
        qc, qd, kc, kd = qz.q_codes[s, h], qz.q_delta[s, h], qz.k_codes[s, h], qz.k_delta[s, h]
        vc = None if qz.v_codes is None else qz.v_codes[s, h]
        vd = None if qz.v_delta is None else qz.v_delta[s, h]
        return qc, qd, kc, kd, vc, vd
    nblk = [(cu[i + 1] - cu[i] + BLK - 1) // BLK for i in range(len(cu) - 1)]
    b0 = sum(nblk[:s]); b1 = b0 + nblk[s]
    qc = qz.q_codes[h, b0 * BLK:b1 * BLK]; kc = qz.k_codes[h, b0 * BLK:b1 * BLK]
    if tok:
        qd = qz.q_delta[h, b0 * BLK:b1 * BLK]; kd = qz.k_delta[h, b0 * BLK:b1 * BLK]
    else:
        qd = qz.q_delta[h, b0:b1]; kd = qz.k_delta[h, b0:b1]
    vc = None if qz.v_codes is None else np.ascontiguousarray(qz.v_codes[cu[s]:cu[s + 1], h])
    vd = None if qz.v_delta is None else qz.v_delta[s, h]
    return qc, qd, kc, kd, vc, vd


def _group(picks):
    groups: dict[tuple[int, int], list[int]] = {}
    for s, h, i in picks:
        groups.setdefault((s, h), []).append(i)
    return groups


def emulate_rows(qz: Quantized, v: torch.Tensor, cu_seqlens, picks, D: int, causal: bool,
                 pv_mode: str, sm_scale: Optional[float] = None,
                 seqlens: Optional[list[int]] = None, gran: str = "block",
                 k: Optional[torch.Tensor] = None, kv: int = BLK, tau: float = 0.0,
                 p8_exp: bool = False, bias_order: str = "fp64") -> dict:
    """E for the listed (seq, head, row) picks -> {pick: fp32 [D]}.  gran
    "block_sq" needs k (one head per query head; dense [B,H,N,D] or packed
    [T,H,D]) for the per-key term of Q smoothing.  The defaults give the plain
    method; kv, tau, p8_exp and bias_order select another evaluation order
    (see attn_emul_rows and q_smooth_bias)."""
    cu = None if cu_seqlens is None else [int(c) for c in cu_seqlens.tolist()]
    sm_scale = default_sm_scale(D) if sm_scale is None else sm_scale
    p16 = "bf16" if v.dtype == torch.bfloat16 else "fp16"
    out = {}
    vf = v.float().numpy() if pv_mode == "fp16" else None
    for (s, h), rows in _group(picks).items():
        n = (cu[s + 1] - cu[s]) if cu is not None else (seqlens[s] if seqlens else v.shape[2])
        qc, qd, kc, kd, vc, vd = _head_view(qz, cu, s, h, gran == "token")
        vv = None
        if pv_mode == "fp16":
            vv = vf[s, h] if cu is None else np.ascontiguousarray(vf[cu[s]:cu[s + 1], h])
        bias = None
        if gran == "block_sq" and cu is None:
            bias = q_smooth_bias(qz.q_mean[s, h], k[s, h].float().numpy(), qz.k_mean[s, h],
                                 sm_scale, order=bias_order)
        elif gran == "block_sq":
            b0 = sum((cu[i + 1] - cu[i] + BLK - 1) // BLK for i in range(s))
            nb = (n + BLK - 1) // BLK
            bias = q_smooth_bias(qz.q_mean[h, b0:b0 + nb],
                                 k[cu[s]:cu[s + 1], h].float().numpy(), qz.k_mean[s, h],
                                 sm_scale, order=bias_order)
        o = attn_emul_rows(qc, qd, kc, kd, n, D, sm_scale, causal, pv_mode, rows, v=vv, p16=p16,
                           vc=vc, vdelta=vd, per_token=gran == "token", bias=bias, kv=kv,
                           tau=tau, p8_exp=p8_exp)
        for r, i in enumerate(rows):
            out[(s, h, i)] = o[r]
    return out


def reference_rows(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens, picks,
                   causal: bool, sm_scale: Optional[float] = None) -> dict:
    """R (fp64) for the listed (seq, head, row) picks -> {pick: fp64 [D]}."""
    cu = None if cu_seqlens is None else [int(c) for c in cu_seqlens.tolist()]
    D = q.shape[-1]
    sm_scale = default_sm_scale(D) if sm_scale is None else sm_scale
    qf, kf, vf = q.float().numpy(), k.float().numpy(), v.float().numpy()
    out = {}
    for (s, h), rows in _group(picks).items():
        if cu is None:
            qq, kk, vv = qf[s, h], kf[s, h], vf[s, h]
        else:
            sl = slice(cu[s], cu[s + 1])
            qq, kk, vv = (np.ascontiguousarray(x[sl, h]) for x in (qf, kf, vf))
        o = attn_ref_rows(qq, kk, vv, sm_scale, causal, rows)
        for r, i in enumerate(rows):
            out[(s, h, i)] = o[r]
    return out

"""Seeded synthetic attention inputs.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no quantisation, no softmax, no mean).  The same host
tensors feed both the CUDA library and the CPU oracle, so the two sides never
see different data.

Workload shapes follow the attention workloads the SageAttention pages talk
about: video-DiT self-attention (long, non-causal, head dim 64) and LLM
attention (causal, head dim 128, variable-length packed batches).  There is no
dataset and there are no weights; every tensor is drawn from a seeded
``torch.Generator`` on the CPU in fp32 and then rounded to the 16-bit input
dtype.

Recipe (per workload):
  * Q, V ~ N(0, 1);  K ~ N(0, 1) + b, with one bias b[d] ~ N(0, sigma_b^2) per
    (sequence, head, channel) shared by every token of that sequence -- the
    channel offset that K smoothing removes.
  * optional outliers: an independent Bernoulli(p) draw per Q and per K entry
    picks entries that are multiplied by a factor (after the bias is added).
  * optional Q channel offset (the offset Q smoothing removes): q[d] += c[d],
    c[d] ~ N(0, sigma_q^2) per (sequence, head, channel), drawn last so the
    other draws do not depend on it.
  * varlen: sequence lengths are drawn uniformly (inclusive) from a range, and
    ``cu_seqlens`` is their prefix sum; the packed layout is [T, H, D].
  * grouped-query attention (Hkv < H): Q, K, V are drawn for H heads as above
    and K, V keep their first Hkv heads ([B, Hkv, N, D]).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int                      # dense sequence length (max length for varlen)
    D: int
    dtype: str                  # "fp16" | "bf16"
    causal: bool
    pv_mode: str                # "fp16" | "fp8"
    bias_sigma: float
    outlier_p: float = 0.0
    outlier_scale: float = 1.0
    varlen: bool = False
    n_seqs: int = 0
    len_lo: int = 0
    len_hi: int = 0
    seed: int = 0
    Hkv: int = 0                # key/value heads (grouped-query attention); 0: = H
    qk_gran: str = "block"      # Q/K deltas per 128-token block, per token, or per block
                                # with Q smoothing ("block_sq")
    q_bias_sigma: float = 0.0   # Q channel offset (see the recipe)

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five workloads: a small one the oracle finishes in seconds, a causal LLM
# block, a video-DiT shape with outliers and FP8 P.V, the long-sequence
# throughput point, and a packed variable-length causal batch.
WORKLOADS = {
    "small_d64": Workload("small_d64", B=1, H=2, N=256, D=64, dtype="fp16", causal=False,
                          pv_mode="fp16", bias_sigma=2.0, seed=20260001),
    "llm_causal_2k": Workload("llm_causal_2k", B=2, H=16, N=2048, D=128, dtype="bf16",
                              causal=True, pv_mode="fp16", bias_sigma=3.0, seed=20260002),
    "dit_8k_fp8": Workload("dit_8k_fp8", B=1, H=24, N=8192, D=64, dtype="fp16", causal=False,
                           pv_mode="fp8", bias_sigma=3.0, outlier_p=0.01, outlier_scale=20.0,
                           seed=20260003),
    "long_32k": Workload("long_32k", B=1, H=32, N=32768, D=128, dtype="fp16", causal=False,
                         pv_mode="fp16", bias_sigma=3.0, seed=20260004),
    "varlen_8seq": Workload("varlen_8seq", B=1, H=32, N=8192, D=128, dtype="bf16", causal=True,
                            pv_mode="fp8", bias_sigma=3.0, varlen=True, n_seqs=8, len_lo=512,
                            len_hi=8192, seed=20260005),
    # LLM prefill with grouped-query attention (32 query heads over 8 key/value
    # heads, the repeat_kv layout of the DeepSeek-VL2 page's attention code)
    "llm_gqa_8k": Workload("llm_gqa_8k", B=1, H=32, N=8192, D=128, dtype="bf16", causal=True,
                           pv_mode="fp16", bias_sigma=3.0, seed=20260006, Hkv=8),
    # the video-DiT shape with one Q/K delta per token (the accurate option for
    # channel outliers)
    "dit_8k_fp8_tok": Workload("dit_8k_fp8_tok", B=1, H=24, N=8192, D=64, dtype="fp16",
                               causal=False, pv_mode="fp8", bias_sigma=3.0, outlier_p=0.01,
                               outlier_scale=20.0, seed=20260003, qk_gran="token"),
    # the video-DiT shape with Q smoothing (SageAttention2), on a Q that carries
    # a channel offset like K
    "dit_8k_fp8_sq": Workload("dit_8k_fp8_sq", B=1, H=24, N=8192, D=64, dtype="fp16",
                              causal=False, pv_mode="fp8", bias_sigma=3.0, outlier_p=0.01,
                              outlier_scale=20.0, seed=20260003, qk_gran="block_sq",
                              q_bias_sigma=3.0),
}


@dataclasses.dataclass
class Inputs:
    """Host (CPU) tensors of one workload instance."""
    q: torch.Tensor                    # [B,H,N,D] dense or [T,H,D] varlen, 16-bit
    k: torch.Tensor
    v: torch.Tensor
    cu_seqlens: Optional[torch.Tensor]  # int32 [n_seqs+1] (varlen only)
    wl: Workload

    @property
    def seqlens(self) -> list[int]:
        if self.cu_seqlens is None:
            return [self.wl.N] * self.wl.B
        c = self.cu_seqlens.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]


def _outliers(x: torch.Tensor, g: torch.Generator, p: float, scale: float) -> torch.Tensor:
    if p <= 0.0:
        return x
    mask = torch.rand(x.shape, generator=g) < p
    return torch.where(mask, x * scale, x)


def make_dense(B: int, H: int, N: int, D: int, dtype: str = "fp16", bias_sigma: float = 3.0,
               outlier_p: float = 0.0, outlier_scale: float = 1.0, seed: int = 0,
               k_const_over_tokens: bool = False,
               q_bias_sigma: float = 0.0) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Dense [B,H,N,D] q, k, v drawn by the recipe in the module docstring."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H, N, D), generator=g)
    k = torch.randn((B, H, N, D), generator=g)
    v = torch.randn((B, H, N, D), generator=g)
    bias = torch.randn((B, H, 1, D), generator=g) * bias_sigma
    if k_const_over_tokens:
        k = torch.zeros_like(k)
    k = k + bias
    q = _outliers(q, g, outlier_p, outlier_scale)
    k = _outliers(k, g, outlier_p, outlier_scale)
    if q_bias_sigma > 0.0:
        q = q + torch.randn((B, H, 1, D), generator=g) * q_bias_sigma
    t = DTYPES[dtype]
    return q.to(t), k.to(t), v.to(t)


def make_varlen(seqlens: list[int], H: int, D: int, dtype: str = "bf16", bias_sigma: float = 3.0,
                seed: int = 0, q_bias_sigma: float = 0.0
                ) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """Packed [T,H,D] q, k, v plus int32 cu_seqlens for the given lengths."""
    g = torch.Generator().manual_seed(seed)
    T = int(sum(seqlens))
    q = torch.randn((T, H, D), generator=g)
    k = torch.randn((T, H, D), generator=g)
    v = torch.randn((T, H, D), generator=g)
    cu = [0]
    for n in seqlens:
        cu.append(cu[-1] + int(n))
    for s, n in enumerate(seqlens):
        b = torch.randn((1, H, D), generator=g) * bias_sigma
        k[cu[s]:cu[s + 1]] += b
    if q_bias_sigma > 0.0:  # drawn last: the other draws do not depend on it
        for s, n in enumerate(seqlens):
            q[cu[s]:cu[s + 1]] += torch.randn((1, H, D), generator=g) * q_bias_sigma
    t = DTYPES[dtype]
    return q.to(t), k.to(t), v.to(t), torch.tensor(cu, dtype=torch.int32)


def draw_seqlens(n_seqs: int, lo: int, hi: int, seed: int) -> list[int]:
    g = torch.Generator().manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n_seqs,), generator=g)]


def make_inputs(wl: Workload) -> Inputs:
    if wl.varlen:
        lens = draw_seqlens(wl.n_seqs, wl.len_lo, wl.len_hi, wl.seed)
        q, k, v, cu = make_varlen(lens, wl.H, wl.D, wl.dtype, wl.bias_sigma, seed=wl.seed + 1)
        return Inputs(q, k, v, cu, wl)
    q, k, v = make_dense(wl.B, wl.H, wl.N, wl.D, wl.dtype, wl.bias_sigma, wl.outlier_p,
                         wl.outlier_scale, seed=wl.seed, q_bias_sigma=wl.q_bias_sigma)
    if wl.kv_heads != wl.H:
        k, v = k[:, :wl.kv_heads].contiguous(), v[:, :wl.kv_heads].contiguous()
    return Inputs(q, k, v, None, wl)


def attention_ops(wl: Workload, seqlens: Optional[list[int]] = None) -> float:
    """Operation count of the metric: 4*H*n^2*D per sequence (halved when causal)."""
    if seqlens is None:
        seqlens = [wl.N] * wl.B
    f = 0.5 if wl.causal else 1.0
    return float(sum(4.0 * wl.H * n * n * wl.D * f for n in seqlens))


def sample_rows(seqlens: list[int], H: int, n_rows: int, seed: int) -> list[tuple[int, int, int]]:
    """Seeded sample of (sequence, head, row) triples; always includes every
    sequence's first and last row (on head 0 and on the last head)."""
    g = torch.Generator().manual_seed(seed)
    picks = set()
    for s, n in enumerate(seqlens):
        for h in (0, H - 1):
            picks.add((s, h, 0))
            picks.add((s, h, n - 1))
    total = sum(seqlens) * H
    while len(picks) < min(n_rows, total):
        u = int(torch.randint(0, total, (1,), generator=g))
        h, rem = divmod(u, sum(seqlens))
        for s, n in enumerate(seqlens):
            if rem < n:
                picks.add((s, h, rem))
                break
            rem -= n
    return sorted(picks)

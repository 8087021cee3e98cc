"""SageAttention 8-bit attention forward pass for NVIDIA B200 (sm_100a).

K smoothing, per-block INT8 Q/K quantisation, INT8 QK^T on tcgen05 tensor
cores with TMEM accumulators, online softmax, and P.V in 16 bits or in FP8
with two-level FP32 accumulation -- as hand-written CUDA kernels behind the C
ABI declared in include/sage.h (libsageb200.so).  This package is the Python
binding of that library.
"""
from .api import (  # noqa: F401
    BLOCK, PV_COSINE_THRESHOLD, PV_MODES, Quantized, SageError, Workspace, alloc_quantized,
    attn_fwd, attn_fwd_host, attn_fwd_varlen, attn_fwd_varlen_host, attn_quantized, attn_ref_rows, calibrate_pv_modes,
    attn_quantized_dump_s, choose_pv_mode, cosine_similarity, pv_mode_similarity, qk_int8_tiles,
    quant_qk, quantize,
    quantize_varlen, sageattn, sageattn_qk_int8_pv_fp16_cuda, sageattn_qk_int8_pv_fp8_cuda,
    sageattn_varlen, sync_status, workspace_bytes, workspace_bytes_gqa, workspace_bytes_varlen,
)

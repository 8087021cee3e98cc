"""ctypes loader of libsageb200.so (the CUDA library built in-tree).

There is no fallback: if the library is missing or was built for nothing this
machine can run, importing the binding raises.  Build it with
``python -m quantized_attention_07_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsageb200.so")

# Every symbol declared in include/sage.h, with its argument and return types.
_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "sage_workspace_bytes": ([_I, _I, _I, _I, _I], _SZ),
    "sage_workspace_bytes_varlen": ([_I, _I, _I, _I, _I], _SZ),
    "sage_scratch_bytes": ([_I, _I, _I], _SZ),
    "sage_workspace_init": ([_P, _SZ, _P], _I),
    "sage_sync_status": ([_P, _P], _I),
    "sage_status_string": ([_I], ctypes.c_char_p),
    "sage_last_cuda_error": ([], ctypes.c_char_p),
    "sage_attn_fwd": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P], _I),
    "sage_workspace_bytes_gqa": ([_I, _I, _I, _I, _I, _I], _SZ),
    "sage_workspace_bytes_varlen_gqa": ([_I, _I, _I, _I, _I, _I], _SZ),
    "sage_workspace_bytes_varlen_sq": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sage_workspace_bytes_sq": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sage_workspace_bytes_varlen_ex": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sage_attn_fwd_varlen_ex": ([_P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                 _I, _P, _SZ, _P], _I),
    "sage_attn_fwd_varlen_gqa": ([_P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                                  _P, _SZ, _P], _I),
    "sage_workspace_bytes_ex": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sage_attn_fwd_ex": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _SZ,
                          _P], _I),
    "sage_quantize_ex": ([_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                          _P, _SZ, _P], _I),
    "sage_quantize_sq": ([_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _P,
                          _P, _P, _P, _P, _SZ, _P], _I),
    "sage_attn_quantized_sq": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                _I, _F, _I, _P, _SZ, _P], _I),
    "sage_attn_quantized_ex": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                _F, _I, _I, _P, _SZ, _P], _I),
    "sage_attn_ref_rows": ([_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _I, _P, _P], _I),
    "sage_attn_fwd_gqa": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P], _I),
    "sage_attn_fwd_varlen": ([_P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P,
                              _SZ, _P], _I),
    "sage_quantize": ([_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                       _P], _I),
    "sage_attn_quantized": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                             _P, _SZ, _P], _I),
    "sage_quantize_varlen": ([_P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                              _P, _P, _SZ, _P], _I),
    "sage_qk_int8_tiles": ([_P, _P, _I, _I, _I, _P, _I, _P, _P, _SZ, _P], _I),
    "sage_quant_qk": ([_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "sage_attn_quantized_dump_s": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                    _F, _I, _P, _P, _SZ, _P], _I),
    "sage_selftest_wait_timeout": ([ctypes.c_longlong, _P, _SZ, _P], _I),
    "sage_selftest_attn_timeout": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                    _F, _I, ctypes.c_longlong, _I, _P, _SZ, _P], _I),
    "sage_quantize_noalloc": ([_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                               _P, _P], _I),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the library (once) and attach the C signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is not built; run `python -m quantized_attention_07_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib

"""ctypes view of libsage.so (the C ABI declared in include/sage.h and include/sage_nvfp4.h).

Loading fails loudly when the shared library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage.so")

SAGE_OK = 0
SAGE_ERR_INVALID_ARG = -1
SAGE_ERR_UNSUPPORTED = -2
SAGE_ERR_ALIGNMENT = -3
SAGE_ERR_WORKSPACE = -4
SAGE_ERR_CUDA = -5
SAGE_ERR_TIMEOUT = -6
SAGE_FP16 = 0
SAGE_BF16 = 1


class SageParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("d", ctypes.c_int), ("dtype", ctypes.c_int), ("causal", ctypes.c_int),
                ("qknorm", ctypes.c_int), ("ksmooth", ctypes.c_int),
                ("q_block", ctypes.c_int), ("k_block", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("qsmooth", ctypes.c_int)]


class SageQBufs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q_codes", "k_codes", "v_codes", "q_scale", "k_scale", "v_scale",
                 "q_inv_rms", "k_inv_rms", "k_mean", "q_mean", "k_bias")]


class SageFp4Bufs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q_fp4", "k_fp4", "q_sf", "k_sf", "q_genc", "k_genc", "q_inv_rms",
                 "k_inv_rms", "k_mean", "q_fp4_t", "k_fp4_t", "q_sf_t", "k_sf_t")]


class SageError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: {text} ({status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsage.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libsage.so not found at {LIB_PATH}; run "
                              "`python -c 'import __graft_entry__ as g; g.build()'` first")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.sage_workspace_bytes.argtypes = [P(SageParams), i]
        L.sage_workspace_bytes.restype = sz
        L.sage_quant_prologue.argtypes = [P(SageParams), vp, vp, vp, P(SageQBufs), vp, sz, vp]
        L.sage_quant_prologue.restype = i
        L.sage_quant_prologue_noalloc.argtypes = [P(SageParams), vp, vp, vp, P(SageQBufs), vp]
        L.sage_quant_prologue_noalloc.restype = i
        L.sage_attn_fwd.argtypes = [P(SageParams), P(SageQBufs), vp, vp, vp, sz, vp]
        L.sage_attn_fwd.restype = i
        L.sage_attn_bwd.argtypes = [P(SageParams), vp, vp, vp, P(SageQBufs), vp, vp, vp, vp,
                                    vp, vp, vp, sz, vp]
        L.sage_attn_bwd.restype = i
        L.sage_attn_bwd_stage.argtypes = [i, P(SageParams), vp, vp, vp, P(SageQBufs), vp, vp,
                                          vp, vp, vp, vp, vp, sz, vp]
        L.sage_attn_bwd_stage.restype = i
        L.sage_fp4_workspace_bytes.argtypes = [P(SageParams), i]
        L.sage_fp4_workspace_bytes.restype = sz
        L.sage_fp4_quant_prologue.argtypes = [P(SageParams), vp, vp, P(SageFp4Bufs), vp, sz, vp]
        L.sage_fp4_quant_prologue.restype = i
        L.sage_fp4_attn_fwd.argtypes = [P(SageParams), P(SageFp4Bufs), vp, vp, vp, vp]
        L.sage_fp4_attn_fwd.restype = i
        L.sage_fp4_attn_bwd.argtypes = [P(SageParams), vp, vp, vp, P(SageFp4Bufs), vp, vp, vp,
                                        vp, vp, vp, vp, sz, vp]
        L.sage_fp4_attn_bwd.restype = i
        L.sage_fp4_attn_bwd_stage.argtypes = [i, P(SageParams), vp, vp, vp, P(SageFp4Bufs), vp,
                                              vp, vp, vp, vp, vp, vp, sz, vp]
        L.sage_fp4_attn_bwd_stage.restype = i
        L.sage_fwd_bwd_host_workspace_bytes.argtypes = [P(SageParams), i]
        L.sage_fwd_bwd_host_workspace_bytes.restype = sz
        L.sage_fwd_bwd_host.argtypes = [P(SageParams), vp, vp, vp, vp, vp, vp, vp, vp, i, vp, sz,
                                        vp, vp, vp]
        L.sage_fwd_bwd_host.restype = i
        L.sage_quant_prologue_part.argtypes = [P(SageParams), vp, vp, vp, P(SageQBufs), vp, sz, i,
                                               vp]
        L.sage_quant_prologue_part.restype = i
        L.sage_attn_fwd_partial.argtypes = [P(SageParams), P(SageQBufs), vp, vp, vp]
        L.sage_attn_fwd_partial.restype = i
        L.sage_attn_merge.argtypes = [P(SageParams), vp, vp, vp, vp, vp, vp]
        L.sage_attn_merge.restype = i
        L.sage_attn_bwd_partial.argtypes = [P(SageParams), vp, P(SageQBufs), vp, vp, vp, vp, i,
                                            vp, sz, vp]
        L.sage_attn_bwd_partial.restype = i
        L.sage_kv_finalize.argtypes = [P(SageParams), vp, P(SageQBufs), vp, vp, vp, vp, vp]
        L.sage_kv_finalize.restype = i
        L.sage_last_device_status.argtypes = [vp]
        L.sage_last_device_status.restype = i
        L.sage_status_string.argtypes = [i]
        L.sage_status_string.restype = ctypes.c_char_p
        L.sage_debug_qk_int32.argtypes = [P(SageParams), P(SageQBufs), i, i, vp, vp]
        L.sage_debug_qk_int32.restype = i
        L.sage_debug_umma_gemm.argtypes = [i, i, i, i, i, vp, vp, vp, vp]
        L.sage_debug_umma_gemm.restype = i
        L.sage_debug_wait_timeout.argtypes = [i, vp]
        L.sage_debug_wait_timeout.restype = i
        L.sage_mma_peak.argtypes = [i, i, i, vp, sz, vp]
        L.sage_mma_peak.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sage_status_string(status).decode()


def check(fn: str, status: int) -> None:
    if status != SAGE_OK:
        raise SageError(fn, status, status_string(status))

"""SageBwd quantized attention training on NVIDIA B200 (sm_100a).

The computation lives in hand-written CUDA kernels behind the C ABI of ``libsage.so``
(``include/sage.h``); this package is the thin PyTorch binding around it.
"""
from .ops import (Config, QuantBufs, attn_bwd, attn_fwd, device_status, quant_prologue,  # noqa
                  sage_attention)

__all__ = ["Config", "QuantBufs", "attn_bwd", "attn_fwd", "device_status", "quant_prologue",
           "sage_attention"]

"""SageBwd quantized attention training on NVIDIA B200 (sm_100a).

The computation lives in hand-written CUDA kernels behind the C ABI of ``libsage.so``
(``include/sage.h``, and ``include/sage_nvfp4.h`` for the NVFP4 Q-Attn variant, bound in
``fwd_bwd_b200.nvfp4``); this package is the thin PyTorch binding around it.
"""
from .ops import (Config, QuantBufs, attn_bwd, attn_fwd, device_status, quant_prologue,  # noqa
                  sage_attention)

__all__ = ["Config", "QuantBufs", "attn_bwd", "attn_fwd", "device_status", "quant_prologue",
           "sage_attention"]

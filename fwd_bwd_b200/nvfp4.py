"""Python binding of the NVFP4 Q-Attn variant (include/sage_nvfp4.h): argument marshalling only.

Every step runs in libsage's CUDA kernels; there is no other path.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from ._lib import SageFp4Bufs, check, lib
from .ops import Config, _check_inputs, _stream


@dataclasses.dataclass
class Fp4Bufs:
    """NVFP4 views of Q and K (codes, E4M3 block scales, global scales), made once, reused."""

    q_fp4: torch.Tensor
    k_fp4: torch.Tensor
    q_sf: torch.Tensor
    k_sf: torch.Tensor
    q_genc: torch.Tensor
    k_genc: torch.Tensor
    q_inv_rms: Optional[torch.Tensor]
    k_inv_rms: Optional[torch.Tensor]
    k_mean: Optional[torch.Tensor]
    # sequence views (16-token blocks per channel), made only when requested
    q_fp4_t: Optional[torch.Tensor] = None
    k_fp4_t: Optional[torch.Tensor] = None
    q_sf_t: Optional[torch.Tensor] = None
    k_sf_t: Optional[torch.Tensor] = None

    @staticmethod
    def empty(shape, cfg: Config, device, seq: bool = False) -> "Fp4Bufs":
        B, H, N, d = shape
        u8 = dict(dtype=torch.uint8, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        sf = (B, H, N // 128, d // 64, 512)
        sf_t = (B, H, (d + 127) // 128, N // 64, 512)
        opt = (lambda s_: torch.empty(s_, **u8)) if seq else (lambda s_: None)
        return Fp4Bufs(torch.empty((B, H, N, d // 2), **u8), torch.empty((B, H, N, d // 2), **u8),
                       torch.empty(sf, **u8), torch.empty(sf, **u8),
                       torch.empty((B, H), **f32), torch.empty((B, H), **f32),
                       torch.empty((B, H, N), **f32) if cfg.qknorm else None,
                       torch.empty((B, H, N), **f32) if cfg.qknorm else None,
                       torch.empty((B, H, d), **f32) if cfg.ksmooth else None,
                       opt((B, H, d, N // 2)), opt((B, H, d, N // 2)), opt(sf_t), opt(sf_t))

    def c_struct(self) -> SageFp4Bufs:
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        return SageFp4Bufs(p(self.q_fp4), p(self.k_fp4), p(self.q_sf), p(self.k_sf),
                           p(self.q_genc), p(self.k_genc), p(self.q_inv_rms), p(self.k_inv_rms),
                           p(self.k_mean), p(self.q_fp4_t), p(self.k_fp4_t), p(self.q_sf_t),
                           p(self.k_sf_t))


def workspace_bytes(cfg: Config, like: torch.Tensor) -> int:
    return int(lib().sage_fp4_workspace_bytes(ctypes.byref(cfg.params(like)), 0))


def quant_prologue(q, k, cfg: Config, out: Optional[Fp4Bufs] = None,
                   workspace: Optional[torch.Tensor] = None, seq: bool = False) -> Fp4Bufs:
    """QK-norm, K-smoothing and NVFP4 quantization of q and k (sage_fp4_quant_prologue);
    ``seq`` also makes the sequence views (when ``out`` is None)."""
    _check_inputs(q, k)
    prm = cfg.params(q)
    fb = out if out is not None else Fp4Bufs.empty(tuple(q.shape), cfg, q.device, seq=seq)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(cfg, q), dtype=torch.uint8, device=q.device)
    st = fb.c_struct()
    check("sage_fp4_quant_prologue", lib().sage_fp4_quant_prologue(
        ctypes.byref(prm), q.data_ptr(), k.data_ptr(), ctypes.byref(st), workspace.data_ptr(),
        workspace.numel(), _stream(q.device)))
    return fb


def attn_fwd(fb: Fp4Bufs, v: torch.Tensor, cfg: Config, o=None, lse=None):
    """NVFP4 Q K^T, 16-bit P V forward (sage_fp4_attn_fwd): returns (o, lse)."""
    _check_inputs(v)
    prm = cfg.params(v)
    B, H, N, d = v.shape
    if o is None:
        o = torch.empty_like(v)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=v.device)
    st = fb.c_struct()
    check("sage_fp4_attn_fwd", lib().sage_fp4_attn_fwd(
        ctypes.byref(prm), ctypes.byref(st), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
        _stream(v.device)))
    return o, lse


def bwd_workspace_bytes(cfg: Config, like: torch.Tensor) -> int:
    return int(lib().sage_fp4_workspace_bytes(ctypes.byref(cfg.params(like)), 2))


def attn_bwd(q, k, v, fb: Fp4Bufs, o, lse, do, cfg: Config, dq=None, dk=None, dv=None,
             workspace: Optional[torch.Tensor] = None, stage: Optional[int] = None):
    """Backward with dS in NVFP4, P^T dO and dO V^T in 16 bits (sage_fp4_attn_bwd): returns
    (dq, dk, dv).  ``fb`` must hold the sequence views (``quant_prologue(..., seq=True)``).
    ``stage`` in {0, 1, 2} runs only that stage (sage_fp4_attn_bwd_stage); the caller then owns
    ``workspace`` across the three calls."""
    _check_inputs(q, k, v, o, do)
    prm = cfg.params(q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(cfg, q), dtype=torch.uint8, device=q.device)
    st = fb.c_struct()
    args = (ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
            o.data_ptr(), lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
            dv.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(q.device))
    if stage is None:
        check("sage_fp4_attn_bwd", lib().sage_fp4_attn_bwd(*args))
    else:
        check("sage_fp4_attn_bwd_stage", lib().sage_fp4_attn_bwd_stage(stage, *args))
    return dq, dk, dv


class _QAttn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cfg: Config):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        fb = quant_prologue(q, k, cfg, seq=True)
        o, lse = attn_fwd(fb, v, cfg)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.fb, ctx.cfg = fb, cfg
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attn_bwd(q, k, v, ctx.fb, o, lse, do.contiguous(), ctx.cfg)
        return dq, dk, dv, None


def qattn_attention(q, k, v, causal: bool = True, qknorm: bool = True, ksmooth: bool = True,
                    softmax_scale: float = 0.0, rms_eps: float = 1e-6):
    """NVFP4 Q-Attn attention with autograd (Q K^T and dS in NVFP4, P V, P^T dO and dO V^T in
    16 bits): q, k, v are CUDA [B, H, N, d] fp16 / bf16 tensors.  The forward keeps the NVFP4
    views (with the sequence views the backward multiplies) for the backward."""
    cfg = Config(causal, qknorm, ksmooth, 128, 64, softmax_scale, rms_eps, False)
    return _QAttn.apply(q, k, v, cfg)

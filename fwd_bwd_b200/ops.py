"""PyTorch-facing binding of libsage: argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI; PyTorch provides the
device memory (tensors) and the stream.  Names follow the C ABI: ``quant_prologue``,
``attn_fwd``, ``attn_bwd``; ``sage_attention`` wraps the three in an autograd function.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
from typing import Optional, Tuple

import torch

from . import _lib
from ._lib import SageParams, SageQBufs, check, lib

_DTYPES = {torch.float16: _lib.SAGE_FP16, torch.bfloat16: _lib.SAGE_BF16}


@dataclasses.dataclass
class Config:
    """Problem flags shared by the three calls (see include/sage.h, ``sage_params``)."""

    causal: bool = True
    qknorm: bool = True
    ksmooth: bool = True
    q_block: int = 128
    k_block: int = 64
    softmax_scale: float = 0.0  # <= 0: 1/sqrt(d)
    rms_eps: float = 1e-6
    qsmooth: bool = False

    def params(self, x: torch.Tensor) -> SageParams:
        B, H, N, d = x.shape
        return SageParams(B, H, N, d, _DTYPES[x.dtype], int(self.causal), int(self.qknorm),
                          int(self.ksmooth), self.q_block, self.k_block,
                          float(self.softmax_scale), float(self.rms_eps), int(self.qsmooth))


@dataclasses.dataclass
class QuantBufs:
    """Quantized views of Q, K, V (INT8 codes + per-block scales), reused by fwd and bwd."""

    q_codes: torch.Tensor
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    q_scale: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor
    q_inv_rms: Optional[torch.Tensor]
    k_inv_rms: Optional[torch.Tensor]
    k_mean: Optional[torch.Tensor]
    q_mean: Optional[torch.Tensor] = None
    k_bias: Optional[torch.Tensor] = None

    @staticmethod
    def empty(shape, cfg: Config, device) -> "QuantBufs":
        B, H, N, d = shape
        f32 = dict(dtype=torch.float32, device=device)
        i8 = dict(dtype=torch.int8, device=device)
        return QuantBufs(
            torch.empty(shape, **i8), torch.empty(shape, **i8), torch.empty(shape, **i8),
            torch.empty((B, H, N // cfg.q_block), **f32),
            torch.empty((B, H, N // cfg.k_block), **f32),
            torch.empty((B, H, N // cfg.k_block), **f32),
            torch.empty((B, H, N), **f32) if cfg.qknorm else None,
            torch.empty((B, H, N), **f32) if cfg.qknorm else None,
            torch.empty((B, H, d), **f32) if cfg.ksmooth else None,
            torch.empty((B, H, d), **f32) if cfg.qsmooth else None,
            torch.empty((B, H, N), **f32) if cfg.qsmooth else None)

    def c_struct(self) -> SageQBufs:
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        return SageQBufs(p(self.q_codes), p(self.k_codes), p(self.v_codes), p(self.q_scale),
                         p(self.k_scale), p(self.v_scale), p(self.q_inv_rms),
                         p(self.k_inv_rms), p(self.k_mean), p(self.q_mean), p(self.k_bias))


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_inputs(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("libsage works on CUDA tensors only")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")


def workspace_bytes(params: SageParams, which: int) -> int:
    return int(lib().sage_workspace_bytes(ctypes.byref(params), which))


def _workspace(params: SageParams, which: int, device) -> Tuple[Optional[torch.Tensor], int]:
    n = workspace_bytes(params, which)
    if n == 0:
        return None, 0
    return torch.empty(n, dtype=torch.uint8, device=device), n


def quant_prologue(q, k, v, cfg: Config, out: Optional[QuantBufs] = None,
                   workspace: Optional[torch.Tensor] = None) -> QuantBufs:
    """QK-norm, K-smoothing and per-block INT8 quantization of q, k, v (sage_quant_prologue)."""
    _check_inputs(q, k, v)
    prm = cfg.params(q)
    qb = out if out is not None else QuantBufs.empty(tuple(q.shape), cfg, q.device)
    if workspace is None:
        workspace, n = _workspace(prm, 0, q.device)
    else:
        n = workspace.numel()
    st = qb.c_struct()
    check("sage_quant_prologue", lib().sage_quant_prologue(
        ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
        None if workspace is None else workspace.data_ptr(), n, _stream(q.device)))
    return qb


def attn_fwd(qb: QuantBufs, like: torch.Tensor, cfg: Config, o=None, lse=None):
    """INT8 forward attention (sage_attn_fwd): returns (o, lse)."""
    prm = cfg.params(like)
    B, H, N, d = like.shape
    if o is None:
        o = torch.empty_like(like)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=like.device)
    st = qb.c_struct()
    check("sage_attn_fwd", lib().sage_attn_fwd(ctypes.byref(prm), ctypes.byref(st),
                                               o.data_ptr(), lse.data_ptr(), None, 0,
                                               _stream(like.device)))
    return o, lse


def attn_bwd(q, k, v, qb: QuantBufs, o, lse, dout, cfg: Config, dq=None, dk=None, dv=None,
             workspace: Optional[torch.Tensor] = None, stage: Optional[int] = None):
    """INT8 backward attention (sage_attn_bwd): returns (dq, dk, dv).

    ``stage`` in {0, 1, 2} runs only that stage (sage_attn_bwd_stage); the caller then owns
    ``workspace`` across the three calls.
    """
    _check_inputs(q, k, v, o, dout)
    prm = cfg.params(q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace, n = _workspace(prm, 2, q.device)
    else:
        n = workspace.numel()
    st = qb.c_struct()
    args = (ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(st),
            o.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
            dv.data_ptr(), workspace.data_ptr(), n, _stream(q.device))
    if stage is None:
        check("sage_attn_bwd", lib().sage_attn_bwd(*args))
    else:
        check("sage_attn_bwd_stage", lib().sage_attn_bwd_stage(stage, *args))
    return dq, dk, dv


def device_status(device=None) -> int:
    """Synchronize the current stream and read (and clear) the device status word."""
    return int(lib().sage_last_device_status(_stream(device)))


class _SageAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cfg: Config):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        qb = quant_prologue(q, k, v, cfg)
        o, lse = attn_fwd(qb, q, cfg)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.qb, ctx.cfg = qb, cfg
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attn_bwd(q, k, v, ctx.qb, o, lse, do.contiguous(), ctx.cfg)
        return dq, dk, dv, None


def sage_attention(q, k, v, causal: bool = True, qknorm: bool = True, ksmooth: bool = True,
                   q_block: int = 128, k_block: int = 64, softmax_scale: float = 0.0,
                   rms_eps: float = 1e-6, qsmooth: bool = False):
    """SageBwd attention with autograd: q, k, v are CUDA [B, H, N, d] fp16/bf16 tensors."""
    cfg = Config(causal, qknorm, ksmooth, q_block, k_block, softmax_scale, rms_eps, qsmooth)
    return _SageAttention.apply(q, k, v, cfg)


def umma_gemm_debug(kind: int, a: torch.Tensor, b: torch.Tensor, a_mn: bool, b_mn: bool,
                    N: int, K: int) -> torch.Tensor:
    """Run the tensor-core path on one 128 x N x K product (sage_debug_umma_gemm)."""
    c = torch.empty((128, N), dtype=torch.int32 if kind == 0 else torch.float32,
                    device=a.device)
    check("sage_debug_umma_gemm", lib().sage_debug_umma_gemm(
        kind, int(a_mn), int(b_mn), N, K, a.data_ptr(), b.data_ptr(), c.data_ptr(),
        _stream(a.device)))
    return c


def wait_timeout_debug(limit_us: int, device=None) -> None:
    """Launch a kernel whose bounded barrier wait runs out (sage_debug_wait_timeout)."""
    check("sage_debug_wait_timeout",
          lib().sage_debug_wait_timeout(int(limit_us), _stream(device)))


def mma_peak(kind: int, n_ctas: int, groups: int, fill: torch.Tensor) -> None:
    """Launch the tensor-core throughput loop (sage_mma_peak) on the current stream.

    ``kind`` 0 = INT8, 1 = fp16, 2 = bf16; ``fill`` is a device tensor of at least 48 KB whose
    bytes become the operands.  Ops per launch: see ``mma_peak_ops``.
    """
    check("sage_mma_peak", lib().sage_mma_peak(kind, n_ctas, groups, fill.data_ptr(),
                                               fill.numel() * fill.element_size(),
                                               _stream(fill.device)))


def mma_peak_ops(kind: int, n_ctas: int, groups: int) -> float:
    """Operations of one sage_mma_peak launch: 4 MMAs of 128 x 256 x K per group and CTA."""
    k = 32 if kind == 0 else 16
    return float(n_ctas) * groups * 4 * 2 * 128 * 256 * k


def qk_int32_debug(qb: QuantBufs, like: torch.Tensor, cfg: Config, bh: int,
                   q_tile: int) -> torch.Tensor:
    """INT8 score tile Qc Kc^T of the forward kernel's MMA path (sage_debug_qk_int32)."""
    prm = cfg.params(like)
    N = like.shape[2]
    s = torch.empty((128, N), dtype=torch.int32, device=like.device)
    st = qb.c_struct()
    check("sage_debug_qk_int32", lib().sage_debug_qk_int32(
        ctypes.byref(prm), ctypes.byref(st), bh, q_tile, s.data_ptr(), _stream(like.device)))
    return s


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def host_workspace_bytes(cfg: Config, like: torch.Tensor, chunks: int) -> int:
    """Device workspace of fwd_bwd_host (sage_fwd_bwd_host_workspace_bytes)."""
    return int(lib().sage_fwd_bwd_host_workspace_bytes(ctypes.byref(cfg.params(like)), chunks))


class HostPipeline:
    """Device workspace and streams for repeated ``fwd_bwd_host`` calls on one device."""

    def __init__(self, like: torch.Tensor, cfg: Config, chunks: int = 16, device=None):
        self.device = torch.device("cuda") if device is None else torch.device(device)
        self.chunks = chunks
        n = host_workspace_bytes(cfg, like, chunks)
        self.workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=self.device)
        self.streams = [torch.cuda.Stream(self.device) for _ in range(3)]


def fwd_bwd_host(q, k, v, dout, cfg: Config, o=None, dq=None, dk=None, dv=None,
                 chunks: int = 16, device=None, pipeline: Optional[HostPipeline] = None):
    """Prologue + forward + backward on host-resident [B, H, N, d] tensors (sage_fwd_bwd_host).

    The C entry point cuts the batch into ``chunks`` slices and overlaps each slice's
    host-to-device copies, kernels and device-to-host copies on three streams; it returns once
    the results (o, dq, dk, dv; pinned host tensors, allocated when not given) are complete.
    Inputs should be pinned for the copies to run asynchronously.  ``pipeline`` reuses a device
    workspace and streams across calls.
    """
    for t in (q, k, v, dout):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("fwd_bwd_host takes contiguous host tensors")
    outs = []
    for t, ref in ((o, q), (dq, q), (dk, k), (dv, v)):
        outs.append(t if t is not None else torch.empty(ref.shape, dtype=ref.dtype,
                                                         pin_memory=True))
    if pipeline is None:
        pipeline = HostPipeline(q, cfg, chunks, device)
    prm = cfg.params(q)
    ws = pipeline.workspace
    with torch.cuda.device(pipeline.device):
        check("sage_fwd_bwd_host", lib().sage_fwd_bwd_host(
            ctypes.byref(prm), q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
            *(t.data_ptr() for t in outs), pipeline.chunks, ws.data_ptr(), ws.numel(),
            *(s_.cuda_stream for s_ in pipeline.streams)))
    return tuple(outs)

"""Shared helpers for the GPU parity tests: run the CUDA path and the oracle on the same inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.sage_oracle as O
from fwd_bwd_b200 import ops
from fwd_bwd_b200.inputs import Workload, make_inputs

TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def to_device(bits: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
        TORCH_DT[dtype]).cuda()


def cfg_of(w: Workload) -> ops.Config:
    return ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                      k_block=w.k_block, qsmooth=w.qsmooth)


def gpu_run(w: Workload, x: dict, backward: bool = True) -> dict:
    """Prologue, forward (and backward) on the GPU; every result copied to numpy."""
    q, k, v, do = (to_device(x[n], w.dtype) for n in ("q", "k", "v", "do"))
    cfg = cfg_of(w)
    qb = ops.quant_prologue(q, k, v, cfg)
    o, lse = ops.attn_fwd(qb, q, cfg)
    res = {}
    if backward:
        dq, dk, dv = ops.attn_bwd(q, k, v, qb, o, lse, do, cfg)
        res.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    res.update(o=o, lse=lse)
    for name in ("q_codes", "k_codes", "v_codes", "q_scale", "k_scale", "v_scale",
                 "q_inv_rms", "k_inv_rms", "k_mean", "q_mean", "k_bias"):
        t = getattr(qb, name)
        if t is not None:
            res[name] = t
    out = {}
    for kk, t in res.items():
        t = t.float() if t.dtype in (torch.bfloat16, torch.float16) else t
        out[kk] = t.cpu().numpy()
    out["_qb"] = qb
    out["_dev"] = (q, k, v, do)
    return out


def heads_view(a: np.ndarray, w: Workload) -> np.ndarray:
    return a.reshape(w.B * w.H, *a.shape[2:])


def oracle_run(w: Workload, x: dict, quant: bool = True) -> dict:
    args = [x[n + "_f32"] for n in ("q", "k", "v", "do")]
    args = [a.reshape(-1, w.N, w.d) for a in args]
    return O.sage_attention(*args, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth,
                            q_block=w.q_block, k_block=w.k_block, dtype=w.dtype, quant=quant,
                            round_outputs=quant, qsmooth=w.qsmooth)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / math.sqrt(max((a @ a) * (b @ b), 1e-300)))


__all__ = ["gpu_run", "oracle_run", "rel_l2", "cosine", "heads_view", "make_inputs",
           "to_device", "cfg_of", "TORCH_DT"]

"""Tokens-per-step study of the SageBwd quantization bias (a measurement, not part of the operator).

The SageBwd page ("SageBwd: trainable low-bit attention", tokens-per-step and limitation
paragraphs) reports that the INT8 recipe's gap to full precision grows with the number of
tokens per optimizer step: a large batch averages the stochastic part of the gradient away,
which leaves the quantization's systematic bias visible, while at a small batch the sampling
noise masks it.  This module measures that on synthetic inputs with shared structure
(``inputs.make_study_inputs``):

for every tokens-per-step value T (= B * N) and every seed, the gradients of the CUDA path
(Q mode) and of full-precision attention (float64, ``full_precision_grads``) are averaged over
all T tokens and all heads, per channel -- the batch-averaged gradient a per-channel parameter
acting on q or k would receive.  Over the seeds it reports

* ``bias``   = || mean_s (G_Q - G_X) ||   the systematic quantization error of the average;
* ``qnoise`` = rms_s || (G_Q - G_X) - mean ||   its seed-to-seed (random) part;
* ``snoise`` = rms_s || G_X - mean_s G_X ||     the sampling noise of the exact average;
* ``visibility`` = bias / snoise.

Pooled over every run (all T, all seeds), per-token figures give the extrapolation the page's
claim is about: the pooled bias ``b`` (token-weighted mean error, with its standard error), the
per-token gradient spread ``sigma_g = snoise(T) sqrt(T)`` and error spread
``sigma_e = qnoise(T) sqrt(T)`` (both near constant in T), and ``T* = (sigma_g / |b|)^2``, the
tokens per step beyond which the bias would exceed the sampling noise (computed with
``max(|b|, 2 stderr)``, i.e. a lower bound on T* when no bias is resolved).

Run: ``python -m fwd_bwd_b200.tps_study --out result.json`` (one CUDA device).
"""
from __future__ import annotations

import argparse
import json
import math
import time
from typing import Dict, Sequence

import torch

from . import ops
from .inputs import WORKLOADS, Workload, make_study_inputs


def full_precision_grads(q, k, v, do, cfg: ops.Config, dtype=torch.float64):
    """Full-precision attention and its input gradients, one batch element at a time.

    QK-norm (``x * (mean(x^2) + eps)^-1/2`` per token), K-smoothing (per-channel token mean
    subtracted), ``softmax((q^ k~^T) tau)`` with the causal mask, ``o = P v``; gradients of
    ``sum(o * do)`` by autograd, all in ``dtype``.  Q-smoothing is exact in full precision
    and so changes nothing here.  Returns ``(o, dq, dk, dv)`` in ``dtype``.
    """
    B, H, N, d = q.shape
    tau = cfg.softmax_scale if cfg.softmax_scale > 0 else 1.0 / math.sqrt(d)
    outs = [torch.empty((B, H, N, d), dtype=dtype, device=q.device) for _ in range(4)]
    mask = torch.ones(N, N, dtype=torch.bool, device=q.device).triu(1) if cfg.causal else None
    for b in range(B):
        qb, kb, vb = (x[b].to(dtype).requires_grad_(True) for x in (q, k, v))
        qh, kh = qb, kb
        if cfg.qknorm:
            qh = qb * torch.rsqrt((qb * qb).mean(-1, keepdim=True) + cfg.rms_eps)
            kh = kb * torch.rsqrt((kb * kb).mean(-1, keepdim=True) + cfg.rms_eps)
        if cfg.ksmooth:
            kh = kh - kh.mean(-2, keepdim=True)
        s = (qh @ kh.transpose(-1, -2)) * tau
        if mask is not None:
            s = s.masked_fill(mask, float("-inf"))
        o = torch.softmax(s, dim=-1) @ vb
        (o * do[b].to(dtype)).sum().backward()
        for dst, src in zip(outs, (o.detach(), qb.grad, kb.grad, vb.grad)):
            dst[b] = src
    return tuple(outs)


def _avg(g: torch.Tensor) -> torch.Tensor:
    """Per-channel average over batch, heads and tokens, in float64."""
    return g.to(torch.float64).mean(dim=(0, 1, 2))


def measure(w: Workload, batches: Sequence[int], seeds: Sequence[int],
            device: str = "cuda") -> Dict:
    cfg = ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                     k_block=w.k_block, qsmooth=w.qsmooth)
    rows = []
    for B in batches:
        wb = w.replace(B=B)
        g = {n: [] for n in ("q_Q", "q_X", "k_Q", "k_X")}
        for seed in seeds:
            x = make_study_inputs(wb, seed, device)
            qb = ops.quant_prologue(x["q"], x["k"], x["v"], cfg)
            o, lse = ops.attn_fwd(qb, x["q"], cfg)
            dq, dk, _ = ops.attn_bwd(x["q"], x["k"], x["v"], qb, o, lse, x["do"], cfg)
            if ops.device_status() != 0:
                raise RuntimeError("device status not OK")
            _, dqx, dkx, _ = full_precision_grads(x["q"], x["k"], x["v"], x["do"], cfg)
            g["q_Q"].append(_avg(dq))
            g["q_X"].append(_avg(dqx))
            g["k_Q"].append(_avg(dk))
            g["k_X"].append(_avg(dkx))
        row = {"B": B, "tokens_per_step": B * w.N, "seeds": len(seeds)}
        for t in ("q", "k"):
            gq = torch.stack(g[t + "_Q"])
            gx = torch.stack(g[t + "_X"])
            e = gq - gx
            bias = e.mean(0)
            qnoise = ((e - bias) ** 2).sum(1).mean().sqrt()
            snoise = ((gx - gx.mean(0)) ** 2).sum(1).mean().sqrt()
            row[f"d{t}"] = {
                "bias": float(bias.norm()),
                "bias_stderr": float(qnoise / math.sqrt(len(seeds))),
                "qnoise": float(qnoise),
                "snoise": float(snoise),
                "signal": float(gx.mean(0).norm()),
                "visibility": float(bias.norm() / snoise),
            }
        for t in ("q", "k"):
            row[f"_e_{t}"] = torch.stack(g[t + "_Q"]) - torch.stack(g[t + "_X"])
        rows.append(row)
    pooled = {}
    for t in ("q", "k"):
        num = sum(r[f"_e_{t}"].sum(0) * r["tokens_per_step"] for r in rows)
        den = sum(r["tokens_per_step"] * r["seeds"] for r in rows)
        b = num / den
        sig_e = sum(r[f"d{t}"]["qnoise"] * math.sqrt(r["tokens_per_step"]) for r in rows) / len(rows)
        sig_g = sum(r[f"d{t}"]["snoise"] * math.sqrt(r["tokens_per_step"]) for r in rows) / len(rows)
        stderr = sig_e / math.sqrt(den)
        resolved = float(b.norm()) > 2 * stderr
        pooled[f"d{t}"] = {"total_tokens": den, "bias": float(b.norm()), "bias_stderr": stderr,
                           "bias_resolved": resolved, "sigma_e_per_token": sig_e,
                           "sigma_g_per_token": sig_g,
                           "T_star": (sig_g / max(float(b.norm()), 2 * stderr)) ** 2,
                           "T_star_is_lower_bound": not resolved}
    for r in rows:
        for t in ("q", "k"):
            del r[f"_e_{t}"]
    return {"pooled": pooled, "workload": {"H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "dtype": w.dtype,
                         "q_block": w.q_block, "qknorm": w.qknorm, "ksmooth": w.ksmooth,
                         "qsmooth": w.qsmooth},
            "rows": rows}


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--N", type=int, default=2048)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--batches", type=str, default="1,2,4,8,16,32,64")
    ap.add_argument("--seeds", type=int, default=16)
    ap.add_argument("--qsmooth", action="store_true")
    ap.add_argument("--ksmooth-off", action="store_true")
    ap.add_argument("--out", type=str, default="")
    a = ap.parse_args()
    w = WORKLOADS["sweep8192"].replace(N=a.N, H=a.H, qsmooth=a.qsmooth,
                                       ksmooth=not a.ksmooth_off)
    t0 = time.time()
    res = measure(w, [int(b) for b in a.batches.split(",")], list(range(a.seeds)))
    res["seconds"] = time.time() - t0
    txt = json.dumps(res, indent=1)
    if a.out:
        with open(a.out, "w") as f:
            f.write(txt)
    print(txt)


if __name__ == "__main__":
    main()

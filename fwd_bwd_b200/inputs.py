"""Seeded synthetic inputs for SageBwd attention (no method arithmetic lives here).

Both the CUDA path (through the tests and ``bench.py``) and the CPU oracle are fed from the
arrays this module returns, so it is the one piece of code they share.  It only draws random
numbers and stores them as 16-bit floats; it performs none of the quantization, normalization
or attention arithmetic.

Recipe (the same for every workload):

* per flattened head ``bh``, ``numpy.random.Generator(PCG64(SeedSequence([seed, offset,
  bh])))`` with offsets Q:0, K:1, V:2, dO:3, mu:4 (the K-outlier channel offsets), muQ:5
  (the Q-outlier channel offsets);
* ``standard_normal`` in float64, multiplied by the tensor's sigma, rounded to float32;
* float32 rounded to the 16-bit storage type with round-half-to-even (bf16 by bit
  manipulation, fp16 by numpy's own RNE cast).

Arrays are returned as ``uint16`` bit patterns in ``[B, H, N, d]`` order (``d`` innermost),
plus an exact float32 view for CPU consumers.

The workloads are the attention shapes of the SageBwd page ("SageBwd: trainable low-bit
attention", aitrends.kr): the 325M-Llama attention layer it pretrains, a K-outlier stress case
for the K-smoothing ablation, a Q-outlier case for the Q-smoothing variant, a long-sequence
case for the small-dS regime and the tokens-per-step sweep.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence

import numpy as np

OFFSET_Q, OFFSET_K, OFFSET_V, OFFSET_DO, OFFSET_MU, OFFSET_QMU = 0, 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, dtype and value distribution of one synthetic attention problem."""

    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtype: str  # "bf16" or "fp16"
    q_block: int = 128
    k_block: int = 64
    qknorm: bool = True
    ksmooth: bool = True
    sigma_qkv: float = 1.0
    sigma_do: float = 1.0
    k_outlier: bool = False  # per-channel offsets mu_c ~ N(0, 4^2), 4 channels +20
    q_outlier: bool = False  # the same kind of offsets on Q (own stream)
    qsmooth: bool = False    # run with Q-smoothing (an operator flag, carried with the shape)
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.N

    def ops(self, part: str = "fwdbwd") -> float:
        """Tensor-core op count (FlashAttention convention, masked half not credited)."""
        per_gemm = 2.0 * self.N * self.N * self.d * (0.5 if self.causal else 1.0)
        n = {"fwd": 2, "bwd": 5, "fwdbwd": 7}[part]
        return self.B * self.H * n * per_gemm

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # tiny correctness case (oracle finishes instantly)
    "tiny": Workload("tiny", 1, 2, 128, 64, False, "fp16", q_block=64, k_block=64,
                     sigma_do=1e-2),
    # 325M-Llama-like attention layer
    "llama325m": Workload("llama325m", 8, 16, 2048, 64, True, "bf16", sigma_do=1e-3),
    # K-outlier stress (run with the qknorm / ksmooth flags on and off)
    "koutlier": Workload("koutlier", 4, 16, 4096, 128, True, "bf16", k_outlier=True),
    # Q-outlier stress for the Q-smoothing variant (K outliers too, K-smoothing on)
    "qoutlier": Workload("qoutlier", 4, 16, 4096, 128, True, "bf16", k_outlier=True,
                         q_outlier=True, qsmooth=True),
    # long sequence, small-dS regime
    "long16k": Workload("long16k", 1, 32, 16384, 128, True, "bf16", sigma_do=1e-4),
}
# tokens-per-step sweep: B*N = 262144 tokens, H=16, d=128, causal
for _n in (1024, 2048, 4096, 8192):
    WORKLOADS[f"sweep{_n}"] = Workload(f"sweep{_n}", 262144 // _n, 16, _n, 128, True, "bf16")


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-half-to-even) and return the uint16 bit pattern."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bits_to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float32 value of 16-bit storage given as uint16 bit patterns."""
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float32)
    raise ValueError(dtype)


def f32_to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    if dtype == "fp16":
        return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)
    raise ValueError(dtype)


def _rng(w: Workload, offset: int, bh: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, offset, bh])))


def make_head(w: Workload, bh: int) -> Dict[str, np.ndarray]:
    """float32 values (before 16-bit rounding) of q, k, v, dO for flattened head ``bh``."""
    shape = (w.N, w.d)
    out = {}
    for name, off, sig in (("q", OFFSET_Q, w.sigma_qkv), ("k", OFFSET_K, w.sigma_qkv),
                           ("v", OFFSET_V, w.sigma_qkv), ("do", OFFSET_DO, w.sigma_do)):
        out[name] = (_rng(w, off, bh).standard_normal(shape) * sig).astype(np.float32)
    for name, flag, off in (("k", w.k_outlier, OFFSET_MU), ("q", w.q_outlier, OFFSET_QMU)):
        if flag:
            g = _rng(w, off, bh)
            mu = (g.standard_normal(w.d) * 4.0).astype(np.float32)
            chans = g.choice(w.d, size=4, replace=False)
            mu[chans] += np.float32(20.0)
            out[name] = (out[name] + mu[None, :]).astype(np.float32)
    return out


def make_inputs(w: Workload, heads: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Return {'q','k','v','do'} as uint16 bit arrays and '<name>_f32' exact float32 views.

    Each (batch, head) pair -- flattened index ``bh = b * H + h`` -- is drawn from its own
    stream, so any subset of heads can be regenerated alone.  Without ``heads`` the arrays
    are ``[B, H, N, d]``; with ``heads`` they are ``[len(heads), N, d]``.
    """
    idx = list(range(w.B * w.H)) if heads is None else list(heads)
    parts = [make_head(w, bh) for bh in idx]
    out: Dict[str, np.ndarray] = {}
    for name in ("q", "k", "v", "do"):
        arr = np.stack([p[name] for p in parts])
        if heads is None:
            arr = arr.reshape(w.B, w.H, w.N, w.d)
        bits = f32_to_bits(arr, w.dtype)
        out[name] = bits
        out[name + "_f32"] = bits_to_f32(bits, w.dtype)
    return out


def make_inputs_fast(w: Workload, device: str = "cpu"):
    """Large-workload inputs drawn with torch's generator (used only for timing runs).

    Same distributions as :func:`make_inputs` but a different (torch Philox) stream, so values
    are not comparable with ``make_inputs``; parity checks always use ``make_inputs``.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    shape = (w.B, w.H, w.N, w.d)
    res = {}
    for name, sig in (("q", w.sigma_qkv), ("k", w.sigma_qkv), ("v", w.sigma_qkv),
                      ("do", w.sigma_do)):
        res[name] = (torch.randn(shape, generator=g, device=device, dtype=torch.float32)
                     * sig).to(tdt)
    for name, flag in (("k", w.k_outlier), ("q", w.q_outlier)):
        if flag:
            mu = torch.randn((w.B, w.H, 1, w.d), generator=g, device=device) * 4.0
            mu[..., :4] += 20.0
            res[name] = (res[name].float() + mu).to(tdt)
    return res


def make_study_inputs(w: Workload, seed: int, device: str = "cpu"):
    """Inputs for the tokens-per-step study: per-seed noise on top of structure every seed shares.

    Trained activations have fixed outlier channels and gradients with a consistent direction;
    to give the batch-averaged gradient a non-zero expectation that is the same for every seed,
    Q, K and dO carry fixed per-channel offsets (drawn once from a generator seeded by ``d``):
    ``q = e + mu_q`` with ``mu_q ~ N(0, 1)``; ``k = e + mu_k`` with ``mu_k ~ N(0, 4^2)`` and +20 on
    4 channels (the K-outlier recipe); ``v = e``; ``dO = sigma_do (e + mu_do)`` with
    ``mu_do ~ N(0, 0.5^2)``; every ``e`` is fresh standard-normal noise from torch's generator
    seeded by ``seed``.  Values are rounded to the workload's 16-bit type.
    """
    import torch

    gf = torch.Generator(device="cpu")
    gf.manual_seed(10_000 + w.d)
    mu_q = torch.randn(w.d, generator=gf)
    mu_k = torch.randn(w.d, generator=gf) * 4.0
    mu_k[torch.randperm(w.d, generator=gf)[:4]] += 20.0
    mu_do = torch.randn(w.d, generator=gf) * 0.5
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    shape = (w.B, w.H, w.N, w.d)

    def noise():
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32)

    return {"q": (noise() + mu_q.to(device)).to(tdt),
            "k": (noise() + mu_k.to(device)).to(tdt),
            "v": noise().to(tdt),
            "do": ((noise() + mu_do.to(device)) * w.sigma_do).to(tdt)}

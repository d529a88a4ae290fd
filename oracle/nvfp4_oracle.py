"""CPU oracle for the NVFP4 Q-Attn variant -- TEST INFRASTRUCTURE, NOT PRODUCT CODE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module.  It shares no code with the CUDA path (``fwd_bwd_b200``).

What it follows:

* "Full-Stack FP4" (gist.science 2607.04422), section 2.4 "mixed-precision attention (Q-Attn)":
  the robust paths, Q K^T and dS, run in NVFP4; the softmax-sensitive paths, P V, P^T dO and
  dO V^T, stay in BF16; the quantized views of Q, K and V are produced once and reused by the
  forward and the backward pass.
* "Quartet II" (allinfo.ai.kr), plain-language section: the NVFP4 format is E2M1 values in
  blocks of 16 that share one E4M3 (FP8) scale, plus one global scale.

Readings (the pages fix neither rounding rules nor the global scale's extent):

* E2M1 magnitudes are {0, 0.5, 1, 1.5, 2, 3, 4, 6}; rounding is to nearest, ties to the code
  with an even low bit, and magnitudes above 6 saturate to 6.  The sign bit is the input's, so
  a negative value (or -0) that rounds to zero gets the -0 code 8, as IEEE rounding keeps the
  sign of a result that rounds to zero.  (``e2m1_encode``)
* Block scales are unsigned E4M3 (4 exponent bits, bias 7, 3 mantissa bits, subnormals,
  largest finite 448): round to nearest, ties to even, values of 448 and above saturate to 448.
  (``e4m3_encode``)
* The global scale covers one (batch, head) matrix -- the operand of one attention GEMM -- and
  maps that matrix's absolute maximum G onto 6 * 448 = 2688, the largest value a block scale
  times an element can reach: ``genc = 2688 / G`` (``genc = 1`` when G = 0).
* Per block of 16 consecutive channels, in float32 with IEEE rounding at every step:
  ``a = max |x|``, ``u = (a * genc) / 6``, ``sd = e4m3(u)`` (the stored scale),
  ``mult = genc / sd`` and ``code = e2m1(x * mult)``; ``sd = 0`` gives codes of value zero
  (``mult = 0``, so +0 or -0 by the sign of x).
  The value a code stands for is ``e2m1_value(code) * sd / genc``.
* Q and K are quantized along the head dimension (the contraction of Q K^T), after the same
  QK-norm and K-smoothing as the INT8 recipe (``sage_oracle.rms_norm_rows_f32``,
  ``sage_oracle.k_smooth_f32``).  V is not quantized (P V runs in BF16).
* Forward: scores from the dequantized operands (exact in float64), softmax and
  ``O = softmax(z) V`` in float64.  The kernel feeds P to the tensor core in BF16; the oracle
  keeps P exact, and the tests bound the difference that BF16 rounding of P can make.
* Backward (``qattn_bwd_head``): S recomputed from the same views, ``dP = dO V^T`` and
  ``dV = P^T dO`` from 16-bit operands, ``dS = P o (dP - D)``; dS is quantized per 128 x 128
  tile with the tile's maximum as its global scale, in 16-key blocks for ``dQ = tau dS K`` and
  in 16-query blocks for ``dK = tau dS^T Q``, whose K and Q operands are NVFP4 views along the
  sequence (blocks of 16 tokens, one global scale per head).
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import sage_oracle as S8

F32 = np.float32
F64 = np.float64

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=F64)
GLOBAL_RANGE = 2688.0  # 6 (largest E2M1 value) * 448 (largest E4M3 value)
NVFP4_BLOCK = 16


def e2m1_encode(y: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes (bit 3 = sign) of float32 values: nearest, ties to even, saturating.

    The magnitude code counts the rounding boundaries ``|y|`` has passed.  Between two
    neighbours the midpoint goes to the one whose code is even: 0.25 -> 0, 0.75 -> 1,
    1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4 (codes 0, 2, 2, 4, 4, 6, 6).  The sign
    bit is the sign bit of ``y`` (so -0.1 and -0.0 give the -0 code 8).
    """
    y = np.asarray(y, dtype=F32)
    a = np.abs(y)
    mag = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5)
           + (a >= 3.5) + (a > 5.0)).astype(np.uint8)
    return (mag | (np.signbit(y).astype(np.uint8) << 3)).astype(np.uint8)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    v = E2M1_VALUES[code & 7]
    return np.where(code & 8, -v, v)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """Value of an unsigned E4M3 byte (bias 7; exponent field 0 is subnormal, m * 2^-9)."""
    code = np.asarray(code, dtype=np.int64)
    e = (code >> 3) & 15
    m = code & 7
    return np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e - 10.0)).astype(F64)


def e4m3_encode(u: np.ndarray) -> np.ndarray:
    """Unsigned E4M3 code of non-negative float32 ``u``: nearest, ties to even, saturating.

    Below 2^-6 the grid is ``m * 2^-9`` (m = 0..8; m = 8 is the smallest normal, whose code
    is 8 too).  From 2^-6 on, with ``u = f * 2^e`` (1 <= f < 2), ``q = rne(8 f)`` in 8..16
    (16 carries into the exponent) and the code is ``(e + 7) << 3 | (q - 8)``.  448 and above
    give 448 (code 0x7E).  Scaling by powers of two is exact, so only ``rne`` rounds.
    """
    u = np.asarray(u, dtype=F32).astype(F64)
    sub = u < 2.0 ** -6
    q_sub = np.rint(u * 512.0)
    _, ex = np.frexp(np.where(sub, 1.0, u))  # u = f' 2^ex with f' in [0.5, 1)
    e = ex - 1
    q = np.rint(np.where(sub, 8.0, u) * np.exp2(3.0 - e))
    carry = q == 16
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 8, q)
    normal = ((e + 7) << 3) | (q.astype(np.int64) - 8)
    code = np.where(sub, q_sub.astype(np.int64), normal)
    code = np.where(u >= 448.0, 0x7E, code)
    return code.astype(np.uint8)


def nvfp4_quantize(x: np.ndarray) -> Dict[str, np.ndarray]:
    """NVFP4 quantization of ``x[..., N, d]`` along its last axis (blocks of 16 channels).

    One global scale per matrix (the last two axes).  Returns ``codes`` (uint8 values 0..15,
    one per element, ``x``'s shape), ``sf`` (E4M3 block-scale bytes, ``[..., N, d/16]``) and
    ``genc`` (float32 global encode scale, ``x.shape[:-2]``).
    """
    x = np.asarray(x, dtype=F32)
    *lead, N, d = x.shape
    G = np.max(np.abs(x), axis=(-2, -1)).astype(F32)
    genc = np.where(G > 0, F32(GLOBAL_RANGE) / np.where(G > 0, G, F32(1)), F32(1)).astype(F32)
    xb = x.reshape(*lead, N, d // NVFP4_BLOCK, NVFP4_BLOCK)
    a = np.max(np.abs(xb), axis=-1)
    g = genc.reshape(*genc.shape, 1, 1)
    u = ((a * g).astype(F32) / F32(6.0)).astype(F32)
    sf = e4m3_encode(u)
    sd = e4m3_decode(sf).astype(F32)
    mult = np.where(sd > 0, (g / np.where(sd > 0, sd, F32(1))).astype(F32), F32(0)).astype(F32)
    y = (xb * mult[..., None]).astype(F32)
    codes = e2m1_encode(y).reshape(x.shape)
    return {"codes": codes, "sf": sf, "genc": genc}


def nvfp4_dequantize(codes: np.ndarray, sf: np.ndarray, genc: np.ndarray) -> np.ndarray:
    """float64 values ``e2m1(code) * sd / genc`` of ``nvfp4_quantize``'s output."""
    *lead, N, d = codes.shape
    v = e2m1_decode(codes).reshape(*lead, N, d // NVFP4_BLOCK, NVFP4_BLOCK)
    v = v * e4m3_decode(sf)[..., None]
    return v.reshape(codes.shape) / np.asarray(genc, F64).reshape(*np.shape(genc), 1, 1)


def qattn_prologue(q, k, *, qknorm: bool, ksmooth: bool, eps: float = 1e-6,
                   k_block: int = 64) -> Dict[str, np.ndarray]:
    """QK-norm and K-smoothing (float32, as in the INT8 recipe), then NVFP4 views of Q and K.

    ``q``, ``k`` are float32 ``[BH, N, d]`` holding the exact 16-bit input values.
    """
    out: Dict[str, np.ndarray] = {}
    qh, kh = np.asarray(q, F32), np.asarray(k, F32)
    if qknorm:
        qh, out["q_inv_rms"] = S8.rms_norm_rows_f32(qh, eps)
        kh, out["k_inv_rms"] = S8.rms_norm_rows_f32(kh, eps)
    out["k_hat"] = kh
    if ksmooth:
        kh, out["k_mean"] = S8.k_smooth_f32(kh, k_block)
    out["q_hat"], out["k_tilde"] = qh, kh
    for name, x in (("q", qh), ("k", kh)):
        r = nvfp4_quantize(x)
        out[name + "_codes"], out[name + "_sf"], out[name + "_genc"] = r["codes"], r["sf"], r["genc"]
    return out


def qattn_fwd_head(qd: np.ndarray, kd: np.ndarray, v: np.ndarray, *, causal: bool,
                   tau: float) -> tuple:
    """Forward of one head from dequantized Q, K (float64 ``[N, d]``) and V.

    ``z = tau * qd kd^T`` (causal: key j visible to query i iff j <= i), ``m = max_j z``,
    ``p = exp(z - m)``, ``l = sum_j p``, ``O = (p V) / l``, ``LSE = m + ln l``.
    Returns ``(O, LSE)`` in float64.  Also returns ``W = (p |V|) / l`` per (row, channel), the
    weight the tests use to bound the effect of rounding P to BF16.
    """
    qd, kd, v = (np.asarray(t, F64) for t in (qd, kd, v))
    z = (qd @ kd.T) * tau
    if causal:
        N = z.shape[0]
        z = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, z)
    m = z.max(axis=1)
    p = np.exp(z - m[:, None])
    l = p.sum(axis=1)
    O = (p @ v) / l[:, None]
    W = (p @ np.abs(v)) / l[:, None]
    return O, m + np.log(l), W


def qattn_forward(q, k, v, *, causal: bool, qknorm: bool, ksmooth: bool,
                  tau: float | None = None, eps: float = 1e-6) -> Dict[str, np.ndarray]:
    """Prologue plus forward over every (batch, head); inputs float32 ``[BH, N, d]``."""
    q = np.asarray(q, F32)
    d = q.shape[-1]
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    pro = qattn_prologue(q, k, qknorm=qknorm, ksmooth=ksmooth, eps=eps)
    qd = nvfp4_dequantize(pro["q_codes"], pro["q_sf"], pro["q_genc"])
    kd = nvfp4_dequantize(pro["k_codes"], pro["k_sf"], pro["k_genc"])
    BH, N, _ = q.shape
    o = np.zeros((BH, N, d), F64)
    lse = np.zeros((BH, N), F64)
    w = np.zeros((BH, N, d), F64)
    for h in range(BH):
        o[h], lse[h], w[h] = qattn_fwd_head(qd[h], kd[h], v[h], causal=causal, tau=tau)
    pro.update(o=o, lse=lse, w=w, q_deq=qd, k_deq=kd)
    return pro


# ----------------------------------------------------------------------------------------------
# Backward (Full-Stack FP4 section 2.4: dS in NVFP4, P^T dO and dO V^T in BF16)
# ----------------------------------------------------------------------------------------------
def nvfp4_quantize_tile(x: np.ndarray, axis: int) -> np.ndarray:
    """Dequantized NVFP4 value of a tile ``x`` (2-D, float32) with ONE global scale for the
    whole tile and blocks of 16 along ``axis``; same float32 steps as ``nvfp4_quantize``.

    Reading (the pages fix no granularity for the operand made inside the backward): dS is
    quantized per 128 x 128 (query, key) tile -- the unit the kernel holds -- with the tile's
    absolute maximum as its global scale, so that both orientations (16-key blocks for
    ``dQ = dS K``, 16-query blocks for ``dK = dS^T Q``) share it.
    """
    x = np.asarray(x, F32)
    t = np.moveaxis(x, axis, -1)[None]
    r = nvfp4_quantize(t)
    deq = nvfp4_dequantize(r["codes"], r["sf"], r["genc"])[0]
    return np.moveaxis(deq, -1, axis)


def qattn_bwd_head(qd, kd, q_seq, k_seq, v, o, lse, do, *, causal: bool, tau: float,
                   quant: bool = True, tile: int = 128) -> tuple:
    """Backward of one head: returns ``(dQhat, dKtilde, dV)`` float64 ``[N, d]``.

    ``qd``/``kd``: the forward's dequantized NVFP4 views (along d); ``q_seq``/``k_seq``: the
    dequantized NVFP4 views along the sequence (blocks of 16 tokens, ``nvfp4_quantize`` of the
    transposed matrix, one global scale per head) -- the K-major operands of dQ and dK; ``v``,
    ``do``: exact 16-bit inputs; ``o``, ``lse``: the forward's outputs.  Steps:

    1. ``z = tau qd kd^T`` (causal mask), ``P = exp(z - LSE)``;
    2. ``dP = dO V^T`` (16-bit operands, exact products), ``D_i = sum_c dO_ic O_ic``,
       ``dS = P o (dP - D)``;
    3. per 128 x 128 tile, dS (rounded to float32, the kernel's precision) is quantized twice
       with the tile's global scale: in 16-key blocks (``dS_k``) and in 16-query blocks
       (``dS_q``) -- ``nvfp4_quantize_tile``;
    4. ``dV = P^T dO`` (16-bit operands: P exact here, the tests bound its BF16 rounding),
       ``dQ = tau dS_k k_seq``, ``dK = tau dS_q^T q_seq``.

    With ``quant=False`` every quantizer is the identity (``qd = q_seq`` = the exact Q etc.),
    which is plain attention's gradient.  The gradient for K is the one for the smoothed K,
    which equals the one for the normalized K (every row of dS sums to zero).
    """
    qd, kd, q_seq, k_seq, v, o, do = (np.asarray(t, F64) for t in (qd, kd, q_seq, k_seq, v, o, do))
    N, d = qd.shape
    z = (qd @ kd.T) * tau
    if causal:
        z = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, z)
    P = np.exp(z - np.asarray(lse, F64)[:, None])
    dP = do @ v.T
    D = (do * o).sum(axis=1)
    dS = P * (dP - D[:, None])
    dV = P.T @ do
    if quant:
        dS_k = np.zeros_like(dS)
        dS_q = np.zeros_like(dS)
        for i0 in range(0, N, tile):
            for j0 in range(0, N, tile):
                t = dS[i0:i0 + tile, j0:j0 + tile].astype(F32)
                dS_k[i0:i0 + tile, j0:j0 + tile] = nvfp4_quantize_tile(t, axis=1)
                dS_q[i0:i0 + tile, j0:j0 + tile] = nvfp4_quantize_tile(t, axis=0)
    else:
        dS_k = dS_q = dS
    dQ = (dS_k @ k_seq) * tau
    dK = (dS_q.T @ q_seq) * tau
    return dQ, dK, dV


def qattn_attention(q, k, v, do, *, causal: bool, qknorm: bool, ksmooth: bool,
                    tau: float | None = None, eps: float = 1e-6,
                    quant: bool = True, dtype: str | None = None) -> Dict[str, np.ndarray]:
    """NVFP4 Q-Attn forward and backward over every (batch, head).

    Inputs float32 ``[BH, N, d]`` (exact 16-bit values).  Returns the forward's results
    (``qattn_forward``) plus ``dq, dk, dv`` with respect to the raw q, k, v (RMSNorm backward
    applied when ``qknorm``).  ``quant=False``: full precision (float64, no quantizer).
    ``dtype`` ("bf16" / "fp16"): the outputs are stored in that 16-bit type, as the INT8
    path's ``sage_attention`` does -- ``o`` is rounded before the backward reads it (so
    ``D = rowsum(dO o O)`` takes the stored output) and ``dq, dk, dv`` at the end.
    """
    q, k, v, do = (np.asarray(t, F32) for t in (q, k, v, do))
    BH, N, d = q.shape
    tau = 1.0 / np.sqrt(d) if tau is None else tau
    if quant:
        res = qattn_forward(q, k, v, causal=causal, qknorm=qknorm, ksmooth=ksmooth, tau=tau,
                            eps=eps)
        qs = nvfp4_quantize(np.swapaxes(res["q_hat"], -1, -2))
        ks = nvfp4_quantize(np.swapaxes(res["k_tilde"], -1, -2))
        q_seq = np.swapaxes(nvfp4_dequantize(qs["codes"], qs["sf"], qs["genc"]), -1, -2)
        k_seq = np.swapaxes(nvfp4_dequantize(ks["codes"], ks["sf"], ks["genc"]), -1, -2)
        res.update(q_seq=q_seq, k_seq=k_seq)
        qd, kd = res["q_deq"], res["k_deq"]
    else:
        pro = S8.prologue_fp64(q, k, v, qknorm=qknorm, ksmooth=ksmooth, eps=eps)
        res = {"q_hat": pro["q_hat"], "k_hat": pro["k_hat"], "k_tilde": pro["k_tilde"]}
        if qknorm:
            res.update(q_inv_rms=pro["q_inv_rms"], k_inv_rms=pro["k_inv_rms"])
        qd = q_seq = pro["q_hat"]
        kd = k_seq = pro["k_tilde"]
        o = np.zeros((BH, N, d))
        lse = np.zeros((BH, N))
        for h in range(BH):
            o[h], lse[h], _ = qattn_fwd_head(qd[h], kd[h], v[h], causal=causal, tau=tau)
        res.update(o=o, lse=lse)
    if dtype is not None:
        res["o"] = S8.round_to_storage(res["o"], dtype).astype(F64)
    dq = np.zeros((BH, N, d))
    dk = np.zeros((BH, N, d))
    dv = np.zeros((BH, N, d))
    for h in range(BH):
        dqh, dkh, dv[h] = qattn_bwd_head(qd[h], kd[h], q_seq[h], k_seq[h], v[h], res["o"][h],
                                         res["lse"][h], do[h], causal=causal, tau=tau,
                                         quant=quant)
        if qknorm:  # the RMSNorm backward takes the normalized (unsmoothed) rows
            dqh = S8.rms_norm_bwd(dqh, res["q_hat"][h], res["q_inv_rms"][h])
            dkh = S8.rms_norm_bwd(dkh, res["k_hat"][h], res["k_inv_rms"][h])
        dq[h], dk[h] = dqh, dkh
    if dtype is not None:
        dq, dk, dv = (S8.round_to_storage(t, dtype).astype(F64) for t in (dq, dk, dv))
    res.update(dq=dq, dk=dk, dv=dv, tau=tau)
    return res

"""CPU oracle for SageBwd quantized attention -- TEST INFRASTRUCTURE, NOT PRODUCT CODE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module.  It shares no code with the CUDA path (``fwd_bwd_b200``): it is a plain, slow,
step-by-step restatement of the method, used to prove the GPU kernels right.

What it follows ("SageBwd: trainable low-bit attention", aitrends.kr):

* quantization strategy paragraph -- six of the seven attention matmuls run in INT8
  (S = QK^T, O = PV, the recomputed S, dV = P^T dO, dQ = dS K, dK = dS^T Q); dP = dO V^T stays
  in 16-bit float;
* QK-norm paragraph -- RMSNorm applied to every token vector of Q and K;
* K-smoothing paragraph -- a mean is subtracted from K just before quantization
  (read here as the per-channel mean over tokens, see ``k_smooth``);
* Q-smoothing paragraph (limitations) -- smoothing Q as well needs the bias correction
  ``dK_bias = (dS^T 1) mu_Q^T`` (optional ``qsmooth`` flag; see ``bias_dot_f32`` and
  ``attn_bwd_head``);
* Triton-kernel paragraph -- per-block quantization;
* error-propagation paragraph -- dQ = dS K and dK = dS^T Q.

The page gives no reduction orders, block shapes, rounding rules or scale granularities for P
and dS; every such choice below is a stated reading (the module docstrings of each function
say which).  Two modes come from the same attention functions:

* Q mode (``quant=True``): the recipe, with INT8 codes, exact integer products and the
  continuous arithmetic (dequantization, softmax, dP, D) in float64.  Every decision that
  produces an integer code is taken in float32, the precision the GPU kernels take it in.
  The prologue (RMSNorm, smoothing, quantization of Q, K, V) runs entirely in float32 in a
  fixed operation order, because its INT8 codes and scales are compared bit for bit.
* X mode (``quant=False``): every quantizer replaced by the identity, all arithmetic in
  float64 -- full-precision attention, the reference the Q-mode error is measured against.

Integer GEMMs are evaluated as float64 matrix products of integer-valued arrays: every product
of two codes is at most 127^2 and every sum at most 127^2 * 16384 < 2^53, so each result is the
exact integer.
"""
from __future__ import annotations

import math
from typing import Dict

import numpy as np

F32 = np.float32
F64 = np.float64


# ----------------------------------------------------------------------------------------------
# 16-bit rounding of outputs (the oracle's own; round-half-to-even)
# ----------------------------------------------------------------------------------------------
def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the 16-bit output type (via float32) and return the exact float32 values."""
    x32 = np.ascontiguousarray(x, dtype=F32)
    if dtype == "fp16":
        return x32.astype(np.float16).astype(F32)
    if dtype == "bf16":
        u = x32.view(np.uint32).astype(np.uint64)
        u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
        return u.astype(np.uint32).view(F32)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------------------------
# Per-block symmetric INT8 quantization (Triton-kernel paragraph: "per-block quantization")
# ----------------------------------------------------------------------------------------------
def quantize_groups(x: np.ndarray, axes) -> tuple:
    """Symmetric INT8 quantization with one scale per group.

    ``axes`` are the axes one group spans.  Per group, in float32: ``a = max|x|``,
    ``s = a / 127`` (IEEE division), ``code = clamp(rne(x / s), -127, 127)``; a group with
    ``a == 0`` gets ``s = 0`` and all-zero codes.  Returns ``(codes int8, scales float32)`` with
    the scales keeping the reduced axes as length-1 dimensions.
    """
    x = np.asarray(x, dtype=F32)
    a = np.max(np.abs(x), axis=axes, keepdims=True)
    s = (a / F32(127.0)).astype(F32)
    nz = s > 0
    safe = np.where(nz, s, F32(1.0))
    c = np.rint(x / safe)  # float32 / float32 -> float32, then round-half-to-even
    c = np.where(nz, c, F32(0.0))
    c = np.clip(c, -127, 127).astype(np.int8)
    return c, s


def quantize_token_blocks(x: np.ndarray, blk: int) -> tuple:
    """Quantize ``x[..., N, d]`` in blocks of ``blk`` consecutive tokens spanning all channels.

    Returns codes with ``x``'s shape and scales of shape ``[..., N // blk]``.
    """
    *lead, N, d = x.shape
    xb = np.asarray(x, dtype=F32).reshape(*lead, N // blk, blk, d)
    c, s = quantize_groups(xb, axes=(-2, -1))
    return c.reshape(x.shape), s.reshape(*lead, N // blk)


# ----------------------------------------------------------------------------------------------
# Prologue: QK-norm, K-smoothing, quantization (float32, fixed order: compared bit for bit)
# ----------------------------------------------------------------------------------------------
def rms_norm_rows_f32(x: np.ndarray, eps: float) -> tuple:
    """Per-token RMSNorm over the head dimension in float32 (QK-norm paragraph).

    The page fixes neither the reduction order nor epsilon; the reading taken is: the row's
    ``d`` channels are split into ``d/8`` lanes of 8 consecutive channels; each lane sums
    ``x_c * x_c`` (each product and each sum rounded to float32) in ascending channel order from
    +0; the lane partials are combined by a butterfly (for ``o = L/2, ..., 1``:
    ``p_l <- p_l + p_(l xor o)``) and lane 0's value is the sum of squares ``ss``.  Then
    ``inv = 1 / sqrt(ss / d + eps)`` and ``xhat = x * inv``, each operation correctly rounded
    in float32.  No learnable gain (the page mentions none).  ``x`` is ``[..., N, d]``.
    """
    x = np.asarray(x, dtype=F32)
    d = x.shape[-1]
    L = d // 8
    xl = x.reshape(*x.shape[:-1], L, 8)
    p = np.zeros(x.shape[:-1] + (L,), dtype=F32)
    for c in range(8):
        p = p + xl[..., c] * xl[..., c]
    lanes = np.arange(L)
    o = L // 2
    while o >= 1:
        p = p + p[..., lanes ^ o]
        o //= 2
    ss = p[..., 0]
    ms = ss / F32(d)
    r = np.sqrt(ms + F32(eps))
    inv = (F32(1.0) / r).astype(F32)
    return (x * inv[..., None]).astype(F32), inv


def k_smooth_f32(khat: np.ndarray, k_block: int) -> tuple:
    """Subtract the per-channel mean over all tokens from K (K-smoothing paragraph).

    The page says the mean is removed from K right before quantization to suppress outliers
    concentrated in particular channels; the reading taken is the per-channel mean over the
    sequence (the only reading under which softmax is unchanged, since every score of a query
    row shifts by the same ``q_i . m``), over all N tokens even when causal.  Summation order
    (float32): per block of ``k_block`` tokens, each channel is summed over the block's tokens
    in ascending order from +0; the block sums are added in ascending block order from +0;
    ``m = S / N``.  ``khat`` is ``[..., N, d]``; returns ``(khat - m, m)``.
    """
    khat = np.asarray(khat, dtype=F32)
    N = khat.shape[-2]
    S = np.zeros(khat.shape[:-2] + khat.shape[-1:], dtype=F32)
    for t in range(N // k_block):
        c = np.zeros_like(S)
        for r in range(t * k_block, (t + 1) * k_block):
            c = c + khat[..., r, :]
        S = S + c
    m = (S / F32(N)).astype(F32)
    return (khat - m[..., None, :]).astype(F32), m


def bias_dot_f32(m: np.ndarray, x: np.ndarray) -> np.ndarray:
    """Per-token bias ``b_j = sum_c m_c x_jc`` in float32 (Q-smoothing bias, see ``prologue``).

    ``m`` is ``[..., d]``, ``x`` is ``[..., N, d]``.  Reduction order (a reading; the page gives
    none): the same lane structure as ``rms_norm_rows_f32`` -- ``d/8`` lanes of 8 consecutive
    channels, each summing ``m_c * x_c`` (product and sum each rounded to float32) in ascending
    channel order from +0, then the butterfly over lanes; lane 0 holds the result.
    """
    m = np.asarray(m, dtype=F32)
    x = np.asarray(x, dtype=F32)
    d = x.shape[-1]
    L = d // 8
    xl = x.reshape(*x.shape[:-1], L, 8)
    ml = m.reshape(*m.shape[:-1], 1, L, 8)
    p = np.zeros(x.shape[:-1] + (L,), dtype=F32)
    for c in range(8):
        p = p + (ml[..., c] * xl[..., c]).astype(F32)
    lanes = np.arange(L)
    o = L // 2
    while o >= 1:
        p = p + p[..., lanes ^ o]
        o //= 2
    return p[..., 0].astype(F32)


def prologue(q, k, v, *, q_block: int, k_block: int, qknorm: bool, ksmooth: bool,
             eps: float = 1e-6, qsmooth: bool = False) -> Dict[str, np.ndarray]:
    """QK-norm -> smoothing -> per-block INT8 quantization of Q, K and V (float32 exact).

    Inputs are float32 arrays ``[BH, N, d]`` holding the exact values of the 16-bit inputs.
    Order (K-smoothing paragraph: smoothing comes right before quantization): normalize, then
    smooth, then quantize.  Q uses blocks of ``q_block`` tokens, K and V blocks of ``k_block``
    tokens; every block spans all ``d`` channels.

    ``qsmooth`` (Q-smoothing paragraph): ``mu_Q``, the per-channel mean of the normalized Q over
    all tokens (same summation order as K's, blocks of ``k_block`` tokens), is subtracted before
    Q is quantized.  Scores then lose the term ``mu_Q . k~_j``, which -- unlike K's row-constant
    shift -- differs per key and so changes softmax; it is restored as a per-key bias
    ``k_bias_j = mu_Q . k~_j`` (``bias_dot_f32``, from the unquantized smoothed K) that the
    attention adds to every score of key j.
    """
    q = np.asarray(q, dtype=F32)
    k = np.asarray(k, dtype=F32)
    v = np.asarray(v, dtype=F32)
    out: Dict[str, np.ndarray] = {}
    qh, kh = q, k
    if qknorm:
        qh, out["q_inv_rms"] = rms_norm_rows_f32(q, eps)
        kh, out["k_inv_rms"] = rms_norm_rows_f32(k, eps)
    out["k_hat"] = kh
    if ksmooth:
        kh, out["k_mean"] = k_smooth_f32(kh, k_block)
    out["q_hat"], out["k_tilde"] = qh, kh
    qt = qh
    if qsmooth:
        qt, out["q_mean"] = k_smooth_f32(qh, k_block)
        out["k_bias"] = bias_dot_f32(out["q_mean"], kh)
    out["q_tilde"] = qt
    out["q_codes"], out["q_scale"] = quantize_token_blocks(qt, q_block)
    out["k_codes"], out["k_scale"] = quantize_token_blocks(kh, k_block)
    out["v_codes"], out["v_scale"] = quantize_token_blocks(v, k_block)
    return out


def prologue_fp64(q, k, v, *, qknorm: bool, ksmooth: bool, eps: float = 1e-6,
                  qsmooth: bool = False) -> Dict:
    """X-mode prologue: RMSNorm and mean subtraction in float64 with no quantization."""
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    out = {"v": np.asarray(v, dtype=F64)}
    qh, kh = q, k
    d = q.shape[-1]
    if qknorm:
        out["q_inv_rms"] = 1.0 / np.sqrt((q * q).sum(-1) / d + eps)
        out["k_inv_rms"] = 1.0 / np.sqrt((k * k).sum(-1) / d + eps)
        qh = q * out["q_inv_rms"][..., None]
        kh = k * out["k_inv_rms"][..., None]
    out["k_hat"] = kh
    if ksmooth:
        out["k_mean"] = kh.mean(axis=-2)
        kh = kh - out["k_mean"][..., None, :]
    out["q_hat"], out["k_tilde"] = qh, kh
    out["q_tilde"] = qh
    if qsmooth:
        out["q_mean"] = qh.mean(axis=-2)
        out["q_tilde"] = qh - out["q_mean"][..., None, :]
        out["k_bias"] = np.einsum("...nc,...c->...n", kh, out["q_mean"])
    return out


# ----------------------------------------------------------------------------------------------
# Attention forward and backward for one (batch, head), Q mode or X mode
# ----------------------------------------------------------------------------------------------
class _Quant:
    """The quantizers of one mode: Q mode quantizes, X mode passes values through."""

    def __init__(self, quant: bool):
        self.quant = quant

    def rows_per_block(self, x: np.ndarray):
        """One scale per row of a [rows, cols] chunk (forward P: per query row per K block)."""
        if not self.quant:
            return np.asarray(x, F64), np.ones((x.shape[0], 1), F64)
        c, s = quantize_groups(np.asarray(x, F32), axes=(1,))
        return c.astype(F64), s.astype(F64)

    def tile(self, x: np.ndarray):
        """One scale for a whole [BQ, BK] tile (backward P and dS)."""
        if not self.quant:
            return np.asarray(x, F64), F64(1.0)
        c, s = quantize_groups(np.asarray(x, F32), axes=(0, 1))
        return c.astype(F64), F64(s.reshape(()))

    def tokens(self, x: np.ndarray, blk: int):
        """One scale per block of ``blk`` tokens (dO in the backward pass)."""
        if not self.quant:
            return np.asarray(x, F64), np.ones(x.shape[0] // blk, F64)
        c, s = quantize_token_blocks(np.asarray(x, F32), blk)
        return c.astype(F64), s.astype(F64)


def _scores(qc, sq_row, kc, sk_col, tau, causal, i0, k_bias=None):
    """z = (A * (sQ * sK) + b) * tau with A = Qc Kc^T exact; causal keys > query get -inf.

    ``k_bias`` (Q-smoothing only) is the per-key bias ``b_j``; without it ``b = 0``.  ``qc``
    holds the query rows ``i0 .. i0 + rows``; causal alignment is square and top-left (key j is
    visible to query i iff j <= i).
    """
    A = qc @ kc.T
    z = A * (sq_row[:, None] * sk_col[None, :])
    if k_bias is not None:
        z = z + np.asarray(k_bias, F64)[None, :]
    z = z * tau
    if causal:
        qi = np.arange(i0, i0 + qc.shape[0])[:, None]
        kj = np.arange(kc.shape[0])[None, :]
        z = np.where(kj > qi, -np.inf, z)
    return z


def attn_fwd_head(qc, q_scale, kc, k_scale, vc, v_scale, *, q_block: int, k_block: int,
                  causal: bool, tau: float, quant: bool = True, k_bias=None,
                  q_mean=None) -> tuple:
    """Forward attention of one head: returns ``(O float64 [N,d], LSE float64 [N])``.

    Inputs are per-token-block codes and scales (Q mode) or float64 values with unit scales
    (X mode).  Steps (quantization-strategy paragraph, FlashAttention block structure):

    1. ``A = Qc Kc^T`` (exact integers), ``z = (A * (sQ sK)) * tau``, causal mask;
    2. row max ``m`` and ``l = sum_j exp(z - m)`` over the unquantized probabilities;
    3. for every K block: ``p = exp(z - m)`` is quantized with one scale per query row
       (``sP = max_j p / 127``), and ``O += (Pc Vc) * (sP sV)``;
    4. ``O /= l``, ``LSE = m + ln l`` (natural log, in units of the scaled scores).

    With Q-smoothing, ``k_bias`` is added to the scores of step 1 (``q_mean`` is unused here).

    Reading: the page only says "per-block"; P gets one scale per (query row, K block).  The
    codes ``rne(p / (max p / 127))`` depend on ``p`` only through ``p / max p``, so they are the
    same whether ``p`` is taken relative to a running maximum (an online softmax) or to the
    final row maximum as here, and so is the dequantized sum; this closed form is what any
    block order computes in exact arithmetic.
    """
    qz = _Quant(quant)
    N, d = qc.shape
    qc = np.asarray(qc, F64)
    kc = np.asarray(kc, F64)
    vc = np.asarray(vc, F64)
    sq_row = np.repeat(np.asarray(q_scale, F64), q_block)
    sk_col = np.repeat(np.asarray(k_scale, F64), k_block)
    O = np.zeros((N, d), F64)
    LSE = np.zeros(N, F64)
    for i0 in range(0, N, q_block):
        rows = slice(i0, i0 + q_block)
        z = _scores(qc[rows], sq_row[rows], kc, sk_col, tau, causal, i0, k_bias)
        m = z.max(axis=1)
        e = np.exp(z - m[:, None])
        l = e.sum(axis=1)
        acc = np.zeros((q_block, d), F64)
        for j in range(N // k_block):
            cols = slice(j * k_block, (j + 1) * k_block)
            pc, sp = qz.rows_per_block(e[:, cols])
            acc += (pc @ vc[cols]) * (sp * F64(v_scale[j]))
        O[rows] = acc / l[:, None]
        LSE[rows] = m + np.log(l)
    return O, LSE


def attn_bwd_head(qc, q_scale, kc, k_scale, vc, v_scale, v_raw, o_out, lse, do_raw, *,
                  q_block: int, k_block: int, causal: bool, tau: float,
                  quant: bool = True, k_bias=None, q_mean=None) -> tuple:
    """Backward attention of one head: returns ``(dQhat, dKtilde, dV)`` as float64 ``[N, d]``.

    ``v_raw``/``do_raw`` are the 16-bit inputs' exact values (the FP16 GEMM operands),
    ``o_out`` the stored forward output, ``lse`` the forward's log-sum-exp.  Steps
    (quantization-strategy and error-propagation paragraphs):

    1. recompute ``z`` exactly as the forward does and ``P = exp(z - LSE)``;
    2. ``dP = dO V^T`` from the 16-bit operands (the one matmul kept in 16-bit float);
    3. ``D_i = sum_c dO_ic O_ic`` from the stored output, ``dS = P o (dP - D)``;
    4. quantize dO per ``q_block`` tokens, and P and dS with one scale per
       ``q_block x k_block`` tile (reading: one dS quantization must serve both ``dQ``, which
       contracts over keys, and ``dK``, which contracts over queries, so its scale has to be
       constant over the tile);
    5. ``dV += (Pc^T dOc)(sP sdO)``, ``dK += (dSc^T Qc)(sdS sQ) tau``,
       ``dQ += (dSc Kc)(sdS sK) tau``.

    The gradient returned for K is the gradient with respect to the smoothed K; it is also the
    gradient with respect to the normalized K, because the mean-subtraction Jacobian
    contributes ``-(1/N) sum_j dK_j``, and ``sum_j dK_j = tau sum_i q_i sum_j dS_ij = 0`` since
    every row of ``dS`` sums to zero (reading: that term is dropped).

    Q-smoothing (``k_bias`` and ``q_mean`` given; ``qc`` then holds the smoothed Q): the scores
    carry the bias of the forward, and dK gains the page's correction term
    ``dK_bias = tau (dS^T 1) mu_Q^T``, the gradient through ``b_j = mu_Q . k~_j``.  Its column
    sums ``dS^T 1`` are taken over the same quantized dS tile the INT8 GEMM uses (reading: the
    page names this term as an added quantization-noise path), i.e. ``sdS * sum_i dSc_ij``.
    dQ needs no term: with respect to the normalized Q, the mean terms of the smoothing and of
    the bias cancel exactly, as for K.
    """
    qz = _Quant(quant)
    N, d = qc.shape
    qc = np.asarray(qc, F64)
    kc = np.asarray(kc, F64)
    vc = np.asarray(vc, F64)
    v_raw = np.asarray(v_raw, F64)
    do_raw = np.asarray(do_raw, F64)
    sq_row = np.repeat(np.asarray(q_scale, F64), q_block)
    sk_col = np.repeat(np.asarray(k_scale, F64), k_block)
    D = (do_raw * np.asarray(o_out, F64)).sum(axis=1)
    doc, sdo = qz.tokens(do_raw, q_block)
    dQ = np.zeros((N, d), F64)
    dK = np.zeros((N, d), F64)
    dV = np.zeros((N, d), F64)
    for bi, i0 in enumerate(range(0, N, q_block)):
        rows = slice(i0, i0 + q_block)
        z = _scores(qc[rows], sq_row[rows], kc, sk_col, tau, causal, i0, k_bias)
        P = np.exp(z - np.asarray(lse, F64)[rows][:, None])
        dP = do_raw[rows] @ v_raw.T
        dS = P * (dP - D[rows][:, None])
        for j in range(N // k_block):
            cols = slice(j * k_block, (j + 1) * k_block)
            pc, sp = qz.tile(P[:, cols])
            dsc, sds = qz.tile(dS[:, cols])
            dV[cols] += (pc.T @ doc[rows]) * (sp * sdo[bi])
            dK[cols] += (dsc.T @ qc[rows]) * (sds * sq_row[i0]) * tau
            if q_mean is not None:
                dK[cols] += np.outer(dsc.sum(axis=0) * sds, np.asarray(q_mean, F64)) * tau
            dQ[rows] += (dsc @ kc[cols]) * (sds * sk_col[j * k_block]) * tau
    return dQ, dK, dV


def rms_norm_bwd(g_hat: np.ndarray, x_hat: np.ndarray, inv: np.ndarray) -> np.ndarray:
    """Gradient through ``xhat = x * inv``, ``inv = (mean(x^2) + eps)^(-1/2)`` (QK-norm).

    ``dx = inv * (dxhat - xhat * (sum_c dxhat_c xhat_c) / d)``, all in float64.
    """
    g_hat = np.asarray(g_hat, F64)
    x_hat = np.asarray(x_hat, F64)
    d = g_hat.shape[-1]
    dot = (g_hat * x_hat).sum(-1, keepdims=True)
    return np.asarray(inv, F64)[..., None] * (g_hat - x_hat * dot / d)


# ----------------------------------------------------------------------------------------------
# Whole operator over [BH, N, d]
# ----------------------------------------------------------------------------------------------
def sage_attention(q, k, v, do, *, causal: bool, qknorm: bool, ksmooth: bool, q_block: int,
                   k_block: int, dtype: str, tau: float = 0.0, eps: float = 1e-6,
                   quant: bool = True, round_outputs: bool = True,
                   qsmooth: bool = False) -> Dict[str, np.ndarray]:
    """Prologue, forward and backward over all heads.

    ``q, k, v, do`` are float32 ``[BH, N, d]`` holding the exact 16-bit input values.  Returns
    the prologue buffers (Q mode), ``o`` (rounded to ``dtype`` when ``round_outputs``),
    ``lse``, and ``dq, dk, dv`` -- gradients with respect to the raw ``q, k, v`` (the RMSNorm
    backward applied when ``qknorm``).
    """
    BH, N, d = q.shape
    tau = tau if tau > 0 else 1.0 / math.sqrt(d)
    if quant:
        pro = prologue(q, k, v, q_block=q_block, k_block=k_block, qknorm=qknorm,
                       ksmooth=ksmooth, eps=eps, qsmooth=qsmooth)
        ops = (pro["q_codes"], pro["q_scale"], pro["k_codes"], pro["k_scale"],
               pro["v_codes"], pro["v_scale"])
    else:
        pro = prologue_fp64(q, k, v, qknorm=qknorm, ksmooth=ksmooth, eps=eps, qsmooth=qsmooth)
        ones_q = np.ones((BH, N // q_block))
        ones_k = np.ones((BH, N // k_block))
        ops = (pro["q_tilde"], ones_q, pro["k_tilde"], ones_k, pro["v"], ones_k)
    res = dict(pro)
    o = np.zeros((BH, N, d))
    lse = np.zeros((BH, N))
    dq = np.zeros((BH, N, d))
    dk = np.zeros((BH, N, d))
    dv = np.zeros((BH, N, d))
    kw = dict(q_block=q_block, k_block=k_block, causal=causal, tau=tau, quant=quant)
    for h in range(BH):
        head_ops = [x[h] for x in ops]
        if qsmooth:
            kw.update(k_bias=pro["k_bias"][h], q_mean=pro["q_mean"][h])
        oh, lse[h] = attn_fwd_head(*head_ops, **kw)
        o[h] = round_to_storage(oh, dtype) if round_outputs else oh
        dqh, dkh, dv[h] = attn_bwd_head(*head_ops, v[h], o[h], lse[h], do[h], **kw)
        if qknorm:
            dqh = rms_norm_bwd(dqh, pro["q_hat"][h], pro["q_inv_rms"][h])
            dkh = rms_norm_bwd(dkh, pro["k_hat"][h], pro["k_inv_rms"][h])
        dq[h], dk[h] = dqh, dkh
    if round_outputs:
        dq, dk, dv = (round_to_storage(x, dtype) for x in (dq, dk, dv))
    res.update(o=o, lse=lse, dq=dq, dk=dk, dv=dv, tau=tau)
    return res


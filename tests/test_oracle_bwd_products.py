"""Pins for the quantized products of the oracle's Q-mode backward (and forward) pass.

The SageBwd page ("SageBwd: trainable low-bit attention", error-propagation paragraph) puts
the recipe's risk in ``dQ = dS K`` and ``dK = dS^T Q``: the quantization error of dS flows
through both.  These tests recompute the three INT8 products of the backward pass (quantization-
strategy paragraph: ``dV = P^T dO``, ``dK = dS^T Q``, ``dQ = dS K``) from scratch -- element
loops over a brute-force per-tile quantizer written here, with every scale looked up by hand
from the block an element lies in -- and require ``attn_bwd_head`` to agree to float64
rounding.  The inputs have strongly different magnitudes per block (QK-norm off), so a scale
taken from the wrong block, a per-row instead of per-tile dS scale, dO quantized on the wrong
token blocks, or a dropped dS scale all change the result; ``test_planted_mistakes`` applies
each of these mistakes to the oracle's source and checks that the pin fails.

The forward pass gets the same treatment: O and LSE recomputed row by row (the softmax over
the visible keys, P quantized with one scale per query row and K block, the integer P V product
of each block dequantized by that scale and the V block's), against ``attn_fwd_head``, with
planted mistakes of the same kind.

Also pinned here: the oracle's bf16 output rounding against torch's bf16 conversion (a library
routine) on ties, large values and subnormals.
"""
import inspect
import math
import textwrap

import numpy as np
import pytest
import torch

import oracle.sage_oracle as O

F32 = np.float32


def _tile_quant_brute(x):
    """Symmetric INT8 with one scale for the whole 2-D tile, element by element in float32:
    a = max |x|, s = a / 127, code = round-half-even(x / s) clamped to +-127; a = 0 -> s = 0,
    codes 0.  Returns (codes as Python ints, s as a float32)."""
    a = F32(0.0)
    for v in np.asarray(x, F32).ravel():
        a = max(a, F32(abs(v)))
    s = F32(a / F32(127.0))
    codes = np.zeros(x.shape, dtype=np.int64)
    if s > 0:
        for idx, v in np.ndenumerate(np.asarray(x, F32)):
            t = float(F32(v / s))
            c = round(t)  # Python rounds half to even
            codes[idx] = max(-127, min(127, c))
    return codes, s


def _token_quant_brute(x, blk):
    """One scale per block of ``blk`` tokens (rows) spanning all channels."""
    N = x.shape[0]
    codes = np.zeros(x.shape, dtype=np.int64)
    scales = []
    for b in range(N // blk):
        c, s = _tile_quant_brute(x[b * blk:(b + 1) * blk])
        codes[b * blk:(b + 1) * blk] = c
        scales.append(s)
    return codes, scales


def _problem(seed, N, d, q_block, k_block, causal):
    """Per-block magnitudes spread over ~3 decades so that every block has its own scale."""
    g = np.random.default_rng(seed)
    def blocks(n, blk):  # magnitudes e^-3 .. e^3 in a seeded order, one per block
        return np.repeat(np.exp(g.permutation(np.linspace(-3, 3, n // blk))), blk)[:, None]

    q = (g.standard_normal((N, d)) * blocks(N, q_block) * 0.3).astype(F32)
    k = (g.standard_normal((N, d)) * blocks(N, k_block) * 0.3).astype(F32)
    v = (g.standard_normal((N, d)) * blocks(N, k_block)).astype(F32)
    do = (g.standard_normal((N, d)) * blocks(N, q_block)).astype(F32)
    o = (g.standard_normal((N, d)) * 0.5).astype(F32)  # any stored output: only D uses it
    pro = O.prologue(q[None], k[None], v[None], q_block=q_block, k_block=k_block, qknorm=False,
                     ksmooth=False)
    tau = 1.0 / math.sqrt(d)
    qc, sq = pro["q_codes"][0], pro["q_scale"][0]
    kc, sk = pro["k_codes"][0], pro["k_scale"][0]
    vc, sv = pro["v_codes"][0], pro["v_scale"][0]
    _, lse = O.attn_fwd_head(qc, sq, kc, sk, vc, sv, q_block=q_block, k_block=k_block,
                             causal=causal, tau=tau)
    return dict(q=q, k=k, v=v, do=do, o=o, qc=qc, sq=sq, kc=kc, sk=sk, vc=vc, sv=sv, lse=lse,
                tau=tau, N=N, d=d, q_block=q_block, k_block=k_block, causal=causal)


def _brute_products(p):
    """dQ, dK, dV of the recipe by explicit loops (float64 continuous arithmetic)."""
    N, d, BQ, BK, tau = p["N"], p["d"], p["q_block"], p["k_block"], p["tau"]
    qc, kc = p["qc"].astype(np.int64), p["kc"].astype(np.int64)
    # z_ij = (sum_c qc_ic kc_jc) * (sQ(block of i) * sK(block of j)) * tau; P = exp(z - LSE_i)
    P = np.zeros((N, N))
    for i in range(N):
        for j in range(N):
            if p["causal"] and j > i:
                continue
            a = int(np.dot(qc[i], kc[j]))
            z = a * (float(p["sq"][i // BQ]) * float(p["sk"][j // BK])) * tau
            P[i, j] = math.exp(z - float(p["lse"][i]))
    do64 = p["do"].astype(np.float64)
    dP = np.array([[float(np.dot(do64[i], p["v"][j].astype(np.float64))) for j in range(N)]
                   for i in range(N)])
    Dv = np.array([float(np.dot(do64[i], p["o"][i].astype(np.float64))) for i in range(N)])
    dS = P * (dP - Dv[:, None])
    doc, sdo = _token_quant_brute(p["do"], BQ)
    dQ = np.zeros((N, d))
    dK = np.zeros((N, d))
    dV = np.zeros((N, d))
    for bi in range(N // BQ):
        for bj in range(N // BK):
            rows = range(bi * BQ, (bi + 1) * BQ)
            cols = range(bj * BK, (bj + 1) * BK)
            pc, sp = _tile_quant_brute(P[bi * BQ:(bi + 1) * BQ, bj * BK:(bj + 1) * BK])
            dsc, sds = _tile_quant_brute(dS[bi * BQ:(bi + 1) * BQ, bj * BK:(bj + 1) * BK])
            iv = np.zeros((BK, d), np.int64)  # sum_i Pc_ij dOc_i
            ik = np.zeros((BK, d), np.int64)  # sum_i dSc_ij Qc_i
            iq = np.zeros((BQ, d), np.int64)  # sum_j dSc_ij Kc_j
            for a_, i in enumerate(rows):
                for b_, j in enumerate(cols):
                    iv[b_] += pc[a_, b_] * doc[i]
                    ik[b_] += dsc[a_, b_] * qc[i]
                    iq[a_] += dsc[a_, b_] * kc[j]
            # the scales: P / dS of this tile, dO and Q of query block bi, K of key block bj
            dV[bj * BK:(bj + 1) * BK] += iv * (float(sp) * float(sdo[bi]))
            dK[bj * BK:(bj + 1) * BK] += ik * (float(sds) * float(p["sq"][bi])) * tau
            dQ[bi * BQ:(bi + 1) * BQ] += iq * (float(sds) * float(p["sk"][bj])) * tau
    return dQ, dK, dV


def _oracle_products(p, bwd=None):
    bwd = bwd or O.attn_bwd_head
    return bwd(p["qc"], p["sq"], p["kc"], p["sk"], p["vc"], p["sv"], p["v"], p["o"], p["lse"],
               p["do"], q_block=p["q_block"], k_block=p["k_block"], causal=p["causal"],
               tau=p["tau"])


CASES = [
    # seed, N, d, q_block, k_block, causal
    (31, 256, 16, 128, 64, True),
    (32, 256, 16, 128, 64, False),
    (33, 192, 8, 64, 64, True),
]
_BRUTE = {}


def _brute(case):
    if case not in _BRUTE:
        p = _problem(*case)
        _BRUTE[case] = (p, _brute_products(p))
    return _BRUTE[case]


def _products_agree(case, bwd=None):
    p, ref = _brute(case)
    got = _oracle_products(p, bwd)
    return all(np.allclose(g, r, rtol=1e-12, atol=1e-12 * np.abs(r).max())
               for g, r in zip(got, ref))


@pytest.mark.parametrize("case", CASES)
def test_qmode_bwd_products_brute_force(case):
    p, ref = _brute(case)
    # the problem really has distinct scales per block (otherwise the pin would be weak)
    assert np.ptp(np.log(p["sq"])) > 2 and np.ptp(np.log(p["sk"])) > 2
    got = _oracle_products(p)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-12, atol=1e-12 * np.abs(r).max(),
                                   err_msg=name)


# Each mutation rewrites one expression of attn_bwd_head's source into a plausible mistake.
MUTATIONS = {
    "Q scale of the wrong block in dK": (
        "(sds * sq_row[i0]) * tau", "(sds * sq_row[(i0 + q_block) % N]) * tau"),
    "dropped dS scale in dK": ("(sds * sq_row[i0]) * tau", "(sq_row[i0]) * tau"),
    "K scale of the wrong block in dQ": (
        "(sds * sk_col[j * k_block]) * tau", "(sds * sk_col[((j + 1) * k_block) % N]) * tau"),
    "dO quantized per K block": ("qz.tokens(do_raw, q_block)", "qz.tokens(do_raw, k_block)"),
    "dO scale of the first block": ("(sp * sdo[bi])", "(sp * sdo[0])"),
    "per-row dS scale": (
        "dsc, sds = qz.tile(dS[:, cols])",
        "dsc, sds = qz.rows_per_block(dS[:, cols]); dsc = dsc * (sds / sds.max()); "
        "sds = F64(sds.max())"),
    "per-row P scale": (
        "pc, sp = qz.tile(P[:, cols])",
        "pc, sp = qz.rows_per_block(P[:, cols]); pc = pc * (sp / sp.max()); sp = F64(sp.max())"),
    "dK contracted with dO codes": ("(dsc.T @ qc[rows])", "(dsc.T @ doc[rows])"),
}


def _mutated(old, new):
    src = textwrap.dedent(inspect.getsource(O.attn_bwd_head))
    assert src.count(old) == 1, old
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutated attn_bwd_head>", "exec"), ns)
    return ns["attn_bwd_head"]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes(name):
    bwd = _mutated(*MUTATIONS[name])
    with np.errstate(invalid="ignore", divide="ignore"):
        assert not all(_products_agree(c, bwd) for c in CASES), name


def test_unmutated_source_passes():
    """The mutation harness itself is sound: the source recompiled unchanged passes."""
    src_fn = _mutated("qz = _Quant(quant)", "qz = _Quant(quant)")
    assert all(_products_agree(c, src_fn) for c in CASES)


# ------------------------------------------------------------------------------------------
# forward products
# ------------------------------------------------------------------------------------------
def _brute_forward(p):
    """O and LSE of the recipe row by row (float64 continuous arithmetic)."""
    N, d, BQ, BK, tau = p["N"], p["d"], p["q_block"], p["k_block"], p["tau"]
    qc, kc = p["qc"].astype(np.int64), p["kc"].astype(np.int64)
    vc = p["vc"].astype(np.int64)
    O_ = np.zeros((N, d))
    lse = np.zeros(N)
    for i in range(N):
        z = [None] * N
        for j in range(N):
            if p["causal"] and j > i:
                continue
            a = int(np.dot(qc[i], kc[j]))
            z[j] = a * (float(p["sq"][i // BQ]) * float(p["sk"][j // BK])) * tau
        m = max(v for v in z if v is not None)
        e = [0.0 if v is None else math.exp(v - m) for v in z]
        l = math.fsum(e)
        acc = np.zeros(d)
        for b in range(N // BK):
            # one scale per (query row, K block), the block's maximum / 127
            codes, s = _tile_quant_brute(np.array(e[b * BK:(b + 1) * BK])[None, :])
            iv = codes[0] @ vc[b * BK:(b + 1) * BK]
            acc += iv * (float(s) * float(p["sv"][b]))
        O_[i] = acc / l
        lse[i] = m + math.log(l)
    return O_, lse


def _oracle_forward(p, fwd=None):
    fwd = fwd or O.attn_fwd_head
    return fwd(p["qc"], p["sq"], p["kc"], p["sk"], p["vc"], p["sv"], q_block=p["q_block"],
               k_block=p["k_block"], causal=p["causal"], tau=p["tau"])


_BRUTE_FWD = {}


def _forward_agrees(case, fwd=None):
    if case not in _BRUTE_FWD:
        p = _problem(*case)
        _BRUTE_FWD[case] = (p, _brute_forward(p))
    p, ref = _BRUTE_FWD[case]
    got = _oracle_forward(p, fwd)
    return all(np.allclose(g, r, rtol=1e-12, atol=1e-12 * np.abs(r).max())
               for g, r in zip(got, ref))


@pytest.mark.parametrize("case", CASES)
def test_qmode_fwd_products_brute_force(case):
    assert _forward_agrees(case)


FWD_MUTATIONS = {
    "V scale of the wrong block": (
        "(sp * F64(v_scale[j]))", "(sp * F64(v_scale[(j + 1) % (N // k_block)]))"),
    "one P scale per tile instead of per row": (
        "pc, sp = qz.rows_per_block(e[:, cols])", "pc, sp = qz.tile(e[:, cols])"),
    "Q scale of the wrong block": (
        "_scores(qc[rows], sq_row[rows],", "_scores(qc[rows], sq_row[::-1][rows],"),
    "LSE in base 2": ("LSE[rows] = m + np.log(l)", "LSE[rows] = m + np.log2(l)"),
}


def _mutated_fwd(old, new):
    src = textwrap.dedent(inspect.getsource(O.attn_fwd_head))
    assert src.count(old) == 1, old
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutated attn_fwd_head>", "exec"), ns)
    return ns["attn_fwd_head"]


@pytest.mark.parametrize("name", sorted(FWD_MUTATIONS))
def test_planted_forward_mistakes(name):
    fwd = _mutated_fwd(*FWD_MUTATIONS[name])
    with np.errstate(invalid="ignore", divide="ignore"):
        assert not all(_forward_agrees(c, fwd) for c in CASES), name


# ------------------------------------------------------------------------------------------
# bf16 output rounding against torch's conversion
# ------------------------------------------------------------------------------------------
def test_round_to_storage_bf16_vs_torch():
    g = np.random.default_rng(40)
    vals = [g.standard_normal(4096) * np.exp(g.uniform(-30, 30, 4096))]
    # exact ties: the low 16 bits are 0x8000 (half-way), with even and odd bf16 mantissas
    base = (g.integers(0, 0x7F80, 2048, dtype=np.uint32) << 16) | 0x8000  # finite
    vals.append(base.view(np.float32))
    vals.append((base ^ 0x80000000).view(np.float32))
    # large magnitudes up to float32's maximum (rounding may carry into the exponent; values
    # at the top round to infinity as in IEEE)
    vals.append(np.array([3.3895314e38, 3.3961775e38, 3.4028235e38, -3.4e38, 65504.0,
                          1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 2 ** 126 * 1.5], np.float64))
    # subnormals and zeros
    vals.append(np.array([1e-40, -1e-40, 1e-45, 0.0, -0.0, 1.1754942e-38], np.float64))
    x = np.concatenate([np.asarray(v, np.float32) for v in vals])
    ours = O.round_to_storage(x, "bf16")
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), ref.view(np.uint32))

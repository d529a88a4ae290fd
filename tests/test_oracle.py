"""Pins for the CPU oracle: checks against things other than the oracle itself.

* hand-derived quantization codes (tests/golden/quantize_rne.txt) and quantizer error bounds;
* float32 RMSNorm / smoothing against their float64 definitions within float32 error bounds,
  and closed forms;
* X mode (full precision) against torch's float64 scaled_dot_product_attention with autograd,
  and against central finite differences;
* invariants the SageBwd page and the mathematics fix: softmax rows sum to one, dS rows sum to
  zero, K-smoothing leaves full-precision attention unchanged, RMS(dS) * sqrt(N) does not grow
  with N (the page's dS-magnitude bound);
* Q mode: exact integer S against brute force, a closed form (uniform attention), an explicit
  error bound for P quantization, cosine >= 0.995 against X mode, and the K-outlier trend.
* Q-smoothing (the optional variant of the Q-smoothing paragraph): in X mode the bias and the
  dK correction term make every output identical to Q-smoothing off; the prologue's mean and
  bias against their float64 definitions; in Q mode, scores of Q-outlier inputs are closer to
  full precision with Q-smoothing than without.
* planted mistakes in the oracle are caught by these pins.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.sage_oracle as O
from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _heads(x, w):
    return x.reshape(w.B * w.H, w.N, w.d)


def _cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / math.sqrt((a @ a) * (b @ b)))


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


# ------------------------------------------------------------------------------------------
# quantizer
# ------------------------------------------------------------------------------------------
def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "quantize_rne.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            xs, s, cs = line.split("|")
            rows.append((np.array(xs.split(), np.float32), np.float32(s),
                         np.array(cs.split(), np.int8)))
    return rows


@pytest.mark.parametrize("row", range(4))
def test_quantize_golden(row):
    x, s_exp, c_exp = _golden_rows()[row]
    c, s = O.quantize_groups(x[None, :], axes=(1,))
    assert s.reshape(()) == s_exp
    np.testing.assert_array_equal(c[0], c_exp)


def test_quantize_bounds():
    g = np.random.default_rng(1)
    x = (g.standard_normal((64, 8, 256)) * np.exp(g.uniform(-20, 5, (64, 1, 1)))).astype(
        np.float32)
    c, s = O.quantize_groups(x, axes=(1, 2))
    assert c.min() >= -127 and c.max() <= 127
    err = np.abs(x.astype(np.float64) - c.astype(np.float64) * s.astype(np.float64))
    # |x - code*s| <= s/2 up to the float32 rounding of x/s (one ulp of at most 127)
    assert np.all(err <= s.astype(np.float64) * (0.5 + 127 * 2.0 ** -23))
    # the element of largest magnitude maps to +-127
    am = np.abs(c.reshape(64, -1)).max(axis=1)
    np.testing.assert_array_equal(am, 127)


def test_quantize_zero_and_tiny_blocks():
    x = np.zeros((2, 64, 8), np.float32)
    x[1, 3, 2] = np.float32(1e-40)  # subnormal absmax: the scale is a subnormal, not zero
    c, s = O.quantize_token_blocks(x, 64)
    assert s[0, 0] == 0 and np.all(c[0] == 0)
    assert s[1, 0] > 0 and c[1, 3, 2] == 127 and np.count_nonzero(c[1]) == 1


# ------------------------------------------------------------------------------------------
# prologue
# ------------------------------------------------------------------------------------------
def test_rmsnorm_closed_form():
    # eps = 0: a row with one entry 16 has ss = 256, mean = 256/d; for d = 64 that is 4,
    # so r = 2 and inv = 0.5 exactly.
    x = np.zeros((3, 64), np.float32)
    x[0, 5] = 16.0
    x[1, :] = 1.0  # mean 1 -> inv 1
    x[2, ::2] = 2.0  # 32 entries of 4 -> ss 128, mean 2 -> inv 1/sqrt(2) (rounded)
    xh, inv = O.rms_norm_rows_f32(x, eps=0.0)
    assert inv[0] == np.float32(0.5) and inv[1] == np.float32(1.0)
    assert inv[2] == np.float32(1.0) / np.sqrt(np.float32(2.0))
    np.testing.assert_array_equal(xh[0], x[0] * np.float32(0.5))


@pytest.mark.parametrize("d", [64, 128])
def test_rmsnorm_f32_vs_fp64(d):
    g = np.random.default_rng(d)
    x = (g.standard_normal((500, d)) * np.exp(g.uniform(-3, 3, (500, 1)))).astype(np.float32)
    xh, inv = O.rms_norm_rows_f32(x, eps=1e-6)
    inv64 = 1.0 / np.sqrt((x.astype(np.float64) ** 2).mean(-1) + np.float64(np.float32(1e-6)))
    # float32 sum of d non-negative terms: relative error <= (d+4) * 2^-24 before the root
    assert np.all(np.abs(inv - inv64) / inv64 <= (d + 8) * 2.0 ** -24)
    np.testing.assert_allclose(xh, x * inv64[:, None], rtol=(d + 10) * 2.0 ** -24, atol=0)
    # rows have RMS sqrt(ms / (ms + eps)) (unit RMS up to epsilon), up to rounding
    ms = (x.astype(np.float64) ** 2).mean(-1)
    rms = np.sqrt((xh.astype(np.float64) ** 2).mean(-1))
    np.testing.assert_allclose(rms, np.sqrt(ms / (ms + np.float32(1e-6))), rtol=1e-6)


def test_ksmooth_mean():
    g = np.random.default_rng(3)
    N, d = 512, 128
    k = (g.standard_normal((2, N, d)) + 5 * g.standard_normal((2, 1, d))).astype(np.float32)
    kt, m = O.k_smooth_f32(k, 64)
    m64 = k.astype(np.float64).mean(axis=1)
    bound = N * 2.0 ** -24 * np.abs(k).max(axis=1) * 2
    assert np.all(np.abs(m - m64) <= bound)
    assert np.all(np.abs(kt.astype(np.float64).mean(axis=1)) <= bound + 2.0 ** -23 * np.abs(
        k).max(axis=1))


def test_prologue_codes_reconstruct():
    w = WORKLOADS["tiny"]
    x = make_inputs(w)
    pro = O.prologue(_heads(x["q_f32"], w), _heads(x["k_f32"], w), _heads(x["v_f32"], w),
                     q_block=64, k_block=64, qknorm=True, ksmooth=True)
    for name, src, blk in (("q", pro["q_hat"], 64), ("k", pro["k_tilde"], 64),
                           ("v", _heads(x["v_f32"], w), 64)):
        c = pro[name + "_codes"].astype(np.float64)
        s = np.repeat(pro[name + "_scale"], blk, axis=1)[..., None].astype(np.float64)
        assert np.all(np.abs(c * s - src) <= s * 0.50001)


# ------------------------------------------------------------------------------------------
# X mode (full precision) against torch float64 and finite differences
# ------------------------------------------------------------------------------------------
def _torch_reference(q, k, v, do, causal, qknorm, ksmooth, eps=1e-6):
    q, k, v, do = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in
                   (q, k, v, do))
    d = q.shape[-1]
    qh, kh = q, k
    if qknorm:
        qh = q * torch.rsqrt((q * q).mean(-1, keepdim=True) + eps)
        kh = k * torch.rsqrt((k * k).mean(-1, keepdim=True) + eps)
    if ksmooth:
        kh = kh - kh.mean(dim=-2, keepdim=True)
    o = torch.nn.functional.scaled_dot_product_attention(qh, kh, v, is_causal=causal,
                                                         scale=1.0 / math.sqrt(d))
    s = (qh @ kh.transpose(-1, -2)) / math.sqrt(d)
    if causal:
        n = s.shape[-1]
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    (o * do).sum().backward()
    return (o.detach().numpy(), lse.detach().numpy(), q.grad.numpy(), k.grad.numpy(),
            v.grad.numpy())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("qknorm,ksmooth", [(True, True), (False, False), (True, False),
                                            (False, True)])
def test_xmode_vs_torch_sdpa(causal, qknorm, ksmooth):
    g = np.random.default_rng(7)
    BH, N, d = 2, 128, 64
    q, k, v, do = (g.standard_normal((BH, N, d)) for _ in range(4))
    k = k + 3.0 * g.standard_normal((BH, 1, d))
    res = O.sage_attention(q, k, v, do, causal=causal, qknorm=qknorm, ksmooth=ksmooth,
                           q_block=64, k_block=32, dtype="bf16", quant=False,
                           round_outputs=False)
    o, lse, dq, dk, dv = _torch_reference(q, k, v, do, causal, qknorm, ksmooth)
    for a, b in ((res["o"], o), (res["lse"], lse), (res["dq"], dq), (res["dk"], dk),
                 (res["dv"], dv)):
        assert _rel(a, b) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_xmode_finite_differences(causal):
    g = np.random.default_rng(11)
    BH, N, d = 1, 16, 16
    q, k, v, do = (g.standard_normal((BH, N, d)) for _ in range(4))
    kw = dict(causal=causal, qknorm=True, ksmooth=True, q_block=8, k_block=4, dtype="bf16",
              quant=False, round_outputs=False)
    res = O.sage_attention(q, k, v, do, **kw)

    def loss(q_, k_, v_):
        return float((O.sage_attention(q_, k_, v_, do, **kw)["o"] * do).sum())

    h = 1e-5
    picks = [(0, 0, 0), (0, 5, 3), (0, 15, 15), (0, 9, 7)]
    for name, idx in (("dq", 0), ("dk", 1), ("dv", 2)):
        for p in picks:
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[idx][p] += h
            args_m[idx][p] -= h
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - res[name][p]) <= 1e-6 * max(1.0, abs(fd)), (name, p)


def test_xmode_invariants():
    g = np.random.default_rng(5)
    BH, N, d = 1, 256, 64
    q, k, v, do = (g.standard_normal((BH, N, d)) for _ in range(4))
    k = k + 4.0 * g.standard_normal((BH, 1, d))
    kw = dict(causal=True, qknorm=True, q_block=64, k_block=64, dtype="bf16", quant=False,
              round_outputs=False)
    on = O.sage_attention(q, k, v, do, ksmooth=True, **kw)
    off = O.sage_attention(q, k, v, do, ksmooth=False, **kw)
    # K-smoothing shifts every score of a query row by the same amount: outputs unchanged
    for n in ("o", "dq", "dk", "dv"):
        assert _rel(on[n], off[n]) < 1e-12
    # softmax rows sum to one; dS rows sum to zero
    pro = O.prologue_fp64(q, k, v, qknorm=True, ksmooth=True)
    z = pro["q_hat"][0] @ pro["k_tilde"][0].T / math.sqrt(d)
    z = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, z)
    P = np.exp(z - on["lse"][0][:, None])
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=0, atol=1e-12)
    dP = do[0] @ v[0].T
    Dv = (do[0] * on["o"][0]).sum(1)
    dS = P * (dP - Dv[:, None])
    assert np.abs(dS.sum(1)).max() < 1e-12 * np.abs(dS).max() * N


def test_rms_ds_bound_trend():
    """RMS(dS) * sqrt(N) does not grow with N (the page's dS magnitude bound, read as a bound)."""
    g = np.random.default_rng(9)
    d = 64
    vals = []
    for N in (128, 256, 512, 1024):
        q, k, v, do = (g.standard_normal((1, N, d)) for _ in range(4))
        pro = O.prologue_fp64(q, k, v, qknorm=True, ksmooth=True)
        z = pro["q_hat"][0] @ pro["k_tilde"][0].T / math.sqrt(d)
        P = np.exp(z - z.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        o = P @ v[0]
        dS = P * (do[0] @ v[0].T - (do[0] * o).sum(1, keepdims=True))
        vals.append(math.sqrt((dS ** 2).mean()) * math.sqrt(N))
    for a, b in zip(vals, vals[1:]):
        assert b <= a * 1.1


# ------------------------------------------------------------------------------------------
# Q mode
# ------------------------------------------------------------------------------------------
def test_qmode_integer_scores_brute_force():
    g = np.random.default_rng(2)
    qc = g.integers(-127, 128, (64, 64)).astype(np.int8)
    kc = g.integers(-127, 128, (128, 64)).astype(np.int8)
    A = np.zeros((64, 128), np.int64)
    for i in range(64):
        for j in range(128):
            A[i, j] = sum(int(qc[i, c]) * int(kc[j, c]) for c in range(64))
    z = O._scores(qc.astype(np.float64), np.ones(64), kc.astype(np.float64), np.ones(128), 1.0,
                  False, 0)
    np.testing.assert_array_equal(z, A.astype(np.float64))


def _lossless(g, shape, blk):
    """Integer-valued data with a +-127 in every block: per-block quantization is exact."""
    x = g.integers(-126, 127, shape).astype(np.float32)
    x.reshape(shape[0], shape[1] // blk, blk, shape[2])[:, :, 0, 0] = 127.0
    return x


def test_qmode_uniform_attention_closed_form():
    """Identical keys + K-smoothing -> zero scores -> O is the running mean of V."""
    g = np.random.default_rng(4)
    BH, N, d = 1, 256, 64
    q = g.standard_normal((BH, N, d)).astype(np.float32)
    # small integers: the float32 block sums and the mean are exact, so K - mean(K) is 0
    k = np.repeat(g.integers(-8, 9, (BH, 1, d)).astype(np.float32), N, axis=1)
    v = _lossless(g, (BH, N, d), 64)
    do = _lossless(g, (BH, N, d), 64)
    for causal in (False, True):
        res = O.sage_attention(q, k, v, do, causal=causal, qknorm=False, ksmooth=True,
                               q_block=64, k_block=64, dtype="bf16", round_outputs=False)
        assert np.all(res["k_codes"] == 0)
        cnt = np.arange(1, N + 1)[:, None] if causal else N
        mean_v = np.cumsum(v[0].astype(np.float64), 0) / cnt if causal else \
            v[0].astype(np.float64).mean(0, keepdims=True)
        np.testing.assert_allclose(res["o"][0], np.broadcast_to(mean_v, (N, d)), rtol=1e-6,
                                   atol=1e-6 * np.abs(v).max())
        assert np.all(res["dq"] == 0)  # dS K with all-zero K codes
        if not causal:
            np.testing.assert_allclose(res["dv"][0], np.broadcast_to(
                do[0].astype(np.float64).mean(0), (N, d)), rtol=1e-6, atol=1e-5)


def test_qmode_forward_error_bound():
    """With lossless Q, K, V only P is quantized: |O_q - O_x| <= sum_j (sP_j / 2) |v|_j / l."""
    g = np.random.default_rng(6)
    N, d, BK = 256, 64, 64
    q = _lossless(g, (1, N, d), 128) / 16  # scaled so softmax is not one-hot
    k = _lossless(g, (1, N, d), BK) / 16
    v = _lossless(g, (1, N, d), BK)
    for causal in (False, True):
        kw = dict(causal=causal, qknorm=False, ksmooth=False, q_block=128, k_block=BK,
                  dtype="bf16", round_outputs=False)
        oq = O.sage_attention(q, k, v, v, **kw)["o"][0]
        ox = O.sage_attention(q, k, v, v, quant=False, **kw)["o"][0]
        z = (q[0].astype(np.float64) @ k[0].T.astype(np.float64)) / 8.0
        if causal:
            z = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, z)
        e = np.exp(z - z.max(1, keepdims=True))
        l = e.sum(1)
        bound = np.zeros((N, d))
        for j in range(N // BK):
            cols = slice(j * BK, (j + 1) * BK)
            sp = e[:, cols].astype(np.float32).max(1).astype(np.float64) / 127
            bound += (sp / 2 + 1e-7)[:, None] * np.abs(v[0][cols]).sum(0)[None, :]
        assert np.all(np.abs(oq - ox) <= bound / l[:, None] + 1e-9)


@pytest.mark.parametrize("name", ["tiny", "small_causal"])
def test_qmode_cosine_vs_full_precision(name):
    if name == "tiny":
        w = WORKLOADS["tiny"]
    else:
        w = WORKLOADS["llama325m"].replace(B=1, H=2, N=512, d=128, sigma_do=1e-3)
    x = make_inputs(w)
    args = [_heads(x[n + "_f32"], w) for n in ("q", "k", "v", "do")]
    kw = dict(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
              k_block=w.k_block, dtype=w.dtype)
    rq = O.sage_attention(*args, **kw)
    rx = O.sage_attention(*args, quant=False, round_outputs=False, **kw)
    for n in ("o", "dq", "dk", "dv"):
        assert _cos(rq[n], rx[n]) >= 0.995, n


def test_qmode_k_outlier_trend():
    """With K outliers, K-smoothing lowers the quantization error (K-smoothing paragraph)."""
    w = WORKLOADS["koutlier"].replace(B=1, H=2, N=256)
    x = make_inputs(w)
    args = [_heads(x[n + "_f32"], w) for n in ("q", "k", "v", "do")]
    errs = {}
    for ks in (True, False):
        kw = dict(causal=True, qknorm=False, ksmooth=ks, q_block=128, k_block=64,
                  dtype="bf16")
        rq = O.sage_attention(*args, **kw)
        rx = O.sage_attention(*args, quant=False, round_outputs=False, **kw)
        errs[ks] = _rel(rq["o"], rx["o"])
    assert errs[True] < errs[False]


def test_qmode_k_outlier_ablation():
    """The K-outlier workload's four runs (K-smoothing on/off x QK-norm on/off; two heads at
    N = 1024): the recipe's accuracy against full precision.  K-smoothing is what keeps dQ
    accurate (the error-propagation paragraph: dQ = dS K inherits K's quantization error), and
    with both on every output keeps cosine >= 0.995."""
    w = WORKLOADS["koutlier"].replace(B=1, H=2, N=1024)
    x = make_inputs(w)
    args = [_heads(x[n + "_f32"], w) for n in ("q", "k", "v", "do")]
    err, cos = {}, {}
    for qn in (True, False):
        for ks in (True, False):
            kw = dict(causal=True, qknorm=qn, ksmooth=ks, q_block=128, k_block=64,
                      dtype="bf16")
            rq = O.sage_attention(*args, **kw)
            rx = O.sage_attention(*args, quant=False, round_outputs=False, **kw)
            for n in ("o", "dq", "dk", "dv"):
                a, b = rq[n].ravel(), rx[n].ravel()
                err[qn, ks, n] = _rel(rq[n], rx[n])
                cos[qn, ks, n] = float(a @ b / np.sqrt((a @ a) * (b @ b)))
    for qn in (True, False):
        assert err[qn, False, "dq"] > 3 * err[qn, True, "dq"]  # smoothing matters most for dQ
        assert err[qn, False, "o"] > err[qn, True, "o"]
    for ks in (True, False):
        assert err[False, ks, "o"] > err[True, ks, "o"]  # QK-norm helps too
    for n in ("o", "dq", "dk", "dv"):
        assert cos[True, True, n] >= 0.995, n


# ------------------------------------------------------------------------------------------
# Q-smoothing
# ------------------------------------------------------------------------------------------
def _q_outlier_inputs(seed, BH=2, N=128, d=64):
    g = np.random.default_rng(seed)
    q, k, v, do = (g.standard_normal((BH, N, d)) for _ in range(4))
    mu = 4.0 * g.standard_normal((BH, 1, d))
    mu[..., [3, 17, 40, 60]] += 20.0
    q = q + mu
    k = k + 3.0 * g.standard_normal((BH, 1, d))
    return q, k, v, do


def _qsmooth_xmode_gap(causal, ksmooth, seed=21):
    """Largest relative difference of the X-mode outputs between Q-smoothing on and off."""
    q, k, v, do = _q_outlier_inputs(seed)
    kw = dict(causal=causal, qknorm=True, ksmooth=ksmooth, q_block=64, k_block=32,
              dtype="bf16", quant=False, round_outputs=False)
    on = O.sage_attention(q, k, v, do, qsmooth=True, **kw)
    off = O.sage_attention(q, k, v, do, qsmooth=False, **kw)
    return max(_rel(on[n], off[n]) for n in ("o", "lse", "dq", "dk", "dv"))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("ksmooth", [False, True])
def test_qsmooth_xmode_invariance(causal, ksmooth):
    """Q-smoothing with the score bias and dK_bias = (dS^T 1) mu_Q^T is exact in full precision:
    the scores q~_i . k_j + mu_Q . k_j equal q^_i . k_j, and dK = tau dS^T q~ + tau (dS^T 1)
    mu_Q^T = tau dS^T q^, so every output equals Q-smoothing off up to float64 rounding."""
    assert _qsmooth_xmode_gap(causal, ksmooth) < 1e-12


def test_qsmooth_xmode_vs_torch():
    q, k, v, do = _q_outlier_inputs(22)
    res = O.sage_attention(q, k, v, do, causal=True, qknorm=True, ksmooth=True, q_block=64,
                           k_block=32, dtype="bf16", quant=False, round_outputs=False,
                           qsmooth=True)
    o, lse, dq, dk, dv = _torch_reference(q, k, v, do, True, True, True)
    for a, b in ((res["o"], o), (res["lse"], lse), (res["dq"], dq), (res["dk"], dk),
                 (res["dv"], dv)):
        assert _rel(a, b) < 1e-12


def test_qsmooth_prologue_closed_forms():
    q, k, v, _ = _q_outlier_inputs(23, BH=3, N=256, d=128)
    q, k, v = (x.astype(np.float32) for x in (q, k, v))
    pro = O.prologue(q, k, v, q_block=128, k_block=64, qknorm=True, ksmooth=True, qsmooth=True)
    qh = pro["q_hat"].astype(np.float64)
    N, d = qh.shape[-2], qh.shape[-1]
    eps32 = np.finfo(np.float32).eps
    # mu_Q is the per-channel token mean: float32 summation error bound N * eps * sum|x|
    m64 = qh.mean(axis=-2)
    bound = N * eps32 * np.abs(qh).sum(axis=-2) / N + eps32 * np.abs(m64)
    assert np.all(np.abs(pro["q_mean"] - m64) <= bound)
    # smoothed Q has (nearly) zero channel means; the offset channels are removed
    assert np.abs(pro["q_tilde"].astype(np.float64).mean(axis=-2)).max() < 1e-4
    assert np.abs(pro["q_tilde"]).max() < np.abs(pro["q_hat"]).max()
    # k_bias_j = mu_Q . k~_j within the float32 dot-product bound d * eps * sum|m k|
    kt = pro["k_tilde"].astype(np.float64)
    mq = pro["q_mean"].astype(np.float64)
    b64 = np.einsum("bnc,bc->bn", kt, mq)
    bb = d * eps32 * np.einsum("bnc,bc->bn", np.abs(kt), np.abs(mq))
    assert np.all(np.abs(pro["k_bias"] - b64) <= bb)
    # the Q codes are those of the smoothed Q
    c, s = O.quantize_token_blocks(pro["q_tilde"], 128)
    assert np.array_equal(c, pro["q_codes"]) and np.array_equal(s, pro["q_scale"])


def test_qsmooth_qmode_scores_closer_and_cosine():
    """With large per-channel Q offsets, Q-smoothing makes the INT8 scores (plus bias) closer
    to the full-precision scores; the whole operator stays within cosine 0.995 of X mode."""
    q, k, v, do = _q_outlier_inputs(24, BH=2, N=256, d=64)
    q, k, v, do = (x.astype(np.float32) for x in (q, k, v, do))
    tau = 1.0 / 8.0
    errs = {}
    for qs in (False, True):
        pro = O.prologue(q, k, v, q_block=128, k_block=64, qknorm=True, ksmooth=True,
                         qsmooth=qs)
        exact = np.einsum("bic,bjc->bij", pro["q_hat"].astype(np.float64),
                          pro["k_tilde"].astype(np.float64)) * tau
        err = 0.0
        for h in range(q.shape[0]):
            sq = np.repeat(pro["q_scale"][h].astype(np.float64), 128)
            sk = np.repeat(pro["k_scale"][h].astype(np.float64), 64)
            z = O._scores(pro["q_codes"][h].astype(np.float64), sq,
                          pro["k_codes"][h].astype(np.float64), sk, tau, False, 0,
                          pro["k_bias"][h] if qs else None)
            err += float(np.linalg.norm(z - exact[h]) ** 2)
        errs[qs] = math.sqrt(err)
    assert errs[True] < 0.5 * errs[False], errs
    kw = dict(causal=True, qknorm=True, ksmooth=True, q_block=128, k_block=64, dtype="bf16",
              qsmooth=True)
    qm = O.sage_attention(q, k, v, do, **kw)
    xm = O.sage_attention(q, k, v, do, quant=False, round_outputs=False, **kw)
    for n in ("o", "dq", "dk", "dv"):
        assert _cos(qm[n], xm[n]) >= 0.995, n


# ------------------------------------------------------------------------------------------
# planted mistakes are caught
# ------------------------------------------------------------------------------------------
def _xmode_vs_torch_ok():
    try:
        test_xmode_vs_torch_sdpa(True, True, True)
        return True
    except AssertionError:
        return False


def test_planted_mistakes_are_caught(monkeypatch):
    assert _xmode_vs_torch_ok()
    real_bwd = O.attn_bwd_head

    def wrong_sign_ds(*a, **kw):  # dS = P (D - dP)
        dq, dk, dv = real_bwd(*a, **kw)
        return -dq, -dk, dv

    def transposed_dv(*a, **kw):
        dq, dk, dv = real_bwd(*a, **kw)
        return dq, dk, dv[::-1]

    real_scores = O._scores

    def dropped_tau(qc, sq, kc, sk, tau, causal, i0, k_bias=None):
        return real_scores(qc, sq, kc, sk, 1.0, causal, i0, k_bias)

    for name, fake in (("attn_bwd_head", wrong_sign_ds), ("attn_bwd_head", transposed_dv),
                       ("_scores", dropped_tau)):
        with monkeypatch.context() as m:
            m.setattr(O, name, fake)
            assert not _xmode_vs_torch_ok(), name
    # Q-smoothing: a dropped dK correction term, or a bias with the wrong sign
    def no_dk_bias(*a, **kw):
        kw["q_mean"] = None
        return real_bwd(*a, **kw)

    real_fwd = O.attn_fwd_head

    def neg_bias_fwd(*a, **kw):
        if kw.get("k_bias") is not None:
            kw["k_bias"] = -kw["k_bias"]
        return real_fwd(*a, **kw)

    for name, fake in (("attn_bwd_head", no_dk_bias), ("attn_fwd_head", neg_bias_fwd)):
        with monkeypatch.context() as m:
            m.setattr(O, name, fake)
            assert _qsmooth_xmode_gap(True, True) > 1e-6, name
    real_quant = O.quantize_groups

    def round_half_up(x, axes):
        c, s = real_quant(x, axes)
        x = np.asarray(x, np.float32)
        safe = np.where(s > 0, s, 1)
        return np.clip(np.floor(x / safe + 0.5), -127, 127).astype(np.int8), s

    with monkeypatch.context() as m:
        m.setattr(O, "quantize_groups", round_half_up)
        with pytest.raises(AssertionError):
            test_quantize_golden(0)

"""Pins of the NVFP4 Q-Attn oracle against facts fixed outside it.

* E2M1 / E4M3 decoding from the bit formats (sign, exponent bias, subnormals) and, for E4M3,
  torch's own float8_e4m3fn conversion (a library routine);
* rounding checked by brute force against the whole representable grid (nearest, ties to the
  even code, saturation);
* NVFP4 quantization: exact round trip of values planted on the grid, the per-element error
  bound, exact invariance under power-of-two scaling, the global scale's placement;
* the forward: torch's float64 scaled-dot-product attention and logsumexp on the same
  dequantized operands, and the end-to-end wiring on inputs that quantize exactly.

Planted mistakes (at the end) check that these pins catch plausible slips in the oracle.
"""
import numpy as np
import pytest
import torch

import oracle.nvfp4_oracle as F
import oracle.sage_oracle as S8

# ------------------------------------------------------------------------------------------
# E2M1
# ------------------------------------------------------------------------------------------


def _e2m1_from_bits(c):
    """E2M1 from its bit fields: 1 sign, 2 exponent (bias 1), 1 mantissa bit."""
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_decode_matches_bit_format():
    for c in range(16):
        assert F.e2m1_decode(np.array([c], np.uint8))[0] == _e2m1_from_bits(c)


def _e2m1_brute(y):
    """Nearest grid magnitude, ties to the even code, above 6 -> 6; the sign bit is y's."""
    a = abs(float(y))
    if a >= 6.0:
        mag = 7
    else:
        d = np.abs(F.E2M1_VALUES - a)
        best = np.flatnonzero(d == d.min())
        mag = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    return mag | (8 if np.signbit(np.float32(y)) else 0)


def test_e2m1_encode_brute_force():
    ys = np.concatenate([np.arange(-8.0, 8.0, 1.0 / 64.0),
                         [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 1e30, -1e30,
                          -0.0, 0.1, -0.1]]).astype(np.float32)
    got = F.e2m1_encode(ys)
    want = np.array([_e2m1_brute(y) for y in ys], np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_ties_and_saturation():
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    assert F.e2m1_decode(F.e2m1_encode(ties)).tolist() == [0, 1, 1, 2, 2, 4, 4]
    assert F.e2m1_encode(np.array([7.0, 100.0, -6.5], np.float32)).tolist() == [7, 7, 15]
    # rounding to zero keeps the sign, as IEEE rounding does
    assert F.e2m1_encode(np.array([0.1, -0.1, 0.0, -0.0], np.float32)).tolist() == [0, 8, 0, 8]


# ------------------------------------------------------------------------------------------
# E4M3
# ------------------------------------------------------------------------------------------
def _e4m3_torch(codes):
    t = torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_decode_matches_torch():
    codes = np.arange(0, 127, dtype=np.uint8)  # every non-negative finite code (0x7F is NaN)
    assert np.array_equal(F.e4m3_decode(codes), _e4m3_torch(codes))
    assert F.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert F.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert F.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert F.e4m3_decode(np.array([0x38]))[0] == 1.0


def test_e4m3_encode_grid_midpoints_and_torch():
    codes = np.arange(0, 127, dtype=np.uint8)
    vals = F.e4m3_decode(codes)
    # every representable value maps to its own code
    assert np.array_equal(F.e4m3_encode(vals.astype(np.float32)), codes)
    # midpoints go to the neighbour with the even code
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)  # exact in float32
    got = F.e4m3_encode(mids)
    lo = codes[:-1]
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want)
    # random values below 448: torch's round-to-nearest-even conversion
    rng = np.random.default_rng(5)
    u = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(-14, 6, 20000)),
                        rng.uniform(0, 2.0 ** -6, 5000)]).astype(np.float32)
    u = u[u < 448]
    t = torch.tensor(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(u), t)
    # saturation
    assert F.e4m3_encode(np.array([448.0, 460.0, 1e9], np.float32)).tolist() == [0x7E] * 3


# ------------------------------------------------------------------------------------------
# NVFP4 quantization
# ------------------------------------------------------------------------------------------
def _planted(seed, BH=2, N=64, d=128):
    """Values exactly on the NVFP4 grid with a global maximum of 2688 (so genc = 1): every
    block has a largest code of magnitude 6, so the block scale is recovered exactly."""
    rng = np.random.default_rng(seed)
    nb = d // 16
    codes = rng.integers(0, 16, size=(BH, N, nb, 16)).astype(np.uint8)
    pos = rng.integers(0, 16, size=(BH, N, nb))
    sgn = rng.integers(0, 2, size=(BH, N, nb)).astype(np.uint8) << 3
    np.put_along_axis(codes, pos[..., None], (7 | sgn)[..., None], axis=-1)
    sf = rng.integers(1, 0x7F, size=(BH, N, nb)).astype(np.uint8)
    sf[:, 0, 0] = 0x7E  # 448: the block holding the global maximum 6 * 448
    x = F.e2m1_decode(codes) * F.e4m3_decode(sf)[..., None]
    return x.reshape(BH, N, d).astype(np.float32), codes.reshape(BH, N, d), sf


def test_nvfp4_planted_round_trip():
    x, codes, sf = _planted(1)
    assert np.all(np.abs(x).max(axis=(1, 2)) == 2688.0)
    r = F.nvfp4_quantize(x)
    assert np.all(r["genc"] == 1.0)
    assert np.array_equal(r["sf"], sf)
    # every planted code comes back, -0 (code 8) included
    assert np.array_equal(r["codes"], codes)
    assert np.array_equal(F.nvfp4_dequantize(r["codes"], r["sf"], r["genc"]), x)


def test_nvfp4_error_bound_and_global_scale():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 256, 128)) * np.exp(rng.uniform(-3, 3, (3, 1, 128)))).astype(np.float32)
    r = F.nvfp4_quantize(x)
    G = np.abs(x).max(axis=(1, 2))
    assert np.array_equal(r["genc"], (np.float32(2688.0) / G.astype(np.float32)))
    sd = F.e4m3_decode(r["sf"])
    xd = F.nvfp4_dequantize(r["codes"], r["sf"], r["genc"])
    err = np.abs(xd - x).reshape(3, 256, 8, 16).max(axis=-1)
    # scaled values stay within 6 (1 + 2^-4) and the E2M1 grid spacing is at most 2, so the
    # error is at most one scaled unit, sd / genc, wherever the block scale is a normal E4M3
    normal = sd >= 2.0 ** -6
    bound = sd / r["genc"][:, None, None].astype(np.float64) * (1 + 1e-6)
    assert np.all(err[normal] <= bound[normal])
    assert normal.mean() > 0.99
    # the element holding the global maximum is coded +-6 with the largest scale
    for h in range(3):
        n, c = np.unravel_index(np.argmax(np.abs(x[h])), x[h].shape)
        assert r["sf"][h, n, c // 16] == 0x7E and (r["codes"][h, n, c] & 7) == 7


def test_nvfp4_power_of_two_invariance():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 128, 64)).astype(np.float32)
    r0 = F.nvfp4_quantize(x)
    for k in (-7, -1, 3, 11):
        r = F.nvfp4_quantize((x * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(r["codes"], r0["codes"]) and np.array_equal(r["sf"], r0["sf"])
        assert np.array_equal(r["genc"], (r0["genc"] * np.float32(2.0 ** -k)).astype(np.float32))


def test_nvfp4_zero_matrix():
    r = F.nvfp4_quantize(np.zeros((1, 32, 64), np.float32))
    assert np.all(r["genc"] == 1.0) and not r["sf"].any() and not r["codes"].any()


# ------------------------------------------------------------------------------------------
# Q-Attn forward
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_qattn_fwd_head_vs_torch(causal):
    rng = np.random.default_rng(4)
    N, d = 96, 64
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    tau = 0.3
    o, lse, w = F.qattn_fwd_head(q, k, v, causal=causal, tau=tau)
    t = [torch.tensor(a)[None, None] for a in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=causal, scale=tau)
    assert np.allclose(o, ref[0, 0].numpy(), rtol=1e-12, atol=1e-12)
    z = torch.tensor(q) @ torch.tensor(k).T * tau
    if causal:
        z = z.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    assert np.allclose(lse, torch.logsumexp(z, dim=1).numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(w >= np.abs(o) - 1e-12)


def test_qattn_forward_exact_inputs_equal_plain_attention():
    """Without QK-norm and smoothing, inputs on the NVFP4 grid dequantize to themselves, so
    the Q-Attn forward is plain attention of the inputs."""
    x, _, _ = _planted(6, BH=2, N=64, d=64)
    y, _, _ = _planted(7, BH=2, N=64, d=64)
    q, k = x / np.float32(512.0), y / np.float32(256.0)  # powers of two keep them on the grid
    v = np.random.default_rng(8).standard_normal((2, 64, 64)).astype(np.float32)
    tau = 1.0 / 512.0
    r = F.qattn_forward(q, k, v, causal=True, qknorm=False, ksmooth=False, tau=tau)
    assert np.array_equal(r["q_deq"], q.astype(np.float64))
    assert np.array_equal(r["k_deq"], k.astype(np.float64))
    t = [torch.tensor(a.astype(np.float64)) for a in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True, scale=tau)
    assert np.allclose(r["o"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_qattn_forward_close_to_full_precision():
    rng = np.random.default_rng(9)
    BH, N, d = 2, 256, 128
    q, k, v = (rng.standard_normal((BH, N, d)).astype(np.float32) for _ in range(3))
    k += 3.0 * rng.standard_normal((BH, 1, d)).astype(np.float32)  # channel offsets on K
    r = F.qattn_forward(q, k, v, causal=True, qknorm=True, ksmooth=True)
    t = [torch.tensor(a.astype(np.float64)) for a in (r["q_hat"], r["k_tilde"], v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True).numpy()
    cos = (r["o"] * ref).sum() / np.sqrt((r["o"] ** 2).sum() * (ref ** 2).sum())
    assert cos > 0.99, cos


# ------------------------------------------------------------------------------------------
# planted mistakes are caught
# ------------------------------------------------------------------------------------------
def _fails(test, *args):
    try:
        test(*args)
        return False
    except AssertionError:
        return True


def test_planted_mistakes_are_caught(monkeypatch):
    assert not _fails(test_e2m1_encode_brute_force)
    real_e2m1 = F.e2m1_encode

    def ties_up(y):  # ties away from zero instead of to even
        a = np.abs(np.asarray(y, np.float32))
        mag = ((a >= 0.25).astype(np.uint8) + (a >= 0.75) + (a >= 1.25) + (a >= 1.75)
               + (a >= 2.5) + (a >= 3.5) + (a >= 5.0)).astype(np.uint8)
        return (mag | (np.signbit(np.asarray(y, np.float32)).astype(np.uint8) << 3)).astype(np.uint8)

    with monkeypatch.context() as m:
        m.setattr(F, "e2m1_encode", ties_up)
        assert _fails(test_e2m1_encode_brute_force)

    real_e4m3 = F.e4m3_encode

    def truncating(u):  # rounds toward zero
        u = np.asarray(u, np.float32).astype(np.float64)
        codes = np.arange(0, 127, dtype=np.uint8)
        vals = F.e4m3_decode(codes)
        idx = np.searchsorted(vals, u, side="right") - 1
        return codes[np.clip(idx, 0, 126)]

    with monkeypatch.context() as m:
        m.setattr(F, "e4m3_encode", truncating)
        assert _fails(test_e4m3_encode_grid_midpoints_and_torch)

    real_q = F.nvfp4_quantize

    def no_global(x):  # global scale left out of the block scale
        r = real_q(x)
        r2 = real_q(x / np.maximum(np.abs(x).max(axis=(-2, -1), keepdims=True), 1e-30) * 2688.0)
        r2["genc"] = np.ones_like(r["genc"])
        return r2

    def sf_transposed(x):  # scale of block b taken from block (nb - 1 - b)
        r = real_q(x)
        r["sf"] = r["sf"][..., ::-1].copy()
        return r

    for fake, test in ((no_global, test_nvfp4_error_bound_and_global_scale),
                       (no_global, test_nvfp4_power_of_two_invariance),
                       (sf_transposed, test_nvfp4_planted_round_trip),
                       (sf_transposed, test_nvfp4_error_bound_and_global_scale)):
        with monkeypatch.context() as m:
            m.setattr(F, "nvfp4_quantize", fake)
            assert _fails(test), (fake.__name__, test.__name__)

    real_head = F.qattn_fwd_head

    def dropped_tau(qd, kd, v, *, causal, tau):
        return real_head(qd, kd, v, causal=causal, tau=1.0)

    with monkeypatch.context() as m:
        m.setattr(F, "qattn_fwd_head", dropped_tau)
        assert _fails(test_qattn_forward_exact_inputs_equal_plain_attention)
    assert F.e2m1_encode is real_e2m1 and F.e4m3_encode is real_e4m3


# ------------------------------------------------------------------------------------------
# Backward
# ------------------------------------------------------------------------------------------
def _torch_grads(q, k, v, do, causal, qknorm, ksmooth, tau=None):
    t = [torch.tensor(a.astype(np.float64), requires_grad=True) for a in (q, k, v)]
    qq, kk = t[0], t[1]
    if qknorm:
        qq = qq * torch.rsqrt((qq * qq).mean(-1, keepdim=True) + 1e-6)
        kk = kk * torch.rsqrt((kk * kk).mean(-1, keepdim=True) + 1e-6)
    if ksmooth:
        kk = kk - kk.mean(-2, keepdim=True)
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, t[2], is_causal=causal,
                                                         scale=tau)
    o.backward(torch.tensor(do.astype(np.float64)))
    return o.detach().numpy(), [g.grad.numpy() for g in t]


@pytest.mark.parametrize("causal,qknorm,ksmooth", [(True, True, True), (False, False, False),
                                                   (True, False, True), (False, True, False)])
def test_qattn_bwd_full_precision_vs_torch_autograd(causal, qknorm, ksmooth):
    rng = np.random.default_rng(21)
    q, k, v, do = (rng.standard_normal((2, 256, 64)).astype(np.float32) for _ in range(4))
    k += 2.0 * rng.standard_normal((2, 1, 64)).astype(np.float32)
    r = F.qattn_attention(q, k, v, do, causal=causal, qknorm=qknorm, ksmooth=ksmooth,
                          quant=False)
    o, grads = _torch_grads(q, k, v, do, causal, qknorm, ksmooth)
    assert np.allclose(r["o"], o, rtol=0, atol=1e-12)
    for name, g in zip(("dq", "dk", "dv"), grads):
        assert np.allclose(r[name], g, rtol=0, atol=1e-11), name


def _quant_tile_brute(t, axis):
    """Per-tile NVFP4 of a float32 tile, element loops (blocks of 16 along `axis`)."""
    G = float(np.max(np.abs(t)))
    genc = np.float32(2688.0) / np.float32(G) if G > 0 else np.float32(1.0)
    out = np.zeros(t.shape, np.float64)
    tt = t if axis == 1 else t.T
    res = np.zeros(tt.shape, np.float64)
    for r in range(tt.shape[0]):
        for b0 in range(0, tt.shape[1], 16):
            blk = tt[r, b0:b0 + 16]
            a = np.float32(np.max(np.abs(blk)))
            u = np.float32(np.float32(a * genc) / np.float32(6.0))
            sd = np.float32(F.e4m3_decode(F.e4m3_encode(np.array([u], np.float32)))[0])
            mult = np.float32(genc / sd) if sd > 0 else np.float32(0.0)
            for c in range(16):
                code = F.e2m1_encode(np.array([np.float32(blk[c] * mult)], np.float32))[0]
                res[r, b0 + c] = F.e2m1_decode(np.array([code]))[0] * float(sd) / float(genc)
    out[:] = res if axis == 1 else res.T
    return out


def test_qattn_bwd_tile_quantizer_brute_force():
    rng = np.random.default_rng(22)
    t = (rng.standard_normal((128, 128)) * np.exp(rng.uniform(-4, 2, (128, 1)))).astype(np.float32)
    for axis in (0, 1):
        assert np.array_equal(F.nvfp4_quantize_tile(t, axis), _quant_tile_brute(t, axis)), axis


def test_qattn_bwd_quantized_products_brute_force():
    """One 128-key tile, d = 32: dQ and dK from explicit sums over the brute-force quantized
    dS (16-key blocks for dQ, 16-query blocks for dK) and the sequence views."""
    rng = np.random.default_rng(23)
    N, d, tau = 128, 32, 0.25
    q, k, v, do = (rng.standard_normal((1, N, d)).astype(np.float32) for _ in range(4))
    r = F.qattn_attention(q, k, v, do, causal=True, qknorm=False, ksmooth=False, tau=tau)
    z = (r["q_deq"][0] @ r["k_deq"][0].T) * tau
    z = np.where(np.arange(N)[None, :] > np.arange(N)[:, None], -np.inf, z)
    P = np.exp(z - r["lse"][0][:, None])
    dS = P * (do[0].astype(np.float64) @ v[0].T.astype(np.float64)
              - (do[0] * r["o"][0]).sum(1)[:, None])
    dS32 = dS.astype(np.float32)
    dSk, dSq = _quant_tile_brute(dS32, 1), _quant_tile_brute(dS32, 0)
    dq = np.zeros((N, d))
    dk = np.zeros((N, d))
    for i in range(N):
        for j in range(N):
            dq[i] += dSk[i, j] * r["k_seq"][0][j]
            dk[j] += dSq[i, j] * r["q_seq"][0][i]
    assert np.allclose(r["dq"][0], dq * tau, rtol=1e-12, atol=1e-12)
    assert np.allclose(r["dk"][0], dk * tau, rtol=1e-12, atol=1e-12)
    assert np.allclose(r["dv"][0], P.T @ do[0].astype(np.float64), rtol=1e-12, atol=1e-12)


def test_qattn_bwd_close_to_full_precision():
    rng = np.random.default_rng(24)
    q, k, v, do = (rng.standard_normal((2, 256, 128)).astype(np.float32) for _ in range(4))
    k += 3.0 * rng.standard_normal((2, 1, 128)).astype(np.float32)
    kw = dict(causal=True, qknorm=True, ksmooth=True)
    qm = F.qattn_attention(q, k, v, do, **kw)
    xm = F.qattn_attention(q, k, v, do, quant=False, **kw)
    cos = lambda a, b: (a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum())  # noqa: E731
    for n in ("o", "dq", "dk", "dv"):
        assert cos(qm[n], xm[n]) > 0.98, n


def test_qattn_bwd_planted_mistakes_are_caught(monkeypatch):
    real_tile = F.nvfp4_quantize_tile

    def wrong_axis(x, axis):  # dS quantized along the other axis
        return real_tile(x, 1 - axis)

    with monkeypatch.context() as m:
        m.setattr(F, "nvfp4_quantize_tile", wrong_axis)
        assert _fails(test_qattn_bwd_quantized_products_brute_force)
    real_bwd = F.qattn_bwd_head

    def dropped_tau_dk(*a, **kw):
        dq, dk, dv = real_bwd(*a, **kw)
        return dq, dk / kw["tau"], dv

    def transposed_ds(*a, **kw):
        dq, dk, dv = real_bwd(*a, **kw)
        return dq, dk[::-1], dv

    for fake in (dropped_tau_dk, transposed_ds):
        with monkeypatch.context() as m:
            m.setattr(F, "qattn_bwd_head", fake)
            assert _fails(test_qattn_bwd_full_precision_vs_torch_autograd, True, True, True)


def test_qattn_attention_storage_rounding():
    """dtype="bf16": O is stored (rounded) before the backward reads it, and the gradients are
    rounded at the end; the stored O changes D = rowsum(dO o O) and so the gradients."""
    rng = np.random.default_rng(5)
    q, k, v, do = (rng.standard_normal((1, 128, 64)).astype(np.float32) for _ in range(4))
    kw = dict(causal=True, qknorm=False, ksmooth=False)
    plain = F.qattn_attention(q, k, v, do, **kw)
    st = F.qattn_attention(q, k, v, do, dtype="bf16", **kw)
    bf = lambda a: np.asarray(a, np.float32).view(np.uint32) & 0xFFFF  # noqa: E731
    for n in ("o", "dq", "dk", "dv"):
        assert (bf(st[n]) == 0).all(), n  # bf16 values
    np.testing.assert_array_equal(st["o"], S8.round_to_storage(plain["o"], "bf16"))
    np.testing.assert_array_equal(st["dv"], S8.round_to_storage(plain["dv"], "bf16"))  # no D
    D_plain = (do[0] * plain["o"][0]).sum(1)
    D_st = (do[0] * st["o"][0]).sum(1)
    assert np.abs(D_plain - D_st).max() > 0
    assert not np.array_equal(st["dq"], S8.round_to_storage(plain["dq"], "bf16"))

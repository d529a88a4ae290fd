"""Degenerate inputs through the whole CUDA path, against the oracle and closed forms.

* all-zero q, k, v, dO: every block scale is 0 and every code 0 (the absmax = 0 rule), the
  attention is uniform, O = 0 and every gradient is 0;
* identical keys with K-smoothing: smoothed K is exactly 0, so the scores vanish and O is the
  running mean of V (causal) -- the closed form the oracle is also pinned to;
* large magnitudes (|x| ~ 1e3, bf16): the quantization is scale-invariant, so parity holds;
* tiny gradients (dO ~ 2^-100) and key blocks whose probabilities -- and so the backward's P and
  dS tile maxima -- lie in float32's subnormal range: every output stays finite and parity
  holds (the code multipliers 127 / max are IEEE quotients; the NVFP4 page on Quartet II
  reports an approximate reciprocal that flushed subnormals to zero and produced NaN).
"""
import numpy as np
import pytest
import torch

from fwd_bwd_b200.inputs import WORKLOADS, bits_to_f32, f32_to_bits, make_inputs

from gpu_helpers import cosine, gpu_run, oracle_run, rel_l2

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["sweep8192"].replace(B=1, H=2, N=384)


def _with(x, w, **arrays):
    for name, arr in arrays.items():
        bits = f32_to_bits(np.ascontiguousarray(arr, np.float32), w.dtype)
        x[name] = bits
        x[name + "_f32"] = bits_to_f32(bits, w.dtype)
    return x


def test_all_zero_inputs():
    w = BASE
    z = np.zeros((w.B, w.H, w.N, w.d), np.float32)
    x = _with(make_inputs(w), w, q=z, k=z, v=z, do=z)
    g = gpu_run(w, x)
    for n in ("q_scale", "k_scale", "v_scale"):
        assert np.all(g[n] == 0), n
    for n in ("q_codes", "k_codes", "v_codes"):
        assert np.all(g[n] == 0), n
    for n in ("o", "dq", "dk", "dv"):
        assert np.all(g[n] == 0), n
    # LSE of a uniform row over the j + 1 visible keys (causal): ln(j + 1)
    lse = g["lse"].reshape(w.B * w.H, w.N)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, w.N + 1)), lse.shape),
                               rtol=0, atol=1e-5)


def test_identical_keys_give_running_mean():
    w = BASE.replace(qknorm=False)
    x = make_inputs(w)
    g0 = np.random.default_rng(3)
    krow = g0.integers(-8, 9, (w.B, w.H, 1, w.d)).astype(np.float32)
    x = _with(x, w, k=np.repeat(krow, w.N, axis=2))
    g = gpu_run(w, x)
    o = oracle_run(w, x)
    assert np.all(g["k_codes"] == 0)
    v = x["v_f32"].reshape(w.B * w.H, w.N, w.d).astype(np.float64)
    mean_v = np.cumsum(v, axis=1) / np.arange(1, w.N + 1)[None, :, None]
    # O is a (quantized-V) running mean: compare with the oracle tightly, with V loosely
    assert rel_l2(g["o"].reshape(v.shape), o["o"]) <= 2e-3
    assert cosine(g["o"].reshape(v.shape), mean_v) >= 0.999
    assert np.all(g["dq"] == 0)  # dS K with all-zero K codes, then the RMSNorm-free finalize


@pytest.mark.parametrize("case", ["large_v_do", "large_qk_normed", "tiny_all"])
def test_extreme_magnitudes(case):
    """Quantization is scale-invariant, so parity holds across magnitudes -- as long as the
    logits stay in the range a float32 LSE resolves (QK-norm's purpose; large raw q, k without
    it give logits ~1e7 where one float32 ulp of the LSE is ~1)."""
    w = BASE.replace(qknorm=False, ksmooth=False)
    x = make_inputs(w)
    if case == "large_v_do":
        x = _with(x, w, v=x["v_f32"] * 1e3, do=x["do_f32"] * 1e3)
    elif case == "large_qk_normed":
        w = w.replace(qknorm=True)
        x = _with(x, w, q=x["q_f32"] * 1e3, k=x["k_f32"] * 1e3)
    else:
        x = _with(x, w, **{n: x[n + "_f32"] * 1e-3 for n in ("q", "k", "v", "do")})
    g = gpu_run(w, x)
    o = oracle_run(w, x)
    BH = w.B * w.H
    for n in ("o", "dq", "dk", "dv"):
        assert rel_l2(g[n].reshape(BH, w.N, w.d), o[n]) <= 2e-3, n


def test_tiny_gradients():
    """dO ~ 2^-100 (bf16 keeps float32's exponent range): the dS and dO scales are ~2^-107,
    their products with the Q / K / P scales stay normal floats, and parity holds."""
    w = BASE.replace(qknorm=False, ksmooth=False)
    x = make_inputs(w)
    x = _with(x, w, do=x["do_f32"] * 2.0 ** -100)
    g = gpu_run(w, x)
    o = oracle_run(w, x)
    BH = w.B * w.H
    for n in ("o", "dq", "dk", "dv"):
        assert np.all(np.isfinite(g[n])), n
        assert rel_l2(g[n].reshape(BH, w.N, w.d), o[n]) <= 2e-3, n


def test_subnormal_tile_maxima():
    """Channel 0 of every query is +30 and key blocks 1, 3 and 5 have channel 0 at -33.5, so their
    scores sit ~89 below the rows' maxima: P ~ e^-89 and dS there are float32 subnormals, and so
    are those tiles' maxima.  Outputs must stay finite and match the oracle (the tiles below
    2^-121 contribute only ~1e-38 to any output)."""
    w = BASE.replace(qknorm=False, ksmooth=False, causal=False)
    x = make_inputs(w)
    q = x["q_f32"].copy()
    k = x["k_f32"].copy()
    q[..., 0] = 30.0
    for blk in (1, 3, 5):
        k[..., blk * 64:(blk + 1) * 64, 0] = -33.5
    x = _with(x, w, q=q, k=k)
    g = gpu_run(w, x)
    o = oracle_run(w, x)
    BH = w.B * w.H
    # the case is what it claims: the far blocks' probabilities are subnormal in float32
    z = np.einsum("hnd,hmd->hnm", q.reshape(BH, w.N, w.d).astype(np.float64),
                  k.reshape(BH, w.N, w.d).astype(np.float64)) / np.sqrt(w.d)
    p = np.exp(z - o["lse"][:, :, None])
    far = p[:, :, 64:128]
    assert far.max() < 1.1754944e-38 and far.max() > 1e-44
    for n in ("o", "dq", "dk", "dv"):
        assert np.all(np.isfinite(g[n])), n
        assert rel_l2(g[n].reshape(BH, w.N, w.d), o[n]) <= 2e-3, n

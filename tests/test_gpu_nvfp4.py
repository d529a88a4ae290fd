"""NVFP4 Q-Attn parity: the CUDA path against the NVFP4 oracle on the same seeded inputs.

* Prologue: E2M1 codes, E4M3 block scales, global scales, inverse RMS and K means bit-exact
  (every quantization decision is a correctly rounded float32 step on both sides).
* Forward: O and LSE element by element.  The kernel rounds P to the 16-bit type of V before
  P V (the tensor-core operand precision) while the oracle keeps P exact; with
  W = sum_j p_j |v_j| / l that rounding moves O by at most u16 * W (u16 = 2^-8 for bf16,
  2^-11 for fp16, relative half-ulp), the 16-bit output rounding by u16 |O|, and the FP32
  accumulation of S and PV and the exp2 approximation by far less.  The test allows twice
  those bounds plus 1e-5 W.  LSE depends only on FP32 sums: |dLSE| <= 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle.nvfp4_oracle as F
from fwd_bwd_b200 import nvfp4, ops
from fwd_bwd_b200.inputs import WORKLOADS

from gpu_helpers import to_device
from fwd_bwd_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["sweep8192"]
CASES = {
    "d128_bf16_causal": BASE.replace(B=1, H=3, N=384),
    "d128_bf16_full": BASE.replace(B=1, H=2, N=256, causal=False),
    "d128_fp16_causal": BASE.replace(B=2, H=1, N=512, dtype="fp16"),
    "d64_bf16_causal": WORKLOADS["llama325m"].replace(B=1, H=3, N=384),
    "d64_fp16_full": WORKLOADS["llama325m"].replace(B=1, H=2, N=256, dtype="fp16",
                                                   causal=False),
    "koutlier_norm_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=256, qknorm=False),
    "koutlier_all_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=384, qknorm=False,
                                                     ksmooth=False),
    "single_tile": BASE.replace(B=1, H=1, N=128),
}


def _cfg(w):
    return ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                      k_block=w.k_block)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[..., d/2] bytes -> [..., d] 4-bit codes (channel 2i in the low nibble of byte i)."""
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = packed & 15
    out[..., 1::2] = packed >> 4
    return out


def unpack_sf(sf: np.ndarray, N: int, d: int) -> np.ndarray:
    """[BH, N/128, d/64, 512] scale atoms -> [BH, N, d/16] (row r, 16-channel block b)."""
    sf = sf.reshape(-1, N // 128, d // 64, 512)
    BH = sf.shape[0]
    r = np.arange(128)
    b = np.arange(4)
    idx = (r[:, None] % 32) * 16 + (r[:, None] // 32) * 4 + b[None, :]  # [128, 4]
    t = sf[..., idx]  # [BH, N/128, d/64, 128, 4]
    return t.transpose(0, 1, 3, 2, 4).reshape(BH, N, d // 16)


def _run(w):
    x = make_inputs(w)
    q, k, v = (to_device(x[n], w.dtype) for n in ("q", "k", "v"))
    cfg = _cfg(w)
    fb = nvfp4.quant_prologue(q, k, cfg)
    o, lse = nvfp4.attn_fwd(fb, v, cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    return x, fb, o, lse


@pytest.mark.parametrize("name", list(CASES))
def test_nvfp4_prologue_and_forward(name):
    w = CASES[name]
    BH, N, d = w.B * w.H, w.N, w.d
    x, fb, o, lse = _run(w)
    qf, kf, vf = (x[n + "_f32"].reshape(BH, N, d) for n in ("q", "k", "v"))
    ref = F.qattn_forward(qf, kf, vf, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth)
    for t in ("q", "k"):
        codes = unpack_codes(getattr(fb, t + "_fp4").cpu().numpy().reshape(BH, N, d // 2))
        np.testing.assert_array_equal(codes, ref[t + "_codes"], err_msg=t + " codes")
        sf = unpack_sf(getattr(fb, t + "_sf").cpu().numpy(), N, d)
        np.testing.assert_array_equal(sf, ref[t + "_sf"], err_msg=t + " scales")
        np.testing.assert_array_equal(getattr(fb, t + "_genc").cpu().numpy().reshape(BH),
                                      ref[t + "_genc"], err_msg=t + " genc")
        if w.qknorm:
            np.testing.assert_array_equal(
                getattr(fb, t + "_inv_rms").cpu().numpy().reshape(BH, N), ref[t + "_inv_rms"])
    if w.ksmooth:
        np.testing.assert_array_equal(fb.k_mean.cpu().numpy().reshape(BH, d), ref["k_mean"])
    u16 = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -11
    og = o.float().cpu().numpy().astype(np.float64).reshape(BH, N, d)
    err = np.abs(og - ref["o"])
    tol = 2 * u16 * (ref["w"] + np.abs(ref["o"])) + 1e-5 * ref["w"] + 1e-7
    bad = err > tol
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside; worst excess "
                           f"{(err - tol).max():.3g}; max err {err.max():.3g}")
    lg = lse.cpu().numpy().astype(np.float64).reshape(BH, N)
    np.testing.assert_allclose(lg, ref["lse"], rtol=0, atol=1e-4)


def test_nvfp4_unsupported_qsmooth():
    w = CASES["single_tile"]
    x = make_inputs(w)
    q, k = (to_device(x[n], w.dtype) for n in ("q", "k"))
    cfg = _cfg(w)
    cfg.qsmooth = True
    with pytest.raises(Exception, match="UNSUPPORTED"):
        nvfp4.quant_prologue(q, k, cfg)


FULL = {
    "sweep8192": [0, 511],   # the bench workload: B32 H16 N8192 d128 causal bf16
    "llama325m": [0, 127],   # B8 H16 N2048 d64 causal bf16
}


@pytest.mark.parametrize("name", sorted(FULL))
def test_nvfp4_full_size_sampled_heads(name):
    """The whole batch in the launch configuration bench.py --variant nvfp4 times; sampled
    (batch, head) pairs carry the seeded per-head inputs and are checked one head at a time
    (each head is independent: its global scales, codes and outputs depend on it alone)."""
    w = WORKLOADS[name]
    heads = FULL[name]
    dev = torch.device("cuda")
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    g = torch.Generator(device=dev).manual_seed(2)
    shape = (w.B * w.H, w.N, w.d)
    t = {n: (torch.randn(shape, generator=g, device=dev) * w.sigma_qkv).to(dt)
         for n in ("q", "k", "v")}
    x = make_inputs(w, heads=heads)
    for n in ("q", "k", "v"):
        for i, bh in enumerate(heads):
            t[n][bh] = torch.from_numpy(x[n][i].view(np.int16)).view(dt).to(dev)
    q, k, v = (t[n].view(w.B, w.H, w.N, w.d) for n in ("q", "k", "v"))
    cfg = _cfg(w)
    fb = nvfp4.quant_prologue(q, k, cfg)
    o, lse = nvfp4.attn_fwd(fb, v, cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    N, d = w.N, w.d
    u16 = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -11
    for i, bh in enumerate(heads):
        one = [x[n + "_f32"][i:i + 1] for n in ("q", "k", "v")]
        ref = F.qattn_forward(*one, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth)
        b_, h_ = divmod(bh, w.H)
        for tname in ("q", "k"):
            codes = unpack_codes(getattr(fb, tname + "_fp4")[b_, h_].cpu().numpy())
            np.testing.assert_array_equal(codes, ref[tname + "_codes"][0], err_msg=tname)
            sf = unpack_sf(getattr(fb, tname + "_sf")[b_, h_].cpu().numpy(), N, d)
            np.testing.assert_array_equal(sf[0], ref[tname + "_sf"][0], err_msg=tname)
            assert getattr(fb, tname + "_genc")[b_, h_].item() == ref[tname + "_genc"][0]
        og = o[b_, h_].float().cpu().numpy().astype(np.float64)
        err = np.abs(og - ref["o"][0])
        tol = 2 * u16 * (ref["w"][0] + np.abs(ref["o"][0])) + 1e-5 * ref["w"][0] + 1e-7
        assert not (err > tol).any(), f"head {bh}: {(err > tol).sum()} outside"
        np.testing.assert_allclose(lse[b_, h_].cpu().numpy(), ref["lse"][0], rtol=0, atol=1e-4)


def _degenerate_inputs(kind, BH=2, N=256, d=128):
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((BH, N, d)).astype(np.float32) for _ in range(3))
    if kind == "zero_head":        # G = 0 for head 0: genc = 1, zero scales, uniform attention
        q[0] = 0.0
        k[0] = 0.0
    elif kind == "wide_range":     # rows from 2^-20 to 2^4: subnormal and zero E4M3 scales
        q *= np.exp2(rng.uniform(-20, 4, (BH, N, 1))).astype(np.float32)
        k *= np.exp2(rng.uniform(-20, 4, (BH, N, 1))).astype(np.float32)
    elif kind == "fp16_large":     # fp16 near its largest values (|x| up to ~3e4 of 65504)
        q *= 6000.0
        k *= 3000.0
    return q, k, v


@pytest.mark.parametrize("kind,dtype,qknorm", [("zero_head", "bf16", True),
                                              ("zero_head", "bf16", False),
                                              ("wide_range", "bf16", False),
                                              ("fp16_large", "fp16", False)])
def test_nvfp4_degenerate(kind, dtype, qknorm):
    q, k, v = _degenerate_inputs(kind)
    BH, N, d = q.shape
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    tq, tk, tv = (torch.from_numpy(a).to(tdt) for a in (q, k, v))
    qf, kf, vf = (t.float().numpy() for t in (tq, tk, tv))  # exact 16-bit values
    assert np.isfinite(qf).all() and np.isfinite(kf).all()
    cfg = ops.Config(causal=True, qknorm=qknorm, ksmooth=True)
    dev = torch.device("cuda")
    shape = (1, BH, N, d)
    fb = nvfp4.quant_prologue(tq.reshape(shape).to(dev), tk.reshape(shape).to(dev), cfg)
    o, lse = nvfp4.attn_fwd(fb, tv.reshape(shape).to(dev), cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    ref = F.qattn_forward(qf, kf, vf, causal=True, qknorm=qknorm, ksmooth=True)
    for t in ("q", "k"):
        codes = unpack_codes(getattr(fb, t + "_fp4").cpu().numpy().reshape(BH, N, d // 2))
        np.testing.assert_array_equal(codes, ref[t + "_codes"], err_msg=t)
        np.testing.assert_array_equal(unpack_sf(getattr(fb, t + "_sf").cpu().numpy(), N, d),
                                      ref[t + "_sf"], err_msg=t)
        np.testing.assert_array_equal(getattr(fb, t + "_genc").cpu().numpy().reshape(BH),
                                      ref[t + "_genc"], err_msg=t)
    if kind == "wide_range":  # the case exercises subnormal and zero block scales (Q is not
        # smoothed; K-smoothing lifts K's small rows to the mean's size)
        assert (ref["q_sf"] < 8).any() and (ref["q_sf"] == 0).any()
    u16 = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11
    og = o.float().cpu().numpy().astype(np.float64).reshape(BH, N, d)
    tol = 2 * u16 * (ref["w"] + np.abs(ref["o"])) + 1e-5 * ref["w"] + 1e-7
    assert not (np.abs(og - ref["o"]) > tol).any()
    # fp16_large has scores near 1e8: float32 rounding of S and of S * c is relative there
    np.testing.assert_allclose(lse.cpu().numpy().reshape(BH, N), ref["lse"], rtol=2e-6, atol=1e-4)


def unpack_sf_t(sf_t: np.ndarray, BH: int, N: int, d: int) -> np.ndarray:
    """[BH, ceil(d/128), N/64, 512] scale atoms -> [BH, d, N/16] (channel c, 16-token block)."""
    sf_t = sf_t.reshape(BH, (d + 127) // 128, N // 64, 512)
    c = np.arange(d)[:, None]
    b = np.arange(N // 16)[None, :]
    byte = (c % 32) * 16 + ((c % 128) // 32) * 4 + b % 4
    return sf_t[:, c // 128, b // 4, byte]


@pytest.mark.parametrize("name", ["d128_bf16_causal", "d64_bf16_causal", "d128_fp16_causal",
                                  "koutlier_all_off"])
def test_nvfp4_sequence_views(name):
    """The views along the tokens (16-token blocks per channel), bit-exact: the oracle's
    nvfp4_quantize of the transposed normalized / smoothed matrices."""
    w = CASES[name]
    BH, N, d = w.B * w.H, w.N, w.d
    x = make_inputs(w)
    q, k = (to_device(x[n], w.dtype) for n in ("q", "k"))
    cfg = _cfg(w)
    fb = nvfp4.quant_prologue(q, k, cfg, seq=True)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    qf, kf = (x[n + "_f32"].reshape(BH, N, d) for n in ("q", "k"))
    pro = F.qattn_prologue(qf, kf, qknorm=w.qknorm, ksmooth=w.ksmooth)
    for t, src in (("q", pro["q_hat"]), ("k", pro["k_tilde"])):
        ref = F.nvfp4_quantize(np.swapaxes(src, -1, -2))
        codes = unpack_codes(getattr(fb, t + "_fp4_t").cpu().numpy().reshape(BH, d, N // 2))
        np.testing.assert_array_equal(codes, ref["codes"], err_msg=t + " codes")
        sf = unpack_sf_t(getattr(fb, t + "_sf_t").cpu().numpy(), BH, N, d)
        np.testing.assert_array_equal(sf, ref["sf"], err_msg=t + " scales")
        np.testing.assert_array_equal(getattr(fb, t + "_genc").cpu().numpy().reshape(BH),
                                      ref["genc"], err_msg=t + " genc")
    # the row views are unchanged by also producing the sequence views
    for t in ("q", "k"):
        np.testing.assert_array_equal(
            unpack_codes(getattr(fb, t + "_fp4").cpu().numpy().reshape(BH, N, d // 2)),
            pro[t + "_codes"])

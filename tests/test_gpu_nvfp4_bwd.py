"""NVFP4 Q-Attn backward parity: the CUDA path (sage_fp4_attn_bwd) against the NVFP4 oracle
(qattn_attention, outputs stored in the 16-bit type) on the same seeded inputs.

Both sides quantize dS per 128 x 128 tile with the tile's own global scale, in 16-key blocks
for dQ and 16-query blocks for dK, and multiply the same NVFP4 sequence views (the prologue is
bit-exact), so dQ and dK share the oracle's quantization error.  What separates them:
  * dS itself: the kernel's P = exp2(S c - lse log2 e) (FP32 arguments, the exp2
    approximation) and dP (FP32 accumulation) move dS by a few float32 ulps.  That changes an
    E2M1 code only where dS sits on a rounding boundary -- rare, but the element then moves by
    a whole code step;
  * dV: the kernel rounds P to the 16-bit type of dO before P^T dO (the tensor-core operand
    precision), the oracle keeps P exact: a relative error of at most u16 per product
    (u16 = 2^-8 for bf16, 2^-11 for fp16), partly cancelling over the queries;
  * the outputs' rounding to the 16-bit type, shared: one ulp where the two sit on either
    side of a rounding boundary.

test_nvfp4_backward_matches_oracle feeds the kernel the oracle's own forward results (O as
stored, LSE in float32), which isolates the backward: gates rel-L2 <= TOL_DQK for dQ, dK
(code flips are rare here: 1e-4 and below on every case) and <= TOL_DV[dtype] for dV (the P
rounding alone gives about u16 / 1.5).

test_nvfp4_fwd_bwd_chain runs the CUDA forward into the CUDA backward.  The forward's O
differs from the oracle's by the P V operand rounding (u16-sized, see test_gpu_nvfp4.py);
through D = rowsum(dO o O) that moves dS by about u16 |D| P, which flips E2M1 codes of dS
far more often.  Gate: the chain's distance to the oracle is at most CHAIN_FRAC of the
oracle's own distance to full-precision (float64, no quantizer) gradients, and its cosine
similarity to those gradients is within COS_SLACK of the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle.nvfp4_oracle as F
from fwd_bwd_b200 import nvfp4, ops
from fwd_bwd_b200.inputs import WORKLOADS, make_inputs

from gpu_helpers import TORCH_DT, cosine, rel_l2, to_device

pytestmark = pytest.mark.gpu

TOL_DQK = 1e-3
TOL_DV = {"bf16": 4e-3, "fp16": 1e-3}
CHAIN_FRAC = 0.25
COS_SLACK = 2e-3

BASE = WORKLOADS["sweep8192"]
CASES = {
    "d128_bf16_causal": BASE.replace(B=1, H=2, N=384),
    "d128_bf16_full": BASE.replace(B=1, H=2, N=256, causal=False),
    "d128_fp16_causal": BASE.replace(B=2, H=1, N=512, dtype="fp16"),
    "d64_bf16_causal": WORKLOADS["llama325m"].replace(B=1, H=2, N=384),
    "d64_fp16_full": WORKLOADS["llama325m"].replace(B=1, H=2, N=256, dtype="fp16",
                                                   causal=False),
    "koutlier_norm_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=256, qknorm=False),
    "koutlier_all_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=384, qknorm=False,
                                                     ksmooth=False),
    "small_ds_regime": WORKLOADS["long16k"].replace(H=1, N=512),
    "single_tile": BASE.replace(B=1, H=1, N=128),
}


def _cfg(w):
    return ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                      k_block=w.k_block)


def _oracle(w, x, quant=True):
    BH = w.B * w.H
    args = [x[n + "_f32"].reshape(BH, w.N, w.d) for n in ("q", "k", "v", "do")]
    return F.qattn_attention(*args, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth,
                             quant=quant, dtype=w.dtype if quant else None)


def _gpu(w, x, o_lse=None):
    """Prologue (with the sequence views), forward unless ``o_lse`` is given, backward."""
    q, k, v, do = (to_device(x[n], w.dtype) for n in ("q", "k", "v", "do"))
    cfg = _cfg(w)
    fb = nvfp4.quant_prologue(q, k, cfg, seq=True)
    if o_lse is None:
        o, lse = nvfp4.attn_fwd(fb, v, cfg)
    else:
        o, lse = o_lse
    dq, dk, dv = nvfp4.attn_bwd(q, k, v, fb, o, lse, do, cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    BH = w.B * w.H
    return {n: t.float().cpu().numpy().astype(np.float64).reshape(BH, w.N, w.d)
            for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}


@pytest.mark.parametrize("name", list(CASES))
def test_nvfp4_backward_matches_oracle(name):
    w = CASES[name]
    x = make_inputs(w)
    ref = _oracle(w, x)
    shape = (w.B, w.H, w.N, w.d)
    o = torch.from_numpy(ref["o"].astype(np.float32).reshape(shape)).to(TORCH_DT[w.dtype])
    lse = torch.from_numpy(ref["lse"].astype(np.float32).reshape(shape[:3]))
    g = _gpu(w, x, (o.cuda(), lse.cuda()))
    for n in ("dq", "dk", "dv"):
        err = rel_l2(g[n], ref[n])
        print(f"{name} {n}: rel_l2 {err:.3e}")
        tol = TOL_DV[w.dtype] if n == "dv" else TOL_DQK
        assert np.isfinite(g[n]).all()
        assert err <= tol, (n, err)


@pytest.mark.parametrize("name", ["d128_bf16_causal", "d64_fp16_full", "koutlier_all_off"])
def test_nvfp4_fwd_bwd_chain(name):
    w = CASES[name]
    x = make_inputs(w)
    ref = _oracle(w, x)
    exact = _oracle(w, x, quant=False)
    g = _gpu(w, x)
    for n in ("dq", "dk", "dv"):
        d_chain, d_quant = rel_l2(g[n], ref[n]), rel_l2(ref[n], exact[n])
        c_chain, c_ref = cosine(g[n], exact[n]), cosine(ref[n], exact[n])
        print(f"{name} {n}: chain-oracle {d_chain:.3e}  oracle-exact {d_quant:.3e}  "
              f"cos chain {c_chain:.5f} oracle {c_ref:.5f}")
        assert d_chain <= CHAIN_FRAC * d_quant, (n, d_chain, d_quant)
        assert c_chain >= c_ref - COS_SLACK, (n, c_chain, c_ref)


FULL_HEADS = [0, 511]  # flattened b*H+h of B32 H16 N8192 d128 (the bench workload)


def test_nvfp4_backward_full_size_sampled_heads():
    """The whole batch in the launch configuration bench.py --variant nvfp4 times (512 heads);
    the sampled heads carry the seeded per-head inputs and, as in the isolated test, the
    oracle's O (stored) and LSE, and are checked one head at a time (heads are independent)."""
    w = WORKLOADS["sweep8192"]
    dev = torch.device("cuda")
    dt = TORCH_DT[w.dtype]
    g = torch.Generator(device=dev).manual_seed(3)
    shape = (w.B * w.H, w.N, w.d)
    sig = {"q": w.sigma_qkv, "k": w.sigma_qkv, "v": w.sigma_qkv, "do": w.sigma_do}
    t = {n: (torch.randn(shape, generator=g, device=dev) * s).to(dt) for n, s in sig.items()}
    x = make_inputs(w, heads=FULL_HEADS)
    for n in t:
        for i, bh in enumerate(FULL_HEADS):
            t[n][bh] = torch.from_numpy(x[n][i].view(np.int16)).view(dt).to(dev)
    q, k, v, do = (t[n].view(w.B, w.H, w.N, w.d) for n in ("q", "k", "v", "do"))
    cfg = _cfg(w)
    fb = nvfp4.quant_prologue(q, k, cfg, seq=True)
    o, lse = nvfp4.attn_fwd(fb, v, cfg)
    refs = []
    for i, bh in enumerate(FULL_HEADS):
        one = [x[n + "_f32"][i:i + 1] for n in ("q", "k", "v", "do")]
        ref = F.qattn_attention(*one, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth,
                                dtype=w.dtype)
        b_, h_ = divmod(bh, w.H)
        o[b_, h_] = torch.from_numpy(ref["o"][0].astype(np.float32)).to(dt).to(dev)
        lse[b_, h_] = torch.from_numpy(ref["lse"][0].astype(np.float32)).to(dev)
        refs.append(ref)
    dq, dk, dv = nvfp4.attn_bwd(q, k, v, fb, o, lse, do, cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for i, bh in enumerate(FULL_HEADS):
        b_, h_ = divmod(bh, w.H)
        for n, tg in (("dq", dq), ("dk", dk), ("dv", dv)):
            got = tg[b_, h_].float().cpu().numpy().astype(np.float64)
            err = rel_l2(got, refs[i][n][0])
            print(f"head {bh} {n}: rel_l2 {err:.3e}")
            tol = TOL_DV[w.dtype] if n == "dv" else TOL_DQK
            assert np.isfinite(got).all() and err <= tol, (bh, n, err)


def _degenerate(kind, BH=2, N=256, d=128):
    rng = np.random.default_rng(17)
    q, k, v, do = (rng.standard_normal((BH, N, d)).astype(np.float32) for _ in range(4))
    if kind == "zero_do_head":     # dS = 0 on head 0: every tile's maximum is 0 (genc = 1)
        do[0] = 0.0
    elif kind == "tiny_do":        # dS ~ 2^-100: tiny (still normal) tile maxima and genc ~ 2^100
        do *= np.float32(2.0 ** -100)
    elif kind == "zero_qk_head":   # S = 0 on head 0: uniform attention, G = 0 for Q and K
        q[0] = 0.0
        k[0] = 0.0
    return q, k, v, do


@pytest.mark.parametrize("kind", ["zero_do_head", "tiny_do", "zero_qk_head"])
def test_nvfp4_backward_degenerate(kind):
    q, k, v, do = _degenerate(kind)
    BH, N, d = q.shape
    dt = torch.bfloat16
    tq, tk, tv, tdo = (torch.from_numpy(a).to(dt) for a in (q, k, v, do))
    qf, kf, vf, dof = (t.float().numpy() for t in (tq, tk, tv, tdo))  # exact bf16 values
    ref = F.qattn_attention(qf, kf, vf, dof, causal=True, qknorm=False, ksmooth=True,
                            dtype="bf16")
    cfg = ops.Config(causal=True, qknorm=False, ksmooth=True)
    dev = torch.device("cuda")
    shape = (1, BH, N, d)
    q_, k_, v_ = (t.reshape(shape).to(dev) for t in (tq, tk, tv))
    fb = nvfp4.quant_prologue(q_, k_, cfg, seq=True)
    o = torch.from_numpy(ref["o"].astype(np.float32).reshape(shape)).to(dt).to(dev)
    lse = torch.from_numpy(ref["lse"].astype(np.float32).reshape(shape[:3])).to(dev)
    dq_, dk_, dv_ = nvfp4.attn_bwd(q_, k_, v_, fb, o, lse, tdo.reshape(shape).to(dev), cfg)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for n, t in (("dq", dq_), ("dk", dk_), ("dv", dv_)):
        got = t.float().cpu().numpy().astype(np.float64).reshape(BH, N, d)
        assert np.isfinite(got).all(), n
        if kind == "zero_do_head":
            assert (got[0] == 0).all(), n  # no gradient flows from a zero output gradient
        err = rel_l2(got, ref[n])
        print(f"{kind} {n}: rel_l2 {err:.3e}")
        assert err <= (TOL_DV["bf16"] if n == "dv" else TOL_DQK), (n, err)


def test_nvfp4_autograd_and_stages_match_direct_calls():
    """nvfp4.qattn_attention (autograd) and the three staged backward calls give the direct
    calls' results: O, dK, dV bit for bit (deterministic kernels), dQ within float32 summation
    order (its tiles are added by asynchronous reductions in no fixed order)."""
    w = CASES["d128_bf16_causal"]
    x = make_inputs(w)
    q, k, v, do = (to_device(x[n], w.dtype) for n in ("q", "k", "v", "do"))
    cfg = _cfg(w)
    fb = nvfp4.quant_prologue(q, k, cfg, seq=True)
    o, lse = nvfp4.attn_fwd(fb, v, cfg)
    dq, dk, dv = nvfp4.attn_bwd(q, k, v, fb, o, lse, do, cfg)
    ws = torch.empty(nvfp4.bwd_workspace_bytes(cfg, q), dtype=torch.uint8, device=q.device)
    sq, sk, sv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for stage in range(3):
        nvfp4.attn_bwd(q, k, v, fb, o, lse, do, cfg, dq=sq, dk=sk, dv=sv, workspace=ws,
                       stage=stage)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    oa = nvfp4.qattn_attention(qa, ka, va, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth)
    oa.backward(do)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    assert torch.equal(oa.detach(), o)
    for a, b in ((sk, dk), (sv, dv), (ka.grad, dk), (va.grad, dv)):
        assert torch.equal(a, b)
    for a in (sq, qa.grad):
        err = rel_l2(a.float().cpu().numpy(), dq.float().cpu().numpy())
        # one bf16 ulp (2^-8 relative) in the rare elements whose float32 sum moves across a
        # rounding boundary: far below 1e-3 over the tensor
        assert err <= 1e-3, err

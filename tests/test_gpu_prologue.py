"""Prologue parity: INT8 codes, block scales, inverse RMS, K means and (Q-smoothing) Q means and
key biases bit-exact vs the oracle."""
import numpy as np
import pytest
import torch

import oracle.sage_oracle as O
from fwd_bwd_b200.inputs import WORKLOADS, f32_to_bits, bits_to_f32, make_inputs

from gpu_helpers import cfg_of, gpu_run, to_device
from fwd_bwd_b200 import ops

pytestmark = pytest.mark.gpu

BASE = WORKLOADS["sweep8192"]
CASES = {
    "tiny_fp16_d64_qb64": WORKLOADS["tiny"],
    "llama_bf16_d64": WORKLOADS["llama325m"].replace(B=2, H=2, N=512),
    "d128_bf16": BASE.replace(B=1, H=3, N=640),
    "d128_fp16_qb64": BASE.replace(B=1, H=2, N=384, dtype="fp16", q_block=64),
    "koutlier_norm_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=512, qknorm=False),
    "koutlier_smooth_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=512, ksmooth=False),
    "koutlier_all_off": WORKLOADS["koutlier"].replace(B=1, H=2, N=256, qknorm=False,
                                                     ksmooth=False),
    "qsmooth_d128_bf16": WORKLOADS["qoutlier"].replace(B=1, H=2, N=512),
    "qsmooth_d64_fp16_qb64": WORKLOADS["tiny"].replace(q_outlier=True, qsmooth=True),
    "qsmooth_ksmooth_off": WORKLOADS["qoutlier"].replace(B=1, H=2, N=256, ksmooth=False),
    "qsmooth_norm_off": WORKLOADS["qoutlier"].replace(B=2, H=1, N=256, qknorm=False),
}


def _compare(w, x, res):
    args = [x[n + "_f32"].reshape(-1, w.N, w.d) for n in ("q", "k", "v")]
    ref = O.prologue(*args, q_block=w.q_block, k_block=w.k_block, qknorm=w.qknorm,
                     ksmooth=w.ksmooth, qsmooth=w.qsmooth)
    BH = w.B * w.H
    for name in ("q_codes", "k_codes", "v_codes"):
        np.testing.assert_array_equal(res[name].reshape(BH, w.N, w.d), ref[name], err_msg=name)
    for name in ("q_scale", "k_scale", "v_scale"):
        np.testing.assert_array_equal(res[name].reshape(ref[name].shape).view(np.uint32),
                                      ref[name].view(np.uint32), err_msg=name)
    if w.qknorm:
        for name in ("q_inv_rms", "k_inv_rms"):
            np.testing.assert_array_equal(res[name].reshape(BH, w.N).view(np.uint32),
                                          ref[name].view(np.uint32), err_msg=name)
    if w.ksmooth:
        np.testing.assert_array_equal(res["k_mean"].reshape(BH, w.d).view(np.uint32),
                                      ref["k_mean"].view(np.uint32), err_msg="k_mean")
    if w.qsmooth:
        np.testing.assert_array_equal(res["q_mean"].reshape(BH, w.d).view(np.uint32),
                                      ref["q_mean"].view(np.uint32), err_msg="q_mean")
        np.testing.assert_array_equal(res["k_bias"].reshape(BH, w.N).view(np.uint32),
                                      ref["k_bias"].view(np.uint32), err_msg="k_bias")


@pytest.mark.parametrize("case", sorted(CASES))
def test_prologue_bit_exact(case):
    w = CASES[case]
    x = make_inputs(w)
    res = gpu_run(w, x, backward=False)
    _compare(w, x, res)


def test_prologue_edge_values():
    """Zero blocks (scale 0), exact ties (x/s = k + 1/2) and a subnormal-scale block."""
    w = BASE.replace(B=1, H=1, N=256, d=128, qknorm=False, ksmooth=False)
    x = make_inputs(w)
    v = x["v_f32"].reshape(w.N, w.d).copy()
    v[0:64] = 0.0                                      # zero block -> scale 0, codes 0
    v[64:128] = 0.0
    v[64, 0] = 127.0                                   # scale 1: ties at x.5 round to even
    v[65, :8] = [2.5, -2.5, 3.5, -0.5, 0.5, 1.5, 126.5, -125.5]
    v[128:192] *= np.float32(2.0 ** -130)              # subnormal-range values
    x["v"] = f32_to_bits(v.reshape(x["v_f32"].shape), w.dtype)
    x["v_f32"] = bits_to_f32(x["v"], w.dtype)
    res = gpu_run(w, x, backward=False)
    _compare(w, x, res)
    codes = res["v_codes"].reshape(w.N, w.d)
    assert np.all(codes[0:64] == 0) and res["v_scale"].ravel()[0] == 0
    np.testing.assert_array_equal(codes[65, :8], [2, -2, 4, 0, 0, 2, 126, -126])


def test_prologue_reuses_buffers_between_calls():
    """The same QuantBufs written twice gives identical bits (no stale state, no races)."""
    w = BASE.replace(B=2, H=2, N=512)
    x = make_inputs(w)
    q, k, v = (to_device(x[n], w.dtype) for n in ("q", "k", "v"))
    cfg = cfg_of(w)
    qb = ops.quant_prologue(q, k, v, cfg)
    first = qb.k_codes.clone(), qb.k_scale.clone(), qb.k_mean.clone()
    ops.quant_prologue(q, k, v, cfg, out=qb)
    torch.cuda.synchronize()
    for a, b in zip(first, (qb.k_codes, qb.k_scale, qb.k_mean)):
        assert torch.equal(a, b)

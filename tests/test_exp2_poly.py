"""CPU pins of the kernels' polynomial exp2 (ptx.cuh exp2_poly2; coefficients from
fwd_bwd_b200/exp2_fit.py), no GPU needed.

* The constants compiled into ptx.cuh are the float32 rounding of the Remez fit.
* The float32 Horner evaluation (each FMA rounded once, emulated exactly) keeps the relative
  error of 2^f below 2.5e-7 on the reduced range [-1/2, 1/2]; the range reduction (the
  1.5 * 2^23 rounding trick, exact) and the exponent insertion extend it to every z in
  [-125, 127], where the same bound holds.
* The bound is sharp enough to catch a wrong coefficient: the Taylor coefficients of the same
  degree miss it.
"""
import math
import os
import re

import numpy as np

from fwd_bwd_b200.exp2_fit import DEGREE, coefficients_f32, eval_f32, remez

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 2.5e-7


def _header_coefficients():
    src = open(os.path.join(ROOT, "fwd_bwd_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("float2 exp2_poly2("):]
    vals = dict(re.findall(r"kC(\d) = ([0-9.e+-]+)f", body))
    return np.array([np.float32(float(vals[str(i)])) for i in range(DEGREE + 1)], np.float32)


def _exp2_emulated(z):
    """ptx.cuh's steps for float32 z: clamp, rint by the magic add, exact f, Horner, exponent."""
    c = _header_coefficients()
    z0 = np.asarray(z, np.float32)
    z = np.maximum(z0, np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (z + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (z - j).astype(np.float32)
    p = eval_f32(c, f)
    jint = t.view(np.uint32).astype(np.int64) - 0x4B400000
    r = (p.view(np.int32).astype(np.int64) + (jint << 23)).astype(np.int32).view(np.float32)
    return np.where(z0 < np.float32(-125.0), np.float32(0.0), r)


def test_header_constants_are_the_fit():
    assert np.array_equal(_header_coefficients().view(np.uint32),
                          coefficients_f32().view(np.uint32))


def test_reduced_range_error_bound():
    f = np.linspace(-0.5, 0.5, 4_000_001).astype(np.float32)
    p = eval_f32(coefficients_f32(), f).astype(np.float64)
    rel = np.abs(p / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    # the float64 minimax level itself is about 7.5e-8 (equioscillation of the fit)
    c64 = remez()
    g = f.astype(np.float64)
    lvl = np.abs(np.polyval(c64[::-1], g) / np.exp2(g) - 1.0).max()
    assert 5e-8 < lvl < 1e-7


def test_full_range_reconstruction():
    rng = np.random.default_rng(0)
    z = np.concatenate([np.linspace(-125.0, 0.0, 1_000_001), rng.uniform(-125.0, 127.0, 200_000),
                        np.arange(-125, 128, dtype=np.float64)]).astype(np.float32)
    got = _exp2_emulated(z).astype(np.float64)
    rel = np.abs(got / np.exp2(z.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    # below the clamp the kernel returns 0 (as the flushing hardware exp2 does below -126)
    assert (_exp2_emulated(np.asarray([-125.5, -130.0, -1e4], np.float32)) == 0).all()


def test_bound_catches_taylor_coefficients():
    taylor = np.array([math.log(2.0) ** k / math.factorial(k) for k in range(DEGREE + 1)],
                      np.float32)
    f = np.linspace(-0.5, 0.5, 100_001).astype(np.float32)
    rel = np.abs(eval_f32(taylor, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() > BOUND

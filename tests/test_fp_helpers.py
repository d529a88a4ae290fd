"""CPU pins of the float32 helper arithmetic the NVFP4 backward kernel uses in place of a
division (no GPU needed).

div6_rn: x / 6 as q = RN(x * r), r = RN(1/6); e = x - 6 q (exact, one FMA); RN(q + e r) -- the
correction step of Markstein's division algorithm.  The kernel only needs the E4M3 code of the
quotient; this test pins the quotient itself.  Scaling x by a power of two scales every
intermediate exactly while the quotient stays normal, so one binade [1, 2) covers every x with
a normal quotient; below that (x < 6 * 2^-126) both quotients are far under 2^-10 and the E4M3
code is 0 either way.
"""
import numpy as np

F32, F64 = np.float32, np.float64


def _rn32(x64):
    return np.asarray(x64, F64).astype(F32)


def _div6_emulated(x):
    """The kernel's three float32 operations, each rounded once (exact emulation in float64 with
    the double-rounding cases of the last step resolved exactly)."""
    r = F32(1.0) / F32(6.0)
    assert r == _rn32(1.0 / 6.0)
    x64 = x.astype(F64)
    q = _rn32(x64 * F64(r))                        # 24 x 24-bit product: exact in float64
    e = _rn32(x64 - 6.0 * q.astype(F64))          # exact residual, exactly representable
    s = q.astype(F64) + e.astype(F64) * F64(r)    # e * r exact; the sum rounded to float64
    out = _rn32(s)
    # float64 rounding of the sum can only mislead the float32 rounding when it lands on a
    # float32 midpoint: resolve those few cases with exact rational arithmetic
    up = np.nextafter(out, F32(np.inf)).astype(F64)
    dn = np.nextafter(out, F32(-np.inf)).astype(F64)
    mid = (s == (out.astype(F64) + up) / 2) | (s == (out.astype(F64) + dn) / 2)
    if mid.any():
        from fractions import Fraction
        for i in np.flatnonzero(mid):
            exact = Fraction(float(q[i])) + Fraction(float(e[i])) * Fraction(float(r))
            cands = [F32(dn[i]), out[i], F32(up[i])]
            best = min(cands, key=lambda c: (abs(Fraction(float(c)) - exact),
                                             int(np.asarray(c).view(np.uint32)) & 1))
            out[i] = best
    return out


def test_div6_correction_is_correctly_rounded_on_a_binade():
    bits = np.arange(0x3F800000, 0x40000000, dtype=np.uint32)  # every float32 in [1, 2)
    x = bits.view(F32)
    got = _div6_emulated(x)
    # x / 6 is never within 2^-53 (relative) of a float32 midpoint (x = M 2^k with M not a
    # multiple of 3 leaves a remainder of a third), so float64 then float32 is RN32(x / 6)
    want = _rn32(x.astype(F64) / 6.0)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_div6_correction_step_is_needed():
    """The pin is sensitive: the product x * RN(1/6) alone, or a correction that uses x - 5 q as
    the residual, is not correctly rounded on the binade."""
    bits = np.arange(0x3F800000, 0x40000000, dtype=np.uint32)
    x = bits.view(F32)
    r = F32(1.0) / F32(6.0)
    want = _rn32(x.astype(F64) / 6.0)
    q = _rn32(x.astype(F64) * F64(r))
    assert not np.array_equal(q.view(np.uint32), want.view(np.uint32))
    e_bad = _rn32(x.astype(F64) - 5.0 * q.astype(F64))
    bad = _rn32(q.astype(F64) + e_bad.astype(F64) * F64(r))
    assert not np.array_equal(bad.view(np.uint32), want.view(np.uint32))


def _quant_fast(x, s):
    """The INT8 prologue quantizer's division-free path (rowops.cuh quant_magic_r), in float32
    numpy operations (each IEEE-rounded, as the kernel's): rint(x * RN(1/s)) unless that product
    lies within 2^-15 of a half-integer, where the correctly rounded quotient decides."""
    x = np.asarray(x, F32)
    s = F32(s)
    r = F32(1.0) / s
    q = x * r
    magic = F32(12582912.0)
    t = q + magic
    f = q - (t - magic)
    amb = ~np.isfinite(r) | (np.abs(f) >= F32(0.5) - F32(2.0 ** -15))
    exact = np.rint(x / s)
    return np.where(amb, exact, (t - magic)), amb


def _blocks(rng, n):
    """Blocks of 8 values with their scale s = RN(absmax / 127), including values planted on
    (and one ulp either side of) half-integer multiples of s, and tiny / huge magnitudes."""
    out = []
    for i in range(n):
        mag = F32(2.0) ** F32(rng.integers(-120, 120))
        x = (rng.standard_normal(8) * mag).astype(F32)
        am = np.abs(x).max()
        s = F32(am) / F32(127.0)
        if i % 3 == 0:  # plant half-integer quotients
            k = rng.integers(-126, 126, 4).astype(F32) + F32(0.5)
            p = (k * s).astype(F32)
            p = np.clip(p, -am, am)
            x[:4] = p
            x[4] = np.nextafter(p[0], F32(np.inf))
            x[5] = np.nextafter(p[1], F32(-np.inf))
        out.append((x, s))
    return out


def test_int8_quantizer_fast_path_is_exact():
    rng = np.random.default_rng(7)
    n_amb = 0
    for x, s in _blocks(rng, 20000):
        got, amb = _quant_fast(x, s)
        want = np.rint(x / s)  # the IEEE quotient, rounded half to even
        assert np.array_equal(got, want), (x, s)
        n_amb += int(amb.sum())
    assert n_amb > 0  # the planted half-integers reach the exact path


def test_int8_quantizer_bound_is_needed():
    """Without the fallback (rint of x * RN(1/s) alone) some planted ties round differently."""
    rng = np.random.default_rng(8)
    bad = 0
    for x, s in _blocks(rng, 20000):
        r = F32(1.0) / s
        bad += int((np.rint(x * r) != np.rint(x / s)).sum())
    assert bad > 0

"""Numeric identities the CUDA kernels rely on, checked on the host with IEEE numpy arithmetic.

The 1x128 quantiser computes fp32(x / s) as fp32(fp64(x) * fp64(1 / s)) (one fp64 reciprocal per
group instead of an fp32 division per element).  The two agree because the fp64 product is within
2^-52 (relative) of x / s, while a quotient of two 24-bit-significand numbers is never an fp32
rounding midpoint and otherwise lies at least 2^-49 (relative) from every midpoint.
"""
from __future__ import annotations

import numpy as np


def _pairs(n, seed):
    rng = np.random.default_rng(seed)
    amax = np.abs(rng.standard_normal(n).astype(np.float32) * np.float32(2.0) ** rng.integers(-60, 60, n)).astype(np.float32)
    amax = (amax + np.float32(1e-30)).astype(np.float32)
    s = (amax / np.float32(448.0)).astype(np.float32)
    x = (amax * rng.uniform(-1, 1, n).astype(np.float32)).astype(np.float32)
    x[::5] = (s[::5] * np.float32(rng.integers(-448, 449, len(x[::5])))).astype(np.float32)  # exact multiples
    x[1::5] = amax[1::5]                                                                     # the group's amax
    return x, s


def test_fp64_reciprocal_product_rounds_like_fp32_division():
    for seed in range(4):
        x, s = _pairs(1_000_000, seed)
        ref = (x / s).astype(np.float32)
        got = (x.astype(np.float64) * (1.0 / s.astype(np.float64))).astype(np.float32)
        assert np.array_equal(ref.view(np.uint32), got.view(np.uint32))


def test_fp64_reciprocal_product_near_fp32_midpoints():
    # quotients steered close to fp32 rounding midpoints: x = s * (m + 1/2 ulp) rounded to fp32
    rng = np.random.default_rng(11)
    s = (rng.uniform(0.5, 2.0, 200_000) * 2.0 ** rng.integers(-30, 30, 200_000)).astype(np.float32)
    m = rng.uniform(1, 448, 200_000).astype(np.float32)
    mid = m.astype(np.float64) + np.spacing(m).astype(np.float64) / 2
    x = (mid * s.astype(np.float64)).astype(np.float32)
    ref = (x / s).astype(np.float32)
    got = (x.astype(np.float64) * (1.0 / s.astype(np.float64))).astype(np.float32)
    assert np.array_equal(ref.view(np.uint32), got.view(np.uint32))


# ---------------------------------------------------------------------------
# The quantisers' fp32 division: q1 = RN(x * r), r = RN(1 / s); rem = RN(x - q1 * s) (one fma, exact);
# q = RN(q1 + rem * r) (one fma), with copysign for a zero x.  Markstein's correction step makes q the
# correctly rounded quotient when the residual does not underflow, which the kernels guarantee by taking
# this path only for group scales s >= 2^-90.  The fma's single rounding is emulated exactly with
# rational arithmetic.
# ---------------------------------------------------------------------------
from fractions import Fraction


def _rn32(x: Fraction) -> np.float32:
    """Round a rational to the nearest fp32, ties to even (normal and subnormal range)."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    n, rem = divmod(a, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    return np.float32(sign * float(n * ulp))


def _fma32(a, b, c) -> np.float32:
    return _rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _quotient_rn(x: np.float32, s: np.float32) -> np.float32:
    r = np.float32(np.float32(1.0) / s)
    q1 = np.float32(x * r)
    rem = _fma32(-q1, s, x)
    q = _fma32(rem, r, q1)
    return np.copysign(q, x).astype(np.float32)


def test_fp32_corrected_quotient_is_the_correctly_rounded_quotient():
    rng = np.random.default_rng(21)
    n = 20_000
    amax = np.ldexp(1.0 + rng.random(n), rng.integers(-80, 120, n)).astype(np.float32)
    s = (amax / np.float32(448.0)).astype(np.float32)
    x = (amax * rng.uniform(-1, 1, n)).astype(np.float32)
    # a third of the quotients steered next to fp32 rounding midpoints, a few exact multiples and zeros
    k = np.arange(n) % 3 == 1
    m = rng.uniform(2.0 ** -11, 448, n)
    mid = (m.astype(np.float32).astype(np.float64) + np.spacing(m.astype(np.float32)).astype(np.float64) / 2)
    x[k] = (mid[k] * s[k].astype(np.float64)).astype(np.float32)
    x[::97] = (s[::97] * np.float32(7.0)).astype(np.float32)
    x[::89] = np.float32(-0.0)
    assert float(s.min()) >= 2.0 ** -90
    for xi, si in zip(x, s):
        ref = np.float32(xi / si)
        got = _quotient_rn(xi, si)
        assert ref.view(np.uint32) == got.view(np.uint32), (float(xi), float(si), float(ref), float(got))


def test_fp32_corrected_quotient_needs_the_correction():
    # the plain reciprocal product alone is not the correctly rounded quotient for some of the same pairs,
    # so the test above would catch a kernel that dropped the correction step
    rng = np.random.default_rng(22)
    s = np.ldexp(1.0 + rng.random(5000), rng.integers(-40, 40, 5000)).astype(np.float32)
    x = (s.astype(np.float64) * rng.uniform(1, 448, 5000)).astype(np.float32)
    r = (np.float32(1.0) / s).astype(np.float32)
    assert np.any((x * r).astype(np.float32) != (x / s).astype(np.float32))


# ---------------------------------------------------------------------------
# The fp32 group scale amax / 448: Markstein's correction step with the fixed reciprocal r = RN(1/448) for
# every amax in [2^-116, FLT_MAX], an IEEE division below.
# ---------------------------------------------------------------------------
_R448 = np.float32(float.fromhex("0x1.24924ap-9"))


def _scale_markstein(a: np.float32) -> np.float32:
    q1 = np.float32(a * _R448)
    return _fma32(_fma32(-q1, np.float32(448.0), a), _R448, q1)


def test_reciprocal_of_448_is_the_rounded_reciprocal():
    assert _R448 == _rn32(Fraction(1, 448))


def test_group_scale_division_by_448_sampled():
    rng = np.random.default_rng(31)
    lo, hi = np.float32(2.0 ** -116), np.finfo(np.float32).max
    a = np.ldexp(1.0 + rng.random(6000), rng.integers(-116, 128, 6000)).astype(np.float32)
    edges = [lo, np.nextafter(lo, np.float32(np.inf)), hi, np.nextafter(hi, np.float32(0)), np.float32(448.0),
             np.float32(448.0 * 2.0 ** 5), np.float32(1.0), np.float32(7.0)]
    # quotients steered next to fp32 rounding midpoints
    m = np.ldexp(1.0 + rng.random(3000), rng.integers(-100, 100, 3000)).astype(np.float32)
    mid = (m.astype(np.float64) + np.spacing(m).astype(np.float64) / 2) * 448.0
    near = mid.astype(np.float32)
    for ai in list(a) + edges + list(near[np.isfinite(near) & (near >= lo)]):
        ref = _rn32(Fraction(float(ai)) / 448)
        got = _scale_markstein(np.float32(ai))
        assert ref.view(np.uint32) == got.view(np.uint32), (float(ai), float(ref), float(got))


_DIV448_C = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static int check(uint32_t u, float r) {
  const float a = f_of(u), q1 = a * r, q = fmaf(fmaf(-q1, 448.0f, a), r, q1);
  return u_of(q) != u_of((float)((double)a / 448.0));  /* double quotient rounded once more: exact here */
}
int main(int argc, char** argv) {
  const uint32_t step = (uint32_t)atoi(argv[1]);
  const float r = 0x1.24924ap-9f;
  const uint32_t lo = u_of(0x1p-116f), hi = u_of(3.40282347e38f);
  unsigned long long bad = 0;
  for (uint32_t u = lo; u < lo + (1u << 20); ++u) bad += check(u, r);
  for (uint32_t u = hi - (1u << 20); u <= hi; ++u) bad += check(u, r);
  for (uint32_t u = lo; u <= hi - step; u += step) bad += check(u, r);
  printf("%llu\n", bad);
  return 0;
}
"""


def test_group_scale_division_by_448_strided_sweep(tmp_path):
    """Every fp32 amax at the two ends of [2^-116, FLT_MAX] (2^20 values each) and every 61st in between, in
    C with hardware fp32 arithmetic (no contraction); the full range was also swept once with step 1."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        import pytest
        pytest.skip("no C compiler")
    src = tmp_path / "div448.c"
    src.write_text(_DIV448_C.replace("#include <math.h>", "#include <math.h>\n#include <stdlib.h>"))
    exe = tmp_path / "div448"
    subprocess.run([gcc, "-O2", "-ffp-contract=off", str(src), "-o", str(exe), "-lm"], check=True)
    out = subprocess.run([str(exe), "61"], check=True, capture_output=True, text=True).stdout
    assert int(out.strip()) == 0

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

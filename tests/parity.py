"""Acceptance checks comparing GPU outputs with the CPU oracle.

FP8 (operations 1 and 3): the tensor-core accumulation order inside a 128-deep
block is unspecified, and the per-block partial and the running accumulator
are fp32, so results are not bit-reproducible against an fp64 definition.
Bound used: |gpu - y| <= 1e-3 * S + ulp(y), where S = sum_kb |s| * sum |a*b|
(the magnitude the accumulation runs over) and ulp(y) is one unit in the last
place of the output format at the oracle value (bf16: 2^(floor(log2|y|) - 7),
fp32: 2^(floor(log2|y|) - 23); the smallest normal when y == 0).  fp32
accumulation of 128-term partials and of K/128 promoted partials stays orders
of magnitude below 1e-3 * S; the ulp term covers the final rounding.

INT8 (operation 2): bit-exact for the int32 accumulator, the fp32
(float(acc) * s_a) * s_b and its bf16 rounding.

e4m3 outputs (scale_result of the rowwise operation): the kernel rounds an
fp32 value z within |s_r| * (1e-3 * S + ulp_f32(y)) + ulp_f32(s_r * y) of
s_r * y, and e4m3 rounding is monotone, so its code must lie between the codes
of the two ends of that interval.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def to_f64(gpu: torch.Tensor) -> np.ndarray:
    return gpu.detach().float().cpu().double().numpy()


def ulp_at(y: np.ndarray, out_dtype: torch.dtype) -> np.ndarray:
    mant = 7 if out_dtype == torch.bfloat16 else 23
    a = np.abs(y)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    u = np.exp2(e - mant)
    return np.where(a > 0, u, 2.0 ** -126)


def fp8_check(gpu: torch.Tensor, y: np.ndarray, S: np.ndarray, out_dtype: torch.dtype, label: str = ""):
    """Asserts the FP8 acceptance bound element by element; returns the worst ratio."""
    g = to_f64(gpu)
    assert g.shape == y.shape, (g.shape, y.shape)
    assert np.all(np.isfinite(g)), f"{label}: non-finite GPU outputs"
    tol = 1e-3 * S + ulp_at(y, out_dtype)
    err = np.abs(g - y)
    ratio = err / tol
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        idx = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        bad = int((ratio > 1.0).sum())
        raise AssertionError(f"{label}: {bad} of {ratio.size} elements outside tolerance; worst at {idx}: "
                             f"gpu={g[idx]!r} oracle={y[idx]!r} S={S[idx]!r} ratio={worst:.3g}")
    return worst


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def f32_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


def rows_sample(M: int, tile: int = 128, extra: int = 8, seed: int = 0):
    """Rows covering the first / last row of several tiles, the ragged tail and a few random rows."""
    rng = np.random.default_rng(seed)
    r = {0, 1, M - 1, M // 2}
    for t in range(0, M, tile * max(1, (M // tile) // 6)):
        r.update({t, min(M - 1, t + tile - 1)})
    r.update(int(v) for v in rng.integers(0, M, extra))
    return sorted(v for v in r if 0 <= v < M)


def oracle_fp8(d, rows=None):
    return oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"], rows=rows)


def e4m3_check(gpu: torch.Tensor, y: np.ndarray, S: np.ndarray, s_r: float, label: str = ""):
    """Asserts an e4m3 output against the oracle value y before the output scale s_r;
    returns the fraction of codes equal to the oracle's own rounding of s_r * y."""
    codes = gpu.detach().cpu().view(torch.uint8).numpy()
    assert codes.shape == y.shape, (codes.shape, y.shape)
    table = oracle.e4m3_table()
    g = table[codes]
    assert not np.any(np.isnan(g)), f"{label}: NaN codes in a saturating output"
    z = s_r * y
    d = abs(s_r) * (1e-3 * S + ulp_at(y, torch.float32)) + ulp_at(z, torch.float32)
    lo, hi = table[oracle.e4m3_encode(z - d)], table[oracle.e4m3_encode(z + d)]
    bad = (g < lo) | (g > hi)
    if np.any(bad):
        idx = np.unravel_index(int(np.argmax(bad)), bad.shape)
        raise AssertionError(f"{label}: {int(bad.sum())} of {bad.size} codes outside the rounding window; first at "
                             f"{idx}: gpu={g[idx]!r} oracle s_r*y={z[idx]!r} window=[{lo[idx]!r}, {hi[idx]!r}]")
    return float(np.mean(codes == oracle.e4m3_encode(z)))


def assert_quantised(gq: np.ndarray, gs: np.ndarray, rq: np.ndarray, rs: np.ndarray, fmt: int):
    """Quantiser parity: codes and scales bit-exact (fmt 0: fp32 scales by bit pattern; 1: e8m0 bytes)."""
    assert gq.shape == rq.shape and gs.shape == rs.shape, (gq.shape, rq.shape, gs.shape, rs.shape)
    bad = np.argwhere(gq != rq)
    assert bad.size == 0, (f"{len(bad)} codes differ, first at {bad[0]}: "
                           f"gpu {gq[tuple(bad[0])]:#x} oracle {rq[tuple(bad[0])]:#x}")
    if fmt == 0:
        assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32)), "fp32 scales differ"
    else:
        assert np.array_equal(gs, rs), "e8m0 bytes differ"

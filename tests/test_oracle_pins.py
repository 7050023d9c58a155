"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test compares the oracle with something other than its own formula:
a library routine computing the same quantity another way, exact rational
arithmetic, a closed form, an invariant, or values printed on the pages
(tests/golden/).  No GPU is involved.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from exact import bf16_bits, bf16_exact, f32_exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# e4m3 decode table
# ---------------------------------------------------------------------------
def test_e4m3_table_matches_torch_decode():
    ours = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan_ours, nan_ref = np.isnan(ours), np.isnan(ref)
    assert (nan_ours == nan_ref).all()
    assert list(np.nonzero(nan_ours)[0]) == [0x7F, 0xFF]
    np.testing.assert_array_equal(ours[~nan_ours], ref[~nan_ref])


def test_e4m3_table_closed_forms():
    t = oracle.e4m3_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0          # largest finite
    assert t[0x01] == 2.0 ** -9                            # smallest subnormal
    assert t[0x08] == 2.0 ** -6                            # smallest normal
    assert t[0x38] == 1.0 and t[0xC0] == -2.0
    assert t[0x80] == 0.0 and math.copysign(1.0, t[0x80]) == -1.0
    finite = t[~np.isnan(t)]
    assert len(np.unique(finite[finite > 0])) == 126


# ---------------------------------------------------------------------------
# fp64 -> bf16 / fp32 rounding
# ---------------------------------------------------------------------------
def test_round_bf16_matches_exact_rational_rounding():
    rng = np.random.default_rng(7)
    vals = list(rng.standard_normal(400) * np.exp2(rng.integers(-140, 130, 400)))
    # ties between adjacent bf16 values, and points just off the ties
    for base in (1.0, 1.5, 3.0 / 1024, 2.0 ** -130, 2.0 ** 120 * 1.25):
        ulp = 2.0 ** (math.floor(math.log2(base)) - 7) if base >= 2.0 ** -126 else 2.0 ** -133
        for k in range(4):
            vals += [base + (k + 0.5) * ulp, -(base + (k + 0.5) * ulp),
                     base + (k + 0.5) * ulp + ulp * 2.0 ** -30]
    vals += [0.0, -0.0, 2.0 ** 128 * 0.999, -3.4e38, 2.0 ** -140, 2.0 ** -134, 2.0 ** -133 * 1.5]
    vals = np.array(vals, dtype=np.float64)
    got = oracle.round_bf16(vals)
    for v, g in zip(vals, got):
        want = bf16_exact(Fraction(float(v)))
        if math.isinf(want):
            assert g & 0x7FFF == 0x7F80
        else:
            assert g == bf16_bits(want) or (want == 0.0 and g & 0x7FFF == 0), (v, hex(g), want)


def test_round_bf16_is_direct_not_double_rounding():
    # 1 + 2^-8 + 2^-30 lies just above the bf16 tie 1 + 2^-8; via fp32 it would
    # collapse onto the tie and round down to 1.0.
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle.bf16_bits_to_f64(oracle.round_bf16(np.array([v])))[0] == 1.0 + 2.0 ** -7


def test_round_bf16_agrees_with_torch_on_fp32_values():
    x = torch.randn(20000, dtype=torch.float32) * torch.exp2(torch.randint(-60, 60, (20000,)).float())
    ours = oracle.round_bf16(x.double().numpy())
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_round_f32_matches_exact():
    rng = np.random.default_rng(3)
    vals = rng.standard_normal(300) * np.exp2(rng.integers(-150, 120, 300))
    got = oracle.round_f32(vals)
    for v, g in zip(vals, got):
        assert float(g) == f32_exact(Fraction(float(v)))


# ---------------------------------------------------------------------------
# input generator (the quantiser the recipe fixes), independent of the oracle
# ---------------------------------------------------------------------------
def test_generator_e4m3_rne_ties_and_saturation():
    t = oracle.e4m3_table()
    pos = np.sort(np.unique(t[(~np.isnan(t)) & (t > 0)]))
    mids = (pos[:-1] + pos[1:]) / 2.0
    codes = wl.to_e4m3_bytes(torch.tensor(mids, dtype=torch.float32)).numpy()
    for mid, lo, hi, c in zip(mids, pos[:-1], pos[1:], codes):
        want_even = lo if (int(np.nonzero(t == lo)[0][0]) & 1) == 0 else hi
        assert t[c] == want_even, (mid, lo, hi, t[c])
    sat = wl.to_e4m3_bytes(torch.tensor([448.0, 449.0, 464.0, 1e9, -1e9], dtype=torch.float32)).numpy()
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_generator_e4m3_is_nearest_value():
    t = oracle.e4m3_table()
    finite = t[~np.isnan(t)]
    x = torch.linspace(-500, 500, 20001, dtype=torch.float32)
    dec = t[wl.to_e4m3_bytes(x).numpy()]
    xc = np.clip(x.double().numpy(), -448, 448)
    best = np.abs(xc[:, None] - finite[None, :]).min(axis=1)
    np.testing.assert_array_equal(np.abs(xc - dec), best)


def test_generator_e8m0_exponent_is_ceil_log2():
    amax = torch.tensor([448.0, 449.0, 224.0, 1.0, 3.5, 0.0, 448.0 * 2 ** -20], dtype=torch.float32)
    e = wl.e8m0_exponent(amax).tolist()
    assert e == [0, 1, -1, math.ceil(math.log2(1 / 448)), math.ceil(math.log2(3.5 / 448)), 0, -20]


# ---------------------------------------------------------------------------
# operation 1: FP8 block-scaled GEMM
# ---------------------------------------------------------------------------
def _int_codes(codes: np.ndarray) -> np.ndarray:
    """e4m3 codes -> integers v with value = v * 2^-9 (every e4m3 value is one)."""
    t = oracle.e4m3_table()
    v = t[codes] * 512.0
    assert np.all(v == np.round(v))
    return v.astype(np.int64)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (2, 256, 256), (3, 128, 512), (129, 256, 128)])
def test_fp8_brute_force_exact_rational(M, N, K):
    d = wl.fp8_blockwise_inputs(M, N, K, seed=900 + M)
    sa, sb = d["scale_a"].numpy(), d["scale_b"].numpy()
    y, S = oracle.fp8_blockwise(d["A"], d["B_t"], sa, sb)
    ai, bi = _int_codes(d["A"].numpy()), _int_codes(d["B_t"].numpy())
    KB = K // 128
    # exact integer partial per K block (integer matmul is exact in int64)
    P = [ai[:, kb * 128:(kb + 1) * 128] @ bi[:, kb * 128:(kb + 1) * 128].T for kb in range(KB)]
    rows = range(M) if M <= 3 else (0, 1, 64, 127, 128)
    for m in rows:
        for n in range(0, N, 7):
            exact = sum(Fraction(float(sa[m, kb])) * Fraction(float(sb[kb, n // 128])) * int(P[kb][m, n])
                        for kb in range(KB)) / (1 << 18)
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(float(S[m, n])) * Fraction(1, 2 ** 50)
            assert oracle.round_bf16(np.array([y[m, n]]))[0] == bf16_bits(bf16_exact(exact))
            assert oracle.round_f32(np.array([y[m, n]]))[0] == np.float32(f32_exact(exact))


def test_fp8_small_integers_give_exact_integer_products():
    rng = np.random.default_rng(11)
    M, N, K = 5, 256, 384
    t = oracle.e4m3_table()
    code_of = {}
    for c, v in enumerate(t):
        if not np.isnan(v) and float(v) not in code_of:
            code_of[float(v)] = c
    ints_a = rng.integers(-4, 5, (M, K))
    ints_b = rng.integers(-4, 5, (N, K))
    enc = np.vectorize(lambda v: code_of[float(v)] if v != 0 else 0)
    A, B = enc(ints_a).astype(np.uint8), enc(ints_b).astype(np.uint8)
    y, _ = oracle.fp8_blockwise(A, B, np.ones((M, K // 128), np.float32), np.ones((K // 128, 2), np.float32))
    np.testing.assert_array_equal(y, (ints_a @ ints_b.T).astype(np.float64))


def test_fp8_matches_fp64_library_matmul_of_dequantised_operands():
    d = wl.fp8_blockwise_inputs(256, 256, 512, seed=0)
    y, S = oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"])
    t = torch.from_numpy(oracle.e4m3_table())
    A = t[d["A"].long()] * d["scale_a"].double().repeat_interleave(128, dim=1)
    B = t[d["B_t"].long()].T * d["scale_b"].double().repeat_interleave(128, 0).repeat_interleave(128, 1)
    ref = (A @ B).numpy()
    assert np.all(np.abs(y - ref) <= 1e-12 * S + 1e-300)


def test_fp8_power_of_two_scale_linearity():
    d = wl.fp8_blockwise_inputs(64, 256, 256, seed=5)
    y0, _ = oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"])
    sa = d["scale_a"].clone()
    sa[3, :] *= 2.0 ** 5
    sa[17, :] *= 2.0 ** -9
    y1, _ = oracle.fp8_blockwise(d["A"], d["B_t"], sa, d["scale_b"])
    np.testing.assert_array_equal(y1[3], y0[3] * 2.0 ** 5)
    np.testing.assert_array_equal(y1[17], y0[17] * 2.0 ** -9)
    keep = [i for i in range(64) if i not in (3, 17)]
    np.testing.assert_array_equal(y1[keep], y0[keep])


def test_fp8_one_hot_scale_b_isolates_its_block():
    M, N, K = 8, 384, 512
    d = wl.fp8_blockwise_inputs(M, N, K, seed=6)
    kb0, nb0 = 2, 1
    sb = np.zeros((K // 128, 3), np.float32)
    sb[kb0, nb0] = 1.0
    y, _ = oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], sb)
    ai, bi = _int_codes(d["A"].numpy()), _int_codes(d["B_t"].numpy())
    P = (ai[:, kb0 * 128:(kb0 + 1) * 128] @ bi[:, kb0 * 128:(kb0 + 1) * 128].T).astype(np.float64) * 2.0 ** -18
    want = np.zeros((M, N))
    want[:, nb0 * 128:(nb0 + 1) * 128] = (P * d["scale_a"].double().numpy()[:, kb0:kb0 + 1])[:, nb0 * 128:(nb0 + 1) * 128]
    np.testing.assert_array_equal(y, want)


def test_fp8_scale_shapes_from_the_blockwise_issue():
    """The compile-error message prints scale_a (16640, 64) and scale_b (64, 40)
    for M=16640, K=8192, N=5120 (tests/golden/scale_shapes_blockwise.json)."""
    g = json.load(open(os.path.join(GOLDEN, "scale_shapes_blockwise.json")))
    M, K, N = g["M"], g["K"], g["N"]
    assert (M, -(-K // 128)) == tuple(g["scale_a"]) and (-(-K // 128), -(-N // 128)) == tuple(g["scale_b"])
    A = np.zeros((M, K), np.uint8)
    A[5, :] = 0x38                                       # row 5 = ones
    B = np.full((N, K), 0x38, np.uint8)                  # all ones
    sa = np.ones(g["scale_a"], np.float32)
    sb = np.ones(g["scale_b"], np.float32)
    y, _ = oracle.fp8_blockwise(A, B, sa, sb, rows=[5, 6])
    assert np.all(y[0] == K) and np.all(y[1] == 0)
    with pytest.raises(AssertionError):                  # the rowwise shapes are not blockwise
        oracle.fp8_blockwise(A[:2], B, np.ones(g["rowwise_scale_a"], np.float32)[:2],
                             np.ones(g["rowwise_scale_b"], np.float32))


# ---------------------------------------------------------------------------
# FP8 with tensorwise / rowwise scales and bias
# ---------------------------------------------------------------------------
def _rowwise_inputs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    A = wl.to_e4m3_bytes(torch.randn(M, K, generator=g) * 4)
    B = wl.to_e4m3_bytes(torch.randn(N, K, generator=g) * 4)
    sa = (torch.rand(M, generator=g) + 0.5).numpy().astype(np.float32)
    sb = (torch.rand(N, generator=g) + 0.5).numpy().astype(np.float32)
    bias = torch.randn(N, generator=g).numpy().astype(np.float32)
    return A, B, sa, sb, bias


@pytest.mark.parametrize("M,N,K", [(3, 5, 48), (2, 129, 128), (4, 7, 300)])
def test_fp8_rowwise_brute_force_exact_rational(M, N, K):
    """Exact rational reference (Fraction) of acc * (s_a * s_b) + bias, K not necessarily a multiple of 128."""
    A, B, sa, sb, bias = _rowwise_inputs(M, N, K, seed=70 + K)
    y, S = oracle.fp8_rowwise(A, B, sa, sb, bias)
    ai, bi = _int_codes(A.numpy()), _int_codes(B.numpy())
    P = ai @ bi.T  # exact integers, scaled by 2^18
    for m in range(M):
        for n in range(N):
            exact = Fraction(int(P[m, n]), 1 << 18) * Fraction(float(sa[m])) * Fraction(float(sb[n])) \
                + Fraction(float(bias[n]))
            bound = (abs(exact) + 1) * Fraction(1, 2 ** 51)   # two fp64 roundings (scale, bias add)
            assert abs(Fraction(float(y[m, n])) - exact) <= bound
            assert S[m, n] == pytest.approx(float(abs(Fraction(int(np.abs(ai[m] * bi[n]).sum()), 1 << 18))
                                                  * Fraction(float(sa[m])) * Fraction(float(sb[n]))), rel=1e-15)


def test_fp8_rowwise_equals_blockwise_with_broadcast_scales():
    """A per-row scale_a and a scale_b constant inside each 128-column block is the block-scaled
    definition with scale_a[m, kb] = s_a[m] and scale_b[kb, nb] = s_b[nb]."""
    d = wl.fp8_blockwise_inputs(16, 384, 512, seed=71)
    sa_row = d["scale_a"][:, 0].numpy().copy()
    sb_blk = d["scale_b"][0, :].numpy().copy()
    sb_col = np.repeat(sb_blk, 128)[:384]
    yr, Sr = oracle.fp8_rowwise(d["A"], d["B_t"], sa_row, sb_col)
    yb, Sb = oracle.fp8_blockwise(d["A"], d["B_t"], np.repeat(sa_row[:, None], 4, 1),
                                  np.repeat(sb_blk[None, :], 4, 0))
    assert np.all(np.abs(yr - yb) <= 1e-12 * Sb)
    np.testing.assert_allclose(Sr, Sb, rtol=1e-12)


def test_fp8_tensorwise_is_rowwise_with_constant_vectors():
    A, B, _, _, bias = _rowwise_inputs(6, 40, 256, seed=72)
    yt, St = oracle.fp8_rowwise(A, B, np.float32(0.75), np.float32(1.5), bias)
    yr, Sr = oracle.fp8_rowwise(A, B, np.full(6, 0.75, np.float32), np.full(40, 1.5, np.float32), bias)
    np.testing.assert_array_equal(yt, yr)
    np.testing.assert_array_equal(St, Sr)


def test_fp8_rowwise_small_integers_unit_scales_and_bias_per_column():
    rng = np.random.default_rng(13)
    M, N, K = 4, 24, 200
    t = oracle.e4m3_table()
    code_of = {float(v): c for c, v in reversed(list(enumerate(t))) if not np.isnan(v)}
    ints_a, ints_b = rng.integers(-4, 5, (M, K)), rng.integers(-4, 5, (N, K))
    enc = np.vectorize(lambda v: code_of[float(v)] if v != 0 else 0)
    A, B = enc(ints_a).astype(np.uint8), enc(ints_b).astype(np.uint8)
    bias = np.arange(N, dtype=np.float32) - 10.0
    y, _ = oracle.fp8_rowwise(A, B, np.ones(M, np.float32), np.ones(N, np.float32), bias)
    np.testing.assert_array_equal(y, (ints_a @ ints_b.T).astype(np.float64) + bias[None, :])
    y0, _ = oracle.fp8_rowwise(A, B, np.ones(M, np.float32), np.ones(N, np.float32))
    np.testing.assert_array_equal(y - y0, np.broadcast_to(bias.astype(np.float64), (M, N)))


def test_fp8_rowwise_scale_shapes_from_the_blockwise_issue():
    """The same compile-error message states the tensorwise (scalar) and rowwise ((16640, 1) and (1, 5120))
    scale shapes (tests/golden/scale_shapes_blockwise.json); the oracle accepts exactly those kinds."""
    g = json.load(open(os.path.join(GOLDEN, "scale_shapes_blockwise.json")))
    M, N = 2, g["N"]
    A = np.full((M, 256), 0x38, np.uint8)
    B = np.full((N, 256), 0x38, np.uint8)
    y, _ = oracle.fp8_rowwise(A, B, np.ones((M, 1), np.float32), np.ones(g["rowwise_scale_b"], np.float32))
    assert tuple(g["rowwise_scale_a"])[1] == 1 and np.all(y == 256)
    y, _ = oracle.fp8_rowwise(A, B, np.float32(2.0), np.float32(0.5))
    assert np.all(y == 256)
    with pytest.raises(AssertionError):  # blockwise-shaped scales are neither kind
        oracle.fp8_rowwise(A, B, np.ones((M, 2), np.float32), np.ones((2, 40), np.float32))


# ---------------------------------------------------------------------------
# operation 2: INT8 with fused (float(acc) * s_a) * s_b
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,N,K", [(17, 33, 64), (64, 128, 4096), (33, 24, 48)])
def test_int8_bit_exact_against_torch_int_mm_and_fp32_ops(M, N, K):
    d = wl.int8_inputs(M, N, K, seed=77 + K)
    acc, y, bf = oracle.int_scaled_mm(d["A"], d["B_t"], d["s_a"], d["s_b"])
    ref_acc = torch._int_mm(d["A"], d["B_t"].T.contiguous())
    np.testing.assert_array_equal(acc, ref_acc.numpy())
    ref_y = (ref_acc.to(torch.float32) * d["s_a"][:, None]) * d["s_b"][None, :]
    np.testing.assert_array_equal(y.view(np.uint32), ref_y.numpy().view(np.uint32))
    np.testing.assert_array_equal(bf, ref_y.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_int8_row_scale_only_is_the_cpu_definition():
    """int_scaled_matmul_cpu: c = _int_mm(a, b); c.to(scales.dtype) * scales."""
    d = wl.int8_inputs(40, 56, 96, seed=12)
    _, y, _ = oracle.int_scaled_mm(d["A"], d["B_t"], d["s_a"], None)
    c = torch._int_mm(d["A"], d["B_t"].T.contiguous())
    ref = c.to(d["s_a"].dtype) * d["s_a"][:, None]
    np.testing.assert_array_equal(y.view(np.uint32), ref.numpy().view(np.uint32))


def test_int8_scale_order_is_fixed():
    """(float(acc)*s_a)*s_b differs from float(acc)*(s_a*s_b) on some inputs;
    the oracle must follow the first."""
    d = wl.int8_inputs(64, 64, 256, seed=13)
    acc, y, _ = oracle.int_scaled_mm(d["A"], d["B_t"], d["s_a"], d["s_b"])
    f = acc.astype(np.float32)
    first = (f * d["s_a"].numpy()[:, None]) * d["s_b"].numpy()[None, :]
    other = f * (d["s_a"].numpy()[:, None] * d["s_b"].numpy()[None, :])
    np.testing.assert_array_equal(y, first)
    assert np.any(first != other)


def test_int8_unit_scales_and_overflow_detection():
    d = wl.int8_inputs(8, 8, 128, seed=14)
    acc, y, _ = oracle.int_scaled_mm(d["A"], d["B_t"], np.ones(8, np.float32), np.ones(8, np.float32))
    np.testing.assert_array_equal(y, acc.astype(np.float32))
    K = 133160  # 127*127*K > 2^31 - 1
    A = np.full((1, K), 127, np.int8)
    with pytest.raises(ValueError):
        oracle.int_scaled_mm(A, A, None, None)


# ---------------------------------------------------------------------------
# operation 3: batched GEMM with e8m0 block scales
# ---------------------------------------------------------------------------
def _e8m0(b):
    return np.ldexp(1.0, b.astype(np.int64) - 127)


@pytest.mark.parametrize("batch_first", [False, True])
def test_bmm_matches_fp64_einsum_of_bf16_dequantised_operands(batch_first):
    """Test criterion of the mxscale BMM PR: fp8 result vs a bf16 einsum.  The
    dequantised operands are exact in bf16, so the einsum is run in fp64."""
    M, G, N, K = 5, 3, 256, 384
    d = wl.bmm_inputs(M, G, N, K, seed=31, batch_first=batch_first)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    t = torch.from_numpy(oracle.e4m3_table())
    xd = t[d["x"].long()] * torch.from_numpy(_e8m0(d["x_scale"].numpy())).repeat_interleave(128, -1)
    ws = torch.from_numpy(_e8m0(d["w_scale"].numpy()))                  # [G, NB, KB]
    wd = t[d["w"].long()] * ws.repeat_interleave(128, 1).repeat_interleave(128, 2)
    assert torch.equal(xd.to(torch.bfloat16).double(), xd) and torch.equal(wd.to(torch.bfloat16).double(), wd)
    ref = torch.einsum("mgk,gnk->mgn", xd.to(torch.bfloat16).double(), wd.to(torch.bfloat16).double()).numpy()
    assert np.all(np.abs(y - ref) <= 1e-12 * S + 1e-300)


def test_bmm_equals_per_g_blockwise_with_transposed_w_scale():
    M, G, N, K = 4, 2, 256, 256
    d = wl.bmm_inputs(M, G, N, K, seed=32)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    for g in range(G):
        sa = _e8m0(d["x_scale"][:, g, :].numpy()).astype(np.float32)
        sb = _e8m0(d["w_scale"][g].numpy()).T.astype(np.float32)     # [KB, NB]
        yg, Sg = oracle.fp8_blockwise(d["x"][:, g, :].contiguous(), d["w"][g], sa, sb)
        np.testing.assert_array_equal(y[:, g, :], yg)
        np.testing.assert_array_equal(S[:, g, :], Sg)


def test_bmm_layouts_agree_and_one_hot_w_scale():
    M, G, N, K = 3, 2, 256, 256
    a = wl.bmm_inputs(M, G, N, K, seed=33)
    b = wl.bmm_inputs(M, G, N, K, seed=33, batch_first=True)
    ya, _ = oracle.bmm_blockscale(a["x"], a["w"], a["x_scale"], a["w_scale"])
    yb, _ = oracle.bmm_blockscale(b["x"], b["w"], b["x_scale"], b["w_scale"])
    np.testing.assert_array_equal(ya, yb)
    # all scales 2^0 except block (g=1, nb=1, kb=0) at 2^3: only that block moves, by exactly 8
    xs = np.full(a["x_scale"].shape, 127, np.uint8)
    ws = np.full(a["w_scale"].shape, 127, np.uint8)
    y1, _ = oracle.bmm_blockscale(a["x"], a["w"], xs, ws)
    ws[1, 1, 0] = 130
    y2, _ = oracle.bmm_blockscale(a["x"], a["w"], xs, ws)
    ai = _int_codes(a["x"][:, 1, :128].numpy())
    bi = _int_codes(a["w"][1, 128:256, :128].numpy())
    delta = (ai @ bi.T).astype(np.float64) * 2.0 ** -18 * 7.0
    np.testing.assert_array_equal(y2[:, 1, 128:] - y1[:, 1, 128:], delta)
    np.testing.assert_array_equal(y2[:, 0, :], y1[:, 0, :])
    np.testing.assert_array_equal(y2[:, 1, :128], y1[:, 1, :128])


def test_oracle_rows_subset_matches_full():
    d = wl.fp8_blockwise_inputs(40, 256, 256, seed=8)
    y, S = oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"])
    ys, Ss = oracle.fp8_blockwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"], rows=[39, 0, 17])
    np.testing.assert_array_equal(ys, y[[39, 0, 17]])
    np.testing.assert_array_equal(Ss, S[[39, 0, 17]])


# ---------------------------------------------------------------------------
# e4m3 encoding and the 1x128 activation quantiser (fused-quantiser operation)
# ---------------------------------------------------------------------------
def _finite_magnitudes():
    t = oracle.e4m3_table()
    return t[:127]  # codes 0..126: 0, subnormals, normals up to 448, ascending


def test_e4m3_encode_round_trips_every_finite_code():
    t = oracle.e4m3_table()
    codes = np.array([c for c in range(256) if not math.isnan(t[c])], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(t[codes]), codes)


def test_e4m3_encode_midpoints_go_to_the_even_code_and_neighbours_to_the_nearest():
    mags = _finite_magnitudes()
    for c in range(126):
        lo, hi = mags[c], mags[c + 1]
        mid = (lo + hi) / 2  # exact in fp64
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode([mid])[0] == even, (c, mid)
        assert oracle.e4m3_encode([-mid])[0] == 0x80 | even
        assert oracle.e4m3_encode([np.nextafter(mid, 0)])[0] == c
        assert oracle.e4m3_encode([np.nextafter(mid, 1e9)])[0] == c + 1


def test_e4m3_encode_saturates_and_keeps_nan():
    enc = oracle.e4m3_encode([448.0, 460.0, 464.0, 1e30, -1e30, -448.0, float("nan")])
    assert list(enc) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


def test_e4m3_encode_agrees_with_torch_cast_inside_the_range():
    g = torch.Generator().manual_seed(7)
    v = (torch.randn(200000, generator=g, dtype=torch.float64) * torch.pow(2.0, torch.randint(-12, 9, (200000,), generator=g)))
    v = v.clamp(-448, 448)
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v.numpy()), ref)


def _torch_quantize_f32(x):
    """The recipe through torch's own cast: scale = amax / 448 (1 if 0), codes = cast(sat(x / scale))."""
    M, K = x.shape
    KB = -(-K // 128)
    xp = torch.zeros(M, KB * 128)
    xp[:, :K] = x
    amax = xp.view(M, KB, 128).abs().amax(-1)
    s = amax / 448.0
    s[s == 0] = 1.0
    q = (xp / s.repeat_interleave(128, 1)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    return q[:, :K].numpy(), s.numpy()


@pytest.mark.parametrize("M,K", [(3, 128), (5, 300), (2, 1000)])
def test_quantize_fp32_scale_matches_torch_cast_of_x_over_scale(M, K):
    x = wl.normal_with_outliers((M, K), 4321 + K)
    q, s = oracle.quantize_1x128(x, 0)
    rq, rs = _torch_quantize_f32(x)
    assert s.dtype == np.float32 and s.shape == (M, -(-K // 128))
    assert np.array_equal(s, rs) and np.array_equal(q, rq)


def test_quantize_group_amax_maps_to_448_and_zero_groups_get_scale_one():
    x = torch.zeros(2, 256)
    x[0, :128] = torch.linspace(-3.0, 2.0, 128)
    x[1, 128:] = torch.linspace(0.5, 7.0, 128)
    q, s = oracle.quantize_1x128(x, 0)
    assert q[0, 0] == 0xFE  # -3.0 is the group's amax, negative
    assert q[1, 255] == 0x7E
    assert s[0, 1] == 1.0 and s[1, 0] == 1.0 and np.all(q[0, 128:] == 0) and np.all(q[1, :128] == 0)
    assert s[0, 0] == np.float32(3.0) / np.float32(448.0)
    # a 1x128 group is one scale: rows and groups do not mix
    q2, s2 = oracle.quantize_1x128(x[:, :128], 0)
    assert np.array_equal(q2, q[:, :128]) and np.array_equal(s2[:, 0], s[:, 0])


def test_quantize_scale_that_underflows_takes_the_zero_group_scale():
    """amax / 448 is computed in fp32: below 448 * 2^-150 it rounds to zero, and
    such a group takes scale 1 like an all-zero group (its codes are e4m3(x),
    zero here) instead of dividing by zero.  Just above, the scale is the
    smallest fp32 subnormal and the amax element still maps to x / 2^-149."""
    x = torch.zeros(3, 128)
    x[0, :5] = torch.tensor([2.0 ** -142, -2.0 ** -143, 2.0 ** -149, 0.0, -2.0 ** -142])  # quotient 2^-150.8 -> 0
    x[1, 0] = 2.0 ** -141                      # quotient 0.57 * 2^-149 -> the smallest subnormal
    x[1, 1] = -2.0 ** -145
    q, s = oracle.quantize_1x128(x, 0)
    table = oracle.e4m3_table()
    assert np.float32(np.float32(2.0 ** -142) / np.float32(448.0)) == 0.0  # the underflow itself
    assert s[0, 0] == 1.0 and np.all(table[q[0]] == 0.0)  # +-0 codes
    assert q[0, 1] == 0x80 and q[0, 0] == 0x00              # the signs survive
    assert s[1, 0] == np.float32(2.0 ** -149)
    assert table[q[1, 0]] == 256.0 and table[q[1, 1]] == -16.0
    assert s[2, 0] == 1.0 and np.all(q[2] == 0)  # all-zero group
    assert not np.any(np.isin(q, [0x7F, 0xFF]))
    # the transposed quantiser follows the same rule (128 x 1 groups of x^T)
    qt, st = oracle.quantize_t(x.t().contiguous(), 0, 0)
    assert np.array_equal(qt, q) and np.array_equal(st, s)


def test_quantize_e8m0_exponent_at_and_around_448_times_powers_of_two():
    cases = []
    for k in (-20, -3, 0, 1, 5, 40):
        exact = 448.0 * 2.0 ** k
        cases += [(exact, 127 + k),
                  (float(np.nextafter(np.float32(exact), np.float32(1e38))), 128 + k),
                  (float(np.float32(exact * 0.6)), 127 + k),
                  (float(np.float32(exact * 0.5)), 126 + k)]
    x = torch.zeros(len(cases), 128)
    for i, (amax, _) in enumerate(cases):
        x[i, 0] = amax
        x[i, 1] = -amax / 3
    q, e = oracle.quantize_1x128(x, 1)
    assert [int(b) for b in e[:, 0]] == [b for _, b in cases]
    for i, (amax, byte) in enumerate(cases):
        assert q[i, 0] == oracle.e4m3_encode([amax * 2.0 ** -(byte - 127)])[0]
    assert oracle.quantize_1x128(torch.zeros(1, 128), 1)[1][0, 0] == 127


@pytest.mark.parametrize("M,K", [(4, 256), (3, 777)])
def test_quantize_e8m0_matches_the_bmm_recipe_through_torch_cast(M, K):
    x = wl.normal_with_outliers((M, K), 99 + K)
    q, e = oracle.quantize_1x128(x, 1)
    KB = -(-K // 128)
    xp = torch.zeros(M, KB * 128)
    xp[:, :K] = x
    amax = xp.view(M, KB, 128).abs().amax(-1).double()
    # ceil(log2(amax / 448)) in exact rational arithmetic
    want = np.zeros((M, KB), dtype=np.int64)
    for i in range(M):
        for g in range(KB):
            a = Fraction(float(amax[i, g]))
            ee = 0
            if a > 0:
                ee = math.floor(math.log2(float(a / 448))) - 2
                while a > 448 * Fraction(2) ** ee:
                    ee += 1
            want[i, g] = min(max(ee + 127, 0), 254)
    assert np.array_equal(e.astype(np.int64), want)
    sc = torch.pow(2.0, -(torch.tensor(want, dtype=torch.float64) - 127)).repeat_interleave(128, 1)
    ref = (xp.double() * sc).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)[:, :K].numpy()
    assert np.array_equal(q, ref)


# ---------------------------------------------------------------------------
# transposed-output quantiser for the backward GEMMs (128x1 and 128x128 groups)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("R,C", [(128, 3), (300, 5), (1000, 2)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_t_128x1_is_the_1x128_quantiser_of_the_transpose(R, C, fmt):
    x = wl.normal_with_outliers((R, C), 77 + R + C)
    q, s = oracle.quantize_t(x, 0, fmt)
    rq, rs = oracle.quantize_1x128(x.t().contiguous(), fmt)
    assert q.shape == (C, R) and s.shape == (C, -(-R // 128))
    assert np.array_equal(q, rq) and np.array_equal(s, rs)


def _torch_quantize_128x128_t(x):
    """128x128 blocks through torch's own cast, codes transposed: scale = amax / 448 (1 if 0)."""
    R, C = x.shape
    RB, CB = -(-R // 128), -(-C // 128)
    xp = torch.zeros(RB * 128, CB * 128)
    xp[:R, :C] = x
    amax = xp.view(RB, 128, CB, 128).abs().amax(dim=(1, 3))
    s = amax / 448.0
    s[s == 0] = 1.0
    full = s.repeat_interleave(128, 0).repeat_interleave(128, 1)
    q = (xp / full).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    return q[:R, :C].t().contiguous().numpy(), s.numpy()


@pytest.mark.parametrize("R,C", [(128, 128), (300, 200), (256, 1000)])
def test_quantize_t_128x128_matches_torch_cast_of_x_over_block_scale(R, C):
    x = wl.normal_with_outliers((R, C), 55 + R + C)
    q, s = oracle.quantize_t(x, 1, 0)
    rq, rs = _torch_quantize_128x128_t(x)
    assert s.dtype == np.float32 and s.shape == (-(-R // 128), -(-C // 128))
    assert np.array_equal(s, rs) and np.array_equal(q, rq)


def test_quantize_t_orientation_block_amax_and_isolation():
    x = torch.zeros(256, 256)
    x[3, 200] = -5.0  # block (0, 1): its amax, negative
    x[130, 7] = 2.0   # block (1, 0)
    x[131, 8] = 1.0
    q, s = oracle.quantize_t(x, 1, 0)
    assert q[200, 3] == 0xFE and q[7, 130] == 0x7E  # q_t[c, r] is the code of x[r, c]
    assert q[8, 131] == oracle.e4m3_encode([1.0 / float(np.float32(2.0) / np.float32(448.0))])[0]
    assert s[0, 0] == 1.0 and s[1, 1] == 1.0  # all-zero blocks
    assert s[0, 1] == np.float32(5.0) / np.float32(448.0) and s[1, 0] == np.float32(2.0) / np.float32(448.0)
    assert int(np.count_nonzero(q)) == 3
    # 128x1: each column of a 128-row block is its own group
    q1, s1 = oracle.quantize_t(x, 0, 0)
    assert q1[7, 130] == 0x7E and q1[8, 131] == 0x7E and s1[8, 1] == np.float32(1.0) / np.float32(448.0)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_t_block_scale_is_the_largest_column_scale_of_the_block(fmt):
    # amax / 448 and ceil(log2(amax / 448)) are monotone in amax: a block's
    # scale is the largest 128x1 scale among its columns, and the column that
    # holds the block amax gets identical codes either way
    x = wl.normal_with_outliers((384, 256), 31 + fmt)
    qb, sb = oracle.quantize_t(x, 1, fmt)
    qc, sc = oracle.quantize_t(x, 0, fmt)
    for rb in range(3):
        for cb in range(2):
            cols = sc[128 * cb:128 * cb + 128, rb]
            assert sb[rb, cb] == cols.max()
            c = 128 * cb + int(np.argmax(cols))
            assert np.array_equal(qb[c, 128 * rb:128 * rb + 128], qc[c, 128 * rb:128 * rb + 128])


def test_backward_gemms_of_the_quantised_operands_approximate_the_exact_gradients():
    # dW = dy^T x and dx = dy W through the transposed quantiser: e4m3 keeps 3
    # mantissa bits, so the result is the exact gradient within a few percent
    # (a transposed or misgrouped operand gives an unrelated matrix)
    M, N, K = 256, 128, 384
    x = wl.normal_with_outliers((M, K), 901)
    dy = wl.normal_with_outliers((M, N), 902)
    W = wl.normal_with_outliers((N, K), 903)
    xd, dyd, Wd = x.double().numpy(), dy.double().numpy(), W.double().numpy()
    a, sa = oracle.quantize_t(dy, 0, 0)
    b, sb = oracle.quantize_t(x, 1, 0)
    dW, _ = oracle.fp8_blockwise(a, b, sa, sb)
    a2, sa2 = oracle.quantize_1x128(dy, 0)
    b2, sb2 = oracle.quantize_t(W, 1, 0)
    dx, _ = oracle.fp8_blockwise(a2, b2, sa2, sb2)
    for got, want in ((dW, dyd.T @ xd), (dx, dyd @ Wd)):
        assert got.shape == want.shape
        assert np.linalg.norm(got - want) / np.linalg.norm(want) < 0.06


# ---------------------------------------------------------------------------
# forward-orientation 128x128 quantiser (the weight operand B_t [N, K])
# ---------------------------------------------------------------------------
def _torch_quantize_blocks(x):
    """torch's own cast of x over its 128x128 block's scale (amax / 448, 1 if that is 0)."""
    R, C = x.shape
    RB, CB = -(-R // 128), -(-C // 128)
    xp = torch.zeros(RB * 128, CB * 128)
    xp[:R, :C] = x
    amax = xp.view(RB, 128, CB, 128).abs().amax(dim=(1, 3))
    s = amax / 448.0
    s[s == 0] = 1.0
    full = s.repeat_interleave(128, 0).repeat_interleave(128, 1)
    q = (xp / full).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    return q[:R, :C].numpy(), s.numpy()


@pytest.mark.parametrize("R,C", [(128, 128), (300, 260), (5, 700), (1000, 1), (256, 384)])
def test_quantize_128x128_matches_torch_cast_of_x_over_block_scale(R, C):
    x = wl.normal_with_outliers((R, C), 9100 + R + C)
    q, s = oracle.quantize_128x128(x, 0)
    rq, rs = _torch_quantize_blocks(x)
    assert q.shape == (R, C) and s.shape == (-(-R // 128), -(-C // 128))
    assert np.array_equal(s, rs) and np.array_equal(q, rq)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_128x128_is_the_transposed_quantiser_transposed_back(fmt):
    x = wl.normal_with_outliers((300, 520), 9200 + fmt)
    q, s = oracle.quantize_128x128(x, fmt)
    qt, st = oracle.quantize_t(x, 1, fmt)  # codes [C, R], block scales [RB, CB]
    assert np.array_equal(q, qt.T) and np.array_equal(s, st)


def test_quantize_128x128_orientation_and_block_isolation():
    x = torch.zeros(256, 384)
    x[5, 200] = 7.0     # block (0, 1): rows 0..127, columns 128..255
    x[130, 3] = -2.0    # block (1, 0)
    q, s = oracle.quantize_128x128(x, 0)
    assert s[0, 1] == np.float32(7.0) / np.float32(448.0) and s[1, 0] == np.float32(2.0) / np.float32(448.0)
    assert s[0, 0] == 1.0 and s[1, 1] == 1.0 and s[0, 2] == 1.0 and s[1, 2] == 1.0
    assert q[5, 200] == 0x7E and q[130, 3] == 0xFE      # +-448
    assert int(np.count_nonzero(q)) == 2
    # e8m0: the byte of the block holding 7.0 is ceil(log2(7 / 448)) + 127 = -6 + 127
    _, b = oracle.quantize_128x128(x, 1)
    assert b[0, 1] == 121 and b[0, 0] == 127


def test_quantize_128x128_weight_in_the_forward_gemm_approximates_the_exact_product():
    M, N, K = 200, 384, 640
    x = wl.normal_with_outliers((M, K), 9300)
    W = wl.normal_with_outliers((N, K), 9301)
    a, sa = oracle.quantize_1x128(x, 0)
    b, sbT = oracle.quantize_128x128(W, 0)  # B_t [N, K], scales [N/128, K/128]
    y, _ = oracle.fp8_blockwise(a, b, sa, sbT.T)
    exact = x.double().numpy() @ W.double().numpy().T
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert rel < 0.06, rel

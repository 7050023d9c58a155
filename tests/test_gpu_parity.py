"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Inputs come from the seeded generators in ``workloads``; expected values come
only from ``oracle``.  FP8 results must meet the bound documented in
tests/parity.py; INT8 results must be bit-exact.  Small shapes compare every
element; the full-size shapes compare sampled rows (all columns) that cover
several tiles and the ragged tail.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import int8_gemm_b200 as bs
import oracle
import workloads as wl
from parity import (assert_quantised, bf16_bits, e4m3_check, f32_bits, fp8_check, oracle_fp8, rows_sample,
                    to_f64)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    bs.lib()
    yield
    assert bs.device_error() == 0, "a kernel reported a timed-out wait"


@pytest.fixture
def path():
    """Force a kernel family for one test, restoring automatic choice after."""
    def set_(p):
        bs.set_path_override(p)
    yield set_
    bs.set_path_override(bs.PATH_AUTO)


def fp8_run(d, out_dtype=torch.bfloat16, out=None):
    A = d["A"].to(DEV)
    B = d["B_t"].to(DEV).t()
    return bs.bs_gemm_fp8_blockwise(A, B, d["scale_a"].to(DEV), d["scale_b"].to(DEV), out_dtype=out_dtype, out=out)


# ---------------------------------------------------------------------------
# operation 1: FP8 block-scaled
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fp8_tiny_full_matrix(out_dtype):
    w = wl.WORKLOADS["fp8_tiny_256x256x512"]
    d = wl.workload_inputs(w)
    y, S = oracle_fp8(d)
    fp8_check(fp8_run(d, out_dtype), y, S, out_dtype, "fp8 256x256x512")


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (129, 384, 256), (300, 520, 640), (1, 256, 128),
                                   (255, 128, 1024), (640, 1280, 384)])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_SINGLE, bs.PATH_SKINNY])
def test_fp8_ragged_shapes_all_kernels(M, N, K, kernel, path):
    path(kernel)
    d = wl.fp8_blockwise_inputs(M, N, K, seed=50 + M + N + K)
    y, S = oracle_fp8(d)
    fp8_check(fp8_run(d), y, S, torch.bfloat16, f"fp8 {M}x{N}x{K} kernel={kernel}")


@pytest.mark.parametrize("M,N,K", [(5, 259, 512), (200, 131, 256), (70, 1001, 1024), (33, 4099, 256)])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_SINGLE, bs.PATH_SKINNY])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fp8_n_not_multiple_of_four(M, N, K, kernel, out_dtype, path):
    """Output rows padded in memory (16-byte row starts), partial 4-wide and
    16-byte groups at the end of every row."""
    path(kernel)
    d = wl.fp8_blockwise_inputs(M, N, K, seed=90 + M + N + K)
    y, S = oracle_fp8(d)
    out = fp8_run(d, out_dtype)
    assert out.shape == (M, N) and (out.stride(0) * out.element_size()) % 16 == 0
    fp8_check(out, y, S, out_dtype, f"fp8 {M}x{N}x{K} kernel={kernel}")


@pytest.mark.parametrize("M,N,K", [(70, 640, 4096), (128, 1032, 4096), (33, 256, 8192)])
def test_fp8_skinny_long_k_32_row_tiles(M, N, K):
    """Long K: the planner takes 32-row activation tiles (several per M, the
    last one ragged) and splits K up to eight ways."""
    d = wl.fp8_blockwise_inputs(M, N, K, seed=95 + M + N)
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, M, 1, N, K, torch.cuda.get_device_properties(0).multi_processor_count)
    assert p["kernel"] == 2 and p["tile_m"] == 32
    y, S = oracle_fp8(d)
    fp8_check(fp8_run(d), y, S, torch.bfloat16, f"fp8 {M}x{N}x{K} 32-row tiles split {p['splits']}")


@pytest.mark.parametrize("M", wl.SKINNY_M_SWEEP)
def test_fp8_skinny_sweep_n7168_k2048(M):
    w = wl.WORKLOADS[f"fp8_skinny_m{M}"]
    d = wl.workload_inputs(w, sweep=wl.sweep_index(wl.SKINNY_M_SWEEP, M))
    out = fp8_run(d)
    rows = None if M <= 255 else rows_sample(M)
    y, S = oracle_fp8(d, rows=rows)
    got = out if rows is None else out[torch.tensor(rows, device=DEV)]
    fp8_check(got, y, S, torch.bfloat16, f"skinny M={M}")


@pytest.mark.slow
def test_fp8_full_size_16640x5120x8192_sampled_rows():
    w = wl.WORKLOADS["fp8_16640x5120x8192"]
    d = wl.workload_inputs(w)
    out = fp8_run(d)
    rows = rows_sample(w.M, extra=6)
    y, S = oracle_fp8(d, rows=rows)
    fp8_check(out[torch.tensor(rows, device=DEV)], y, S, torch.bfloat16, "fp8 16640x5120x8192")


def test_fp8_power_of_two_scale_linearity_on_gpu():
    d = wl.fp8_blockwise_inputs(256, 512, 512, seed=61)
    base = fp8_run(d, torch.float32)
    d2 = dict(d)
    sa = d["scale_a"].clone()
    sa[5, :] *= 2.0 ** 4
    d2["scale_a"] = sa
    moved = fp8_run(d2, torch.float32)
    assert torch.equal(moved[5], base[5] * 16.0)
    keep = torch.ones(256, dtype=torch.bool, device=DEV)
    keep[5] = False
    assert torch.equal(moved[keep], base[keep])


def test_fp8_deterministic_and_no_out_of_bounds_writes():
    M, N, K = 300, 512, 1024
    d = wl.fp8_blockwise_inputs(M, N, K, seed=62)
    canvas = torch.full((M + 3, N + 64), 7.0, dtype=torch.bfloat16, device=DEV)
    view = canvas[1:M + 1, 8:N + 8]
    fp8_run(d, out=view)
    first = view.clone()
    fp8_run(d, out=view)
    assert torch.equal(first, view)
    assert torch.all(canvas[0] == 7.0) and torch.all(canvas[M + 1:] == 7.0)
    assert torch.all(canvas[:, :8] == 7.0) and torch.all(canvas[:, N + 8:] == 7.0)
    y, S = oracle_fp8(d)
    fp8_check(view, y, S, torch.bfloat16, "fp8 strided out")


def test_fp8_empty_and_k0():
    A = torch.zeros(0, 128, dtype=torch.uint8, device=DEV)
    B = torch.zeros(256, 128, dtype=torch.uint8, device=DEV).t()
    out = bs.bs_gemm_fp8_blockwise(A, B, torch.ones(0, 1, device=DEV), torch.ones(1, 2, device=DEV))
    assert out.shape == (0, 256)
    A = torch.zeros(5, 0, dtype=torch.uint8, device=DEV)
    B = torch.zeros(256, 0, dtype=torch.uint8, device=DEV).t()
    out = torch.full((5, 256), 3.0, dtype=torch.bfloat16, device=DEV)
    bs.bs_gemm_fp8_blockwise(A, B, torch.ones(5, 0, device=DEV), torch.ones(0, 2, device=DEV), out=out)
    assert torch.all(out == 0)


def test_fp8_transposed_scale_a_layout():
    d = wl.fp8_blockwise_inputs(256, 256, 512, seed=63)
    y, S = oracle_fp8(d)
    sa_colmajor = d["scale_a"].t().contiguous().to(DEV).t()  # [M, KB] with strides (1, M)
    out = bs.bs_gemm_fp8_blockwise(d["A"].to(DEV), d["B_t"].to(DEV).t(), sa_colmajor, d["scale_b"].to(DEV))
    fp8_check(out, y, S, torch.bfloat16, "column-major scale_a")


# ---------------------------------------------------------------------------
# FP8 with tensorwise / rowwise scales and bias
# ---------------------------------------------------------------------------
def rowwise_run(d, out_dtype=torch.bfloat16, bias=True, out=None, scale_result=None):
    b = d["bias"].to(DEV) if (bias and d["bias"] is not None) else None
    sr = None if scale_result is None else torch.tensor(scale_result, dtype=torch.float32, device=DEV)
    return bs.bs_gemm_fp8_rowwise(d["A"].to(DEV), d["B_t"].to(DEV).t(), d["scale_a"].to(DEV), d["scale_b"].to(DEV), b,
                                  out_dtype=out_dtype, out=out, scale_result=sr)


def oracle_rowwise(d, bias=True, rows=None):
    return oracle.fp8_rowwise(d["A"], d["B_t"], d["scale_a"], d["scale_b"], d["bias"] if bias else None, rows=rows)


@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (300, 520, 640), (1, 256, 128), (129, 384, 176), (640, 1280, 1024),
                                   (5, 259, 48), (2300, 2100, 256)])
@pytest.mark.parametrize("tensorwise", [False, True])
@pytest.mark.parametrize("kernel", [bs.PATH_AUTO, bs.PATH_WIDE_SINGLE])
def test_fp8_rowwise_and_tensorwise(M, N, K, tensorwise, kernel, path):
    path(kernel)
    d = wl.fp8_rowwise_inputs(M, N, K, seed=140 + M + N + K, tensorwise=tensorwise)
    for out_dtype in (torch.bfloat16, torch.float32):
        for bias in (True, False):
            y, S = oracle_rowwise(d, bias)
            fp8_check(rowwise_run(d, out_dtype, bias), y, S, out_dtype,
                      f"fp8 rowwise {M}x{N}x{K} tensorwise={tensorwise} bias={bias}")


@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (300, 520, 640), (1, 256, 128), (129, 384, 176), (5, 259, 48)])
@pytest.mark.parametrize("tensorwise", [False, True])
@pytest.mark.parametrize("kernel", [bs.PATH_AUTO, bs.PATH_WIDE_SINGLE])
def test_fp8_rowwise_e4m3_output_with_scale_result(M, N, K, tensorwise, kernel, path):
    path(kernel)
    d = wl.fp8_rowwise_inputs(M, N, K, seed=160 + M + N + K, tensorwise=tensorwise)
    for bias in (True, False):
        y, S = oracle_rowwise(d, bias)
        top = float(np.abs(y).max())
        # no output scale; one that maps the largest |y| to 300 (no saturation);
        # one that maps it to 3000, so the largest outputs saturate at +-448
        for s_r in (None, np.float32(300.0 / top), np.float32(3000.0 / top)):
            out = rowwise_run(d, torch.float8_e4m3fn, bias, scale_result=None if s_r is None else float(s_r))
            assert out.dtype == torch.float8_e4m3fn and tuple(out.shape) == (M, N)
            same = e4m3_check(out, y, S, 1.0 if s_r is None else float(s_r),
                              f"fp8 rowwise e4m3 {M}x{N}x{K} tensorwise={tensorwise} bias={bias} s_r={s_r}")
            assert same > 0.97, f"only {same:.3f} of codes equal the oracle's rounding"
        sat = rowwise_run(d, torch.float8_e4m3fn, bias, scale_result=float(np.float32(3000.0 / top)))
        assert float(sat.float().abs().max()) == 448.0


def test_fp8_rowwise_e4m3_output_k0_and_use_fast_accum():
    bias = torch.randn(208, generator=torch.Generator().manual_seed(161)).to(DEV) * 100
    A = torch.zeros(16, 0, dtype=torch.uint8, device=DEV)
    B = torch.zeros(208, 0, dtype=torch.uint8, device=DEV).t()
    sr = torch.tensor([2.0], device=DEV)  # a power of two: the fp32 product is exact
    out = bs.bs_gemm_fp8_rowwise(A, B, torch.ones(16, 1, device=DEV), torch.ones(1, 208, device=DEV), bias,
                                 out_dtype=torch.float8_e4m3fn, scale_result=sr)
    want = oracle.e4m3_encode(2.0 * bias.cpu().double().numpy())  # |2 bias| reaches past 448: saturation too
    assert np.array_equal(out.cpu().view(torch.uint8).numpy(), np.broadcast_to(want, (16, 208)))
    # use_fast_accum selects nothing on this hardware: the results are identical
    d = wl.fp8_rowwise_inputs(300, 512, 1024, seed=162)
    for dt in (torch.bfloat16, torch.float8_e4m3fn):
        a = bs.bs_gemm_fp8_rowwise(d["A"].to(DEV), d["B_t"].to(DEV).t(), d["scale_a"].to(DEV), d["scale_b"].to(DEV),
                                   d["bias"].to(DEV), out_dtype=dt, use_fast_accum=True)
        b = rowwise_run(d, dt)
        assert torch.equal(a.view(torch.uint8) if dt != torch.bfloat16 else a,
                           b.view(torch.uint8) if dt != torch.bfloat16 else b)
    with pytest.raises(bs.BsgemmError):  # an output scale is only defined for an e4m3 result
        rowwise_run(d, torch.bfloat16, scale_result=2.0)


def test_fp8_rowwise_k0_writes_bias_and_is_deterministic():
    bias = torch.randn(200, generator=torch.Generator().manual_seed(150)).to(DEV)
    A = torch.zeros(64, 0, dtype=torch.uint8, device=DEV)
    B = torch.zeros(200, 0, dtype=torch.uint8, device=DEV).t()
    out = bs.bs_gemm_fp8_rowwise(A, B, torch.ones(64, 1, device=DEV), torch.ones(1, 200, device=DEV), bias,
                                 out_dtype=torch.float32)
    assert torch.equal(out, bias.expand(64, 200))
    out = bs.bs_gemm_fp8_rowwise(A, B, torch.ones((), device=DEV), torch.ones((), device=DEV), None)
    assert torch.all(out == 0)
    d = wl.fp8_rowwise_inputs(300, 512, 1024, seed=151)
    first = rowwise_run(d)
    assert torch.equal(first, rowwise_run(d))


@pytest.mark.slow
def test_fp8_rowwise_16640x5120x8192_sampled_rows():
    w = wl.WORKLOADS["fp8_rowwise_16640x5120x8192"]
    d = wl.workload_inputs(w)
    out = rowwise_run(d)
    rows = rows_sample(w.M, extra=6)
    y, S = oracle_rowwise(d, rows=rows)
    fp8_check(out[torch.tensor(rows, device=DEV)], y, S, torch.bfloat16, "fp8 rowwise 16640x5120x8192")
    s_r = float(np.float32(400.0 / float(np.abs(y).max())))
    out8 = rowwise_run(d, torch.float8_e4m3fn, scale_result=s_r)
    e4m3_check(out8[torch.tensor(rows, device=DEV)], y, S, s_r, "fp8 rowwise e4m3 16640x5120x8192")


# ---------------------------------------------------------------------------
# operation 2: INT8, bit-exact
# ---------------------------------------------------------------------------
def int8_run(d, out_dtype, s_b=True):
    return bs.int_scaled_mm(d["A"].to(DEV), d["B_t"].to(DEV).t(), d["s_a"].to(DEV),
                            d["s_b"].to(DEV) if s_b else None, out_dtype=out_dtype)


def _int8_assert(d, rows, s_b=True):
    acc, y, bf = oracle.int_scaled_mm(d["A"], d["B_t"], d["s_a"], d["s_b"] if s_b else None, rows=rows)
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.tensor(rows, device=DEV)])
    np.testing.assert_array_equal(sel(int8_run(d, torch.int32, s_b)).cpu().numpy(), acc)
    np.testing.assert_array_equal(f32_bits(sel(int8_run(d, torch.float32, s_b))), y.view(np.uint32))
    np.testing.assert_array_equal(bf16_bits(sel(int8_run(d, torch.bfloat16, s_b))), bf)


# (2300, 2100, 512): 81 ragged tiles, so some CTA pairs run two tiles and reuse their staging buffers and
# staged column scales across tiles
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (300, 520, 1040), (1, 256, 4096), (257, 264, 48),
                                   (600, 1024, 2048), (2300, 2100, 512)])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_SINGLE])
def test_int8_bit_exact_small(M, N, K, kernel, path):
    path(kernel)
    _int8_assert(wl.int8_inputs(M, N, K, seed=70 + M), rows=None)


def test_int8_row_scale_only():
    _int8_assert(wl.int8_inputs(200, 256, 512, seed=71), rows=None, s_b=False)


def test_int8_4096_cubed_sampled_rows():
    w = wl.WORKLOADS["int8_4096x4096x4096"]
    d = wl.workload_inputs(w)
    _int8_assert(d, rows=rows_sample(w.M, extra=8))


# ---------------------------------------------------------------------------
# operation 3: batched, e8m0 block scales
# ---------------------------------------------------------------------------
def bmm_run(d, out_dtype=torch.bfloat16):
    return bs.bmm_a8w8_blockscale(d["x"].to(DEV) if d["x"].is_contiguous() else _batch_first_to(d["x"]),
                                  d["w"].to(DEV), d["x_scale"].to(DEV), d["w_scale"].to(DEV), out_dtype=out_dtype)


def _batch_first_to(x):
    # keep the [G, M, K] storage on the device: copy the storage, then view as [M, G, K]
    return x.permute(1, 0, 2).contiguous().to(DEV).permute(1, 0, 2)


@pytest.mark.parametrize("G", wl.BMM_G)
@pytest.mark.parametrize("M", wl.BMM_M_SWEEP)
def test_bmm_sweep(M, G):
    w = wl.WORKLOADS[f"bmm_g{G}_m{M}"]
    d = wl.workload_inputs(w, sweep=wl.sweep_index(wl.BMM_M_SWEEP, M) + 10 * (G == 2))
    out = bmm_run(d)
    rows = None if M <= 1024 else rows_sample(M, extra=4)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"], rows=rows)
    got = out if rows is None else out[torch.tensor(rows, device=DEV)]
    fp8_check(got, y, S, torch.bfloat16, f"bmm M={M} G={G}")


@pytest.mark.parametrize("M", [16, 300])
def test_bmm_batch_first_layout(M):
    d = wl.bmm_inputs(M, 2, 512, 1024, seed=80 + M, batch_first=True)
    assert not d["x"].is_contiguous()
    out = bmm_run(d, torch.float32)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    fp8_check(out, y, S, torch.float32, f"bmm batch-first M={M}")


@pytest.mark.parametrize("M,G,N", [(3, 4, 300), (100, 2, 130)])
def test_bmm_n_not_multiple_of_four(M, G, N, path):
    d = wl.bmm_inputs(M, G, N, 512, seed=85 + M + N)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    for k in (bs.PATH_WIDE, bs.PATH_SKINNY):
        path(k)
        fp8_check(bmm_run(d), y, S, torch.bfloat16, f"bmm {M}x{G}x{N} kernel={k}")


def test_bmm_both_kernels_agree_with_oracle(path):
    d = wl.bmm_inputs(200, 3, 384, 512, seed=81)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    for k in (bs.PATH_WIDE, bs.PATH_WIDE_PROMOTE, bs.PATH_WIDE_SINGLE, bs.PATH_SKINNY):
        path(k)
        fp8_check(bmm_run(d), y, S, torch.bfloat16, f"bmm kernel={k}")


@pytest.mark.parametrize("M,G,N,K", [(300, 2, 520, 640), (1024, 3, 264, 1280), (513, 1, 1024, 4096)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_bmm_block_scaled_mma_and_promotion(M, G, N, K, out_dtype, path):
    """CTA pairs apply the e8m0 scales in the tensor core (block-scaled MMA);
    path 4 promotes every 128-deep block on the CUDA cores instead.  Both meet
    the bound, on ragged M, N and K tails and partial column blocks."""
    d = wl.bmm_inputs(M, G, N, K, seed=86 + M + N + K)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    for k in (bs.PATH_WIDE, bs.PATH_WIDE_PROMOTE):
        path(k)
        fp8_check(bmm_run(d, out_dtype), y, S, out_dtype, f"bmm {M}x{G}x{N}x{K} kernel={k}")


# ---------------------------------------------------------------------------
# fused quantiser: 1x128 groups to e4m3 with fp32 or e8m0 scales (bit-exact)
# ---------------------------------------------------------------------------
def _quant_check(x_dev, fmt, rows=None, **kw):
    q, s = bs.quantize_fp8_1x128(x_dev, "f32" if fmt == 0 else "e8m0", **kw)
    if rows is not None:
        r = torch.as_tensor(rows, device=x_dev.device)
        x_dev, q, s = x_dev[r], q[r], s[r]
    xr = x_dev.float().cpu()
    rq, rs = oracle.quantize_1x128(xr, fmt)
    assert_quantised(q.cpu().numpy(), s.cpu().numpy(), rq, rs, fmt)


# (1, 128), (256, 4096), (130, 1040) and (16, 272) have 16-byte row strides and K a multiple of 16, so the
# TMA-fed kernel runs them (the last two with ragged tiles); the others take the kernel with plain loads
@pytest.mark.parametrize("M,K", [(1, 128), (7, 300), (64, 1000), (256, 4096), (33, 8200), (130, 1040), (16, 272)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_1x128_bit_exact(M, K, dtype, fmt):
    x = wl.normal_with_outliers((M, K), 7000 + M + K).to(dtype)
    _quant_check(x.to(DEV), fmt)


@pytest.mark.parametrize("fmt", [0, 1])
# K = 528 (a multiple of 16) takes the TMA-fed kernel, whose tensor store must stop at K inside the 544-byte rows
# of q; K = 520 the kernel with plain loads.  The columns of x past K hold huge values, which must not reach a
# group's amax.
@pytest.mark.parametrize("K", [520, 528])
def test_quantize_special_groups_and_strides(fmt, K):
    x = torch.zeros(7, K)
    x[1] = wl.normal_with_outliers((1, K), 7100)[0] * 1e-30       # tiny values
    x[6] = wl.normal_with_outliers((1, K), 7102)[0] * 1e-44       # amax / 448 underflows fp32: scale 1
    x[2, :128] = 448.0 * 2.0 ** 5                                   # amax exactly 448 * 2^5, constant group
    x[2, 128:256] = torch.linspace(-1.0, 1.0, 128)                  # a tie-rich ramp
    x[3] = -0.0
    x[4] = wl.normal_with_outliers((1, K), 7101)[0] * 1e20         # huge values
    x[5, 7] = 1.0                                                   # one non-zero element per group
    base = torch.full((7, 640), 1e30)
    base[:, :K] = x
    xv = base.to(DEV)[:, :K]                                        # row stride 640 > K
    q = torch.full((7, 544), 0x55, dtype=torch.uint8, device=DEV)[:, :K]
    s = torch.zeros((7, 8), dtype=torch.float32 if fmt == 0 else torch.uint8, device=DEV)[:, :5]
    _quant_check(xv, fmt, q=q, scale=s)
    if fmt == 0:
        assert torch.all(s[6] == 1.0)
    full = torch.as_strided(q, (7, 544), (544, 1))
    assert torch.all(full[:, K:] == 0x55), "wrote past K"


def test_quantize_full_size_activations_sampled_rows():
    M, K = 16640, 8192
    x = wl.normal_with_outliers((M, K), 7200).to(torch.bfloat16).to(DEV)
    rows = rows_sample(M, extra=4)
    _quant_check(x, 0, rows=rows)


def test_quantize_then_blockwise_gemm_matches_the_oracle():
    M, N, K = 300, 384, 1024
    x = wl.normal_with_outliers((M, K), 7300)
    w = wl.normal_with_outliers((K, N), 7301)
    Bq, sb = wl.quantize_blocks_128x128(w)
    q, sa = bs.quantize_fp8_1x128(x.to(DEV), "f32")
    out = bs.bs_gemm_fp8_blockwise(q, Bq.t().contiguous().to(DEV).t(), sa, sb.to(DEV))
    rq, rsa = oracle.quantize_1x128(x, 0)
    y, S = oracle.fp8_blockwise(rq, Bq.t().contiguous(), rsa, sb)
    fp8_check(out, y, S, torch.bfloat16, "quantise + blockwise GEMM")


# ---------------------------------------------------------------------------
# transposed-output quantiser (128x1 and 128x128 groups) and the backward GEMMs
# ---------------------------------------------------------------------------
def _quant_t_check(x_dev, group, fmt, **kw):
    qt, s = bs.quantize_fp8_t(x_dev, group, "f32" if fmt == 0 else "e8m0", **kw)
    rq, rs = oracle.quantize_t(x_dev.float().cpu(), 0 if group == "128x1" else 1, fmt)
    assert_quantised(qt.cpu().numpy(), s.cpu().numpy(), rq, rs, fmt)
    return qt, s


# (128, 128), (4096, 640), (1040, 264), (272, 8) and (16, 1000) have 16-byte row strides in x and q_t, so the
# TMA-fed kernel runs them (the last three with ragged tiles); the others take the kernel with plain loads
@pytest.mark.parametrize("R,C", [(1, 1), (128, 128), (300, 5), (5, 300), (130, 260), (1000, 384), (4096, 640),
                                 (1040, 264), (272, 8), (16, 1000)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("group", ["128x1", "128x128"])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_t_bit_exact(R, C, dtype, group, fmt):
    x = wl.normal_with_outliers((R, C), 7400 + R + C).to(dtype)
    _quant_t_check(x.to(DEV), group, fmt)


@pytest.mark.parametrize("group", ["128x1", "128x128"])
@pytest.mark.parametrize("fmt", [0, 1])
# (144, 272): 16-byte rows and R a multiple of 16, the TMA-fed kernel (its tensor store must stop at R inside the
# 288-byte rows); (141, 260) and (144, 260) take the kernel with plain loads and stores
@pytest.mark.parametrize("x_stride,R", [(141, 260), (144, 260), (144, 272)])
def test_quantize_t_special_blocks_strides_and_canaries(group, fmt, x_stride, R):
    C = 136
    x = wl.normal_with_outliers((R, C), 7500)
    x[:128, :128] = 0.0                                  # an all-zero block / columns
    x[128:256, 0] = 448.0 * 2.0 ** 5                     # amax exactly 448 * 2^5
    x[128:256, 1] = torch.linspace(-1.0, 1.0, 128)      # a tie-rich ramp
    x[256:, 5] = 1e-30                                   # tiny values
    x[3, 130] = 3e20                                     # one huge value
    x[:128, 133] = 3e-44 * torch.linspace(-1.0, 1.0, 128)  # a 128x1 group whose amax / 448 underflows
    base = torch.zeros(R, x_stride)                      # row stride 141: no 16-byte loads
    base[:, :C] = x
    xv = base.to(DEV)[:, :C]
    q = torch.full((C, 288), 0x55, dtype=torch.uint8, device=DEV)[:, :R]  # rows of 288 bytes, R used
    sshape = (C, 3) if group == "128x1" else (3, 2)
    s = torch.zeros((sshape[0], sshape[1] + 3), dtype=torch.float32 if fmt == 0 else torch.uint8,
                    device=DEV)[:, :sshape[1]]
    _quant_t_check(xv, group, fmt, q_t=q, scale=s)
    full = torch.as_strided(q, (C, 288), (288, 1))
    assert torch.all(full[:, R:] == 0x55), "wrote past R"


@pytest.mark.parametrize("group", ["128x1", "128x128"])
def test_quantize_t_reads_no_column_past_c(group):
    """x rows of 16-byte strides whose C columns end inside a 16-byte piece: the columns between C and the
    stride hold huge values, which must not reach a 128x128 block's amax."""
    R, C, ld = 256, 132, 136
    base = torch.full((R, ld), 1e30)
    base[:, :C] = wl.normal_with_outliers((R, C), 7550)
    xv = base.to(torch.bfloat16).to(DEV)[:, :C]
    _quant_t_check(xv, group, 0)


def test_quantise_gemm_chains_reuse_buffers_back_to_back():
    """Quantisers and GEMMs launched back to back on one stream with programmatic dependent launch, reusing the
    same code, scale and output buffers: each quantiser must wait for the GEMM before it to finish reading the
    codes it overwrites, and each GEMM and the quantiser that reads a GEMM's output must see the whole of the
    kernel before it.  Every result equals the same computation run one call at a time."""
    M, N, K = 1024, 1024, 2048
    xs = [wl.normal_with_outliers((M, K), 7700 + i).to(torch.bfloat16).to(DEV) for i in range(4)]
    ws = [wl.normal_with_outliers((N, K), 7710 + i).to(torch.bfloat16).to(DEV) for i in range(4)]
    a, sa = torch.empty(M, K, dtype=torch.uint8, device=DEV), torch.empty(M, K // 128, device=DEV)
    b, sb = bs.bs_quantize_fp8_128x128(ws[0], "f32")
    ys = [torch.empty(M, N, dtype=torch.bfloat16, device=DEV) for _ in range(4)]
    qy = [torch.empty(M, N, dtype=torch.uint8, device=DEV) for _ in range(4)]
    sy = [torch.empty(M, N // 128, device=DEV) for _ in range(4)]
    torch.cuda.synchronize()
    for i in range(4):  # no synchronisation inside the chain
        bs.quantize_fp8_1x128(xs[i], "f32", q=a, scale=sa)
        bs.bs_quantize_fp8_128x128(ws[i], "f32", q=b, scale=sb)
        bs.bs_gemm_fp8_blockwise(a, b.t(), sa, sb, out=ys[i])
        bs.quantize_fp8_1x128(ys[i], "f32", q=qy[i], scale=sy[i])
    torch.cuda.synchronize()
    assert bs.device_error() == 0
    for i in range(4):
        ra, rsa = bs.quantize_fp8_1x128(xs[i], "f32")
        rb, rsb = bs.bs_quantize_fp8_128x128(ws[i], "f32")
        torch.cuda.synchronize()
        ry = bs.bs_gemm_fp8_blockwise(ra, rb.t(), rsa, rsb)
        torch.cuda.synchronize()
        rq, rs = bs.quantize_fp8_1x128(ry, "f32")
        torch.cuda.synchronize()
        assert torch.equal(ys[i], ry), f"GEMM {i}"
        assert torch.equal(qy[i], rq) and torch.equal(sy[i], rs), f"quantised output {i}"


def test_quantise_gemm_chain_replays_in_a_cuda_graph():
    """The forward and backward operand quantisers and the blockwise GEMM captured once in a CUDA graph (the
    kernels launch on the capturing stream, with programmatic dependent launch between them) and replayed on
    new inputs copied into the captured buffers: every replay equals the same calls run eagerly."""
    M, N, K = 640, 768, 1024
    x = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    w = torch.empty(N, K, dtype=torch.bfloat16, device=DEV)
    a, sa = torch.empty(M, K, dtype=torch.uint8, device=DEV), torch.empty(M, K // 128, device=DEV)
    b, sb = torch.empty(N, K, dtype=torch.uint8, device=DEV), torch.empty(K // 128, N // 128, device=DEV)
    xt, sxt = torch.empty(K, M, dtype=torch.uint8, device=DEV), torch.empty(M // 128, K // 128, device=DEV)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)

    def step():
        bs.quantize_fp8_1x128(x, "f32", q=a, scale=sa)
        bs.bs_quantize_fp8_128x128(w, "f32", q=b, scale=sb)
        bs.bs_gemm_fp8_blockwise(a, b.t(), sa, sb, out=y)
        bs.quantize_fp8_t(x, "128x128", "f32", q_t=xt, scale=sxt)

    x.copy_(wl.normal_with_outliers((M, K), 7740).to(torch.bfloat16))
    w.copy_(wl.normal_with_outliers((N, K), 7741).to(torch.bfloat16))
    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(side):
        step()  # warm-up on the capturing stream (one-time launch set-up outside the capture)
    torch.cuda.current_stream(DEV).wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    for i in range(3):
        x.copy_(wl.normal_with_outliers((M, K), 7750 + i).to(torch.bfloat16))
        w.copy_(wl.normal_with_outliers((N, K), 7760 + i).to(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (a, sa, b, sb, y, xt, sxt)]
        step()
        torch.cuda.synchronize()
        for name, g, e in zip(("a", "scale_a", "b", "scale_b", "y", "x_t", "scale_x_t"), got, (a, sa, b, sb, y, xt, sxt)):
            assert torch.equal(g, e), f"replay {i}: {name}"
    del graph
    assert bs.device_error() == 0


def test_transposed_quantiser_chain_reuses_buffers_back_to_back():
    """The backward operands of several steps quantised into the same buffers, each followed by its weight-
    gradient GEMM, with no synchronisation in between; equal to the same steps run one call at a time."""
    M, N, K = 1024, 512, 768  # tokens, output features, input features
    dys = [wl.normal_with_outliers((M, N), 7720 + i).to(torch.bfloat16).to(DEV) for i in range(3)]
    xs = [wl.normal_with_outliers((M, K), 7730 + i).to(torch.bfloat16).to(DEV) for i in range(3)]
    a, sa = bs.quantize_fp8_t(dys[0], "128x1", "f32")
    b, sb = bs.quantize_fp8_t(xs[0], "128x128", "f32")
    outs = [torch.empty(N, K, dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    torch.cuda.synchronize()
    for i in range(3):
        bs.quantize_fp8_t(dys[i], "128x1", "f32", q_t=a, scale=sa)
        bs.quantize_fp8_t(xs[i], "128x128", "f32", q_t=b, scale=sb)
        bs.bs_gemm_fp8_blockwise(a, b.t(), sa, sb, out=outs[i])
    torch.cuda.synchronize()
    assert bs.device_error() == 0
    for i in range(3):
        ra, rsa = bs.quantize_fp8_t(dys[i], "128x1", "f32")
        rb, rsb = bs.quantize_fp8_t(xs[i], "128x128", "f32")
        torch.cuda.synchronize()
        ref = bs.bs_gemm_fp8_blockwise(ra, rb.t(), rsa, rsb)
        torch.cuda.synchronize()
        assert torch.equal(outs[i], ref), f"weight gradient {i}"


def test_quantize_t_full_size_output_gradient():
    dy = wl.normal_with_outliers((16640, 5120), 7600).to(torch.bfloat16).to(DEV)
    _quant_t_check(dy, "128x1", 0)


def test_backward_gemms_through_the_transposed_quantiser():
    M, N, K = 384, 256, 640  # tokens, output features, input features of y = x W^T
    x = wl.normal_with_outliers((M, K), 7700)
    dy = wl.normal_with_outliers((M, N), 7701)
    W = wl.normal_with_outliers((N, K), 7702)
    # weight gradient dW [N, K] = dy^T x: contraction over the M tokens
    a, sa = bs.quantize_fp8_t(dy.to(DEV), "128x1")
    b, sb = bs.quantize_fp8_t(x.to(DEV), "128x128")
    dW = bs.bs_gemm_fp8_blockwise(a, b.t(), sa, sb)
    ra, rsa = oracle.quantize_t(dy, 0, 0)
    rb, rsb = oracle.quantize_t(x, 1, 0)
    assert np.array_equal(a.cpu().numpy(), ra) and np.array_equal(b.cpu().numpy(), rb)
    y, S = oracle.fp8_blockwise(ra, rb, rsa, rsb)
    fp8_check(dW, y, S, torch.bfloat16, "weight gradient")
    # input gradient dx [M, K] = dy W: contraction over the N outputs
    a2, sa2 = bs.quantize_fp8_1x128(dy.to(DEV), "f32")
    b2, sb2 = bs.quantize_fp8_t(W.to(DEV), "128x128")
    dx = bs.bs_gemm_fp8_blockwise(a2, b2.t(), sa2, sb2)
    ra2, rsa2 = oracle.quantize_1x128(dy, 0)
    rb2, rsb2 = oracle.quantize_t(W, 1, 0)
    y2, S2 = oracle.fp8_blockwise(ra2, rb2, rsa2, rsb2)
    fp8_check(dx, y2, S2, torch.bfloat16, "input gradient")


# ---------------------------------------------------------------------------
# forward-orientation 128x128 weight quantiser (B_t [N, K] and scale_b) -- bit-exact
# ---------------------------------------------------------------------------
def _near_midpoint_blocks(R, C, bh, bw, seed):
    """fp32 [R, C] whose bh x bw groups have quotients x / (amax / 448) within 3 fp32 ulps of e4m3
    rounding midpoints (normal and subnormal e4m3 range), with group amax from 2^-115 to 2^120 (so
    scales on both sides of 2^-90, the bound of the kernels' fp32 division path).  Element (0, 0) of
    each group holds its amax.  A quotient with too few correct bits rounds to a different code here."""
    rng = np.random.default_rng(seed)
    gr, gc = -(-R // bh), -(-C // bw)
    e = rng.integers(-115, 121, size=(gr, gc))
    amax = np.ldexp(1.0 + rng.random((gr, gc)), e).astype(np.float32)
    s = (amax / np.float32(448.0)).astype(np.float32).astype(np.float64)
    s_full = np.repeat(np.repeat(s, bh, 0), bw, 1)[:R, :C]
    a_full = np.repeat(np.repeat(amax, bh, 0), bw, 1)[:R, :C]
    k = rng.integers(0, 8, (R, C))
    ex = rng.integers(-9, 9, (R, C))
    mids = (8 + k + 0.5) / 8.0 * np.exp2(ex)                       # midpoints between e4m3 normals
    subn = (2 * rng.integers(0, 8, (R, C)) + 1) * 2.0 ** -10          # midpoints in the subnormal range
    mids = np.where(ex < -6, subn, mids)
    v = (mids * s_full).astype(np.float32)
    v = (v.view(np.int32) + rng.integers(-3, 4, (R, C)).astype(np.int32)).view(np.float32)
    v = np.minimum(np.abs(v), a_full) * rng.choice(np.array([-1.0, 1.0], np.float32), (R, C))
    v[::bh, ::bw] = amax[: -(-R // bh), : -(-C // bw)]
    return torch.from_numpy(v.astype(np.float32))


def test_quantizers_quotients_next_to_rounding_midpoints():
    """All three quantisers, fp32 scales, on groups built so that each code sits on a knife edge:
    bit-exact against the oracle (the kernels divide with an fp32 correction step, not in fp64)."""
    x = _near_midpoint_blocks(256, 1024, 1, 128, 9900)
    _quant_check(x.to(DEV), 0)
    xt = _near_midpoint_blocks(1024, 256, 128, 1, 9901)
    _quant_t_check(xt.to(DEV), "128x1", 0)
    xb = _near_midpoint_blocks(512, 640, 128, 128, 9902)
    _quant_t_check(xb.to(DEV), "128x128", 0)
    _quant_b_check(xb.to(DEV), 0)


def _quant_b_check(x_dev, fmt, **kw):
    q, s = bs.bs_quantize_fp8_128x128(x_dev, "f32" if fmt == 0 else "e8m0", **kw)
    rq, rs = oracle.quantize_128x128(x_dev.float().cpu(), fmt)
    assert_quantised(q.cpu().numpy(), s.t().cpu().numpy(), rq, rs, fmt)
    return q, s


# (128, 128), (1000, 384), (1040, 272) and (16, 1008) have 16-byte row strides and C a multiple of 16, so the
# TMA-fed kernel runs them (the last three with ragged tiles); the others take the kernel with plain loads
@pytest.mark.parametrize("R,C", [(1, 1), (128, 128), (300, 5), (5, 300), (130, 260), (1000, 384), (384, 4104),
                                 (1040, 272), (16, 1008)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_128x128_bit_exact(R, C, dtype, fmt):
    x = wl.normal_with_outliers((R, C), 9400 + R + C).to(dtype)
    _quant_b_check(x.to(DEV), fmt)


@pytest.mark.parametrize("fmt", [0, 1])
# (320, 304): 16-byte rows and C a multiple of 16, the TMA-fed kernel (its tensor store must stop at C inside the
# 320-byte rows of q); (303, 300) takes the kernel with plain loads and stores.  The columns of x past C hold
# huge values, which must not reach a block's amax.
@pytest.mark.parametrize("x_stride,C", [(303, 300), (320, 304)])
def test_quantize_128x128_special_blocks_strides_and_canaries(fmt, x_stride, C):
    R = 260
    x = wl.normal_with_outliers((R, C), 9500)
    x[:128, :128] = 0.0                                   # an all-zero block
    x[:128, 128:256] = 3e-44 * torch.linspace(-1.0, 1.0, 128)[None, :]  # amax / 448 underflows: scale 1
    x[128:256, :128] = torch.linspace(-1.0, 1.0, 128)[:, None] * 448.0 * 2.0 ** 5  # amax exactly 448 * 2^5
    x[256:, 7] = 1e-30                                    # tiny values
    x[200, 290] = 3e20                                    # one huge value
    base = torch.full((R, x_stride), 1e30)                # row stride 303: no 16-byte loads
    base[:, :C] = x
    xv = base.to(DEV)[:, :C]
    q = torch.full((R, 320), 0x55, dtype=torch.uint8, device=DEV)[:, :C]
    sfull = torch.full((3, 5), 9, dtype=torch.float32 if fmt == 0 else torch.uint8, device=DEV)
    s = sfull[:, :3]                                     # [CB, RB] with a padded row stride
    _quant_b_check(xv, fmt, q=q, scale=s)
    assert torch.all(torch.as_strided(q, (R, 320), (320, 1))[:, C:] == 0x55), "wrote past C"
    assert torch.all(sfull[:, 3:] == 9), "wrote past the scale rows"
    if fmt == 0:
        assert float(s[1, 0]) == 1.0 and float(s[0, 0]) == 1.0


def test_quantize_128x128_full_size_weight():
    W = wl.normal_with_outliers((5120, 8192), 9600).to(torch.bfloat16).to(DEV)
    _quant_b_check(W, 0)


def test_forward_gemm_through_the_weight_quantiser():
    """y = x W^T with x in 1x128 groups and W in 128x128 blocks, both quantised on the GPU and fed to the
    blockwise GEMM without a copy (B = q.t(), scale_b as returned)."""
    M, N, K = 300, 384, 1024
    x = wl.normal_with_outliers((M, K), 9700)
    W = wl.normal_with_outliers((N, K), 9701)
    a, sa = bs.quantize_fp8_1x128(x.to(DEV), "f32")
    b, sb = bs.bs_quantize_fp8_128x128(W.to(DEV), "f32")
    y_gpu = bs.bs_gemm_fp8_blockwise(a, b.t(), sa, sb)
    ra, rsa = oracle.quantize_1x128(x, 0)
    rb, rsb = oracle.quantize_128x128(W, 0)
    assert np.array_equal(b.cpu().numpy(), rb) and np.array_equal(sb.cpu().numpy(), rsb.T)
    y, S = oracle.fp8_blockwise(ra, rb, rsa, rsb.T)
    fp8_check(y_gpu, y, S, torch.bfloat16, "forward GEMM of the quantised weight")


# ---------------------------------------------------------------------------
# small-M weight stream (M <= 8): warp-level e4m3 MMA, 16 output columns per CTA
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M", [1, 2, 5, 8])
# grids of at most one CTA per SM (N <= 16 * 148), of up to two (N = 3000) and more (N = 4800): the
# kernel keeps four, two or one K blocks per warp in flight accordingly
@pytest.mark.parametrize("N,K", [(7, 128), (130, 640), (1000, 2048), (300, 4224), (3000, 1152), (4800, 640)])
def test_fp8_small_m_weight_stream(M, N, K, path):
    path(bs.PATH_GEMV)
    d = wl.fp8_blockwise_inputs(M, N, K, seed=1100 + M + N + K)
    y, S = oracle_fp8(d)
    for out_dtype in (torch.bfloat16, torch.float32):
        out = fp8_run(d, out_dtype)
        fp8_check(out, y, S, out_dtype, f"small-M {M}x{N}x{K}")
        assert torch.equal(out, fp8_run(d, out_dtype))


@pytest.mark.parametrize("M,G,N,K", [(1, 8, 1024, 4096), (3, 3, 100, 512), (8, 2, 1030, 4096), (7, 1, 260, 1024),
                                     (4, 8, 1000, 1152)])
@pytest.mark.parametrize("batch_first", [False, True])
def test_bmm_small_m_weight_stream(M, G, N, K, batch_first, path):
    path(bs.PATH_GEMV)
    d = wl.bmm_inputs(M, G, N, K, seed=1200 + M + G + N, batch_first=batch_first)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    for out_dtype in (torch.bfloat16, torch.float32):
        fp8_check(bmm_run(d, out_dtype), y, S, out_dtype, f"bmm small-M {M}x{G}x{N}x{K} bf={batch_first}")


def test_small_m_weight_stream_extreme_scales(path):
    """The edge-of-domain inputs on the small-M kernel: extreme e8m0 bytes (8 rows, two halves) and zero
    or subnormal fp32 block scales (rows 2..9 of the blockwise case, which hold all of its planted rows)."""
    path(bs.PATH_GEMV)
    d = _bmm_edge_inputs(8, 384, 1024, seed=1300)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    for out_dtype in (torch.bfloat16, torch.float32):
        fp8_check(bmm_run(d, out_dtype), y, S, out_dtype, "small-M extreme e8m0")
    d = _blockwise_zero_and_subnormal_scales(256, 384, 1024, seed=910)
    d8 = {"A": d["A"][2:10].contiguous(), "B_t": d["B_t"], "scale_a": d["scale_a"][2:10].contiguous(),
          "scale_b": d["scale_b"]}
    y, S = oracle_fp8(d8)
    fp8_check(fp8_run(d8, torch.bfloat16), y, S, torch.bfloat16, "small-M zero/subnormal scales bf16")


# ---------------------------------------------------------------------------
# stream-K: the last, badly filled round of tiles split over every CTA pair
# ---------------------------------------------------------------------------
def _sk_tiles(op, M, G, N, K):
    return bs.plan_for(op, M, G, N, K, torch.cuda.get_device_properties(0).multi_processor_count)["sk_tiles"]


@pytest.fixture
def stream_k():
    """Enables the split (off by default) for one test; calling the fixture's value turns it off again."""
    prev = bs.set_stream_k(True)

    def off():
        bs.set_stream_k(False)
    yield off
    bs.set_stream_k(prev)


@pytest.mark.parametrize("M,N,K", [(1024, 1024, 4096), (1000, 1800, 2080), (300, 1040, 8192)])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_SINGLE])
def test_int8_stream_k_bit_exact(M, N, K, kernel, path, stream_k):
    path(kernel)
    assert _sk_tiles(bs.OP_INT_SCALED_MM, M, 1, N, K) > 0
    _int8_assert(wl.int8_inputs(M, N, K, seed=950 + M), rows=None)


@pytest.mark.parametrize("M,N,K", [(1024, 1024, 4096), (700, 1800, 2048), (300, 1040, 8192)])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_SINGLE])
def test_fp8_stream_k_matches_the_oracle_and_is_deterministic(M, N, K, kernel, path, stream_k):
    path(kernel)
    assert _sk_tiles(bs.OP_FP8_BLOCKWISE, M, 1, N, K) > 0
    d = wl.fp8_blockwise_inputs(M, N, K, seed=960 + M)
    y, S = oracle_fp8(d)
    for out_dtype in (torch.bfloat16, torch.float32):
        first = fp8_run(d, out_dtype)
        fp8_check(first, y, S, out_dtype, f"fp8 stream-K {M}x{N}x{K} kernel={kernel}")
        assert torch.equal(first, fp8_run(d, out_dtype)), "split tiles are summed in a fixed order"
    stream_k()
    fp8_check(fp8_run(d, torch.float32), y, S, torch.float32, "fp8 without the split")


@pytest.mark.parametrize("M,N,K", [(1024, 1024, 4096), (300, 1040, 8192)])
def test_fp8_rowwise_stream_k(M, N, K, stream_k):
    assert _sk_tiles(bs.OP_FP8_ROWWISE, M, 1, N, K) > 0
    d = wl.fp8_rowwise_inputs(M, N, K, seed=970 + M)
    for out_dtype in (torch.bfloat16, torch.float32):
        y, S = oracle_rowwise(d, True)
        fp8_check(rowwise_run(d, out_dtype, True), y, S, out_dtype, f"fp8 rowwise stream-K {M}x{N}x{K}")
    y, S = oracle_rowwise(d, True)
    s_r = float(np.float32(300.0 / float(np.abs(y).max())))
    e4m3_check(rowwise_run(d, torch.float8_e4m3fn, True, scale_result=s_r), y, S, s_r, "rowwise e4m3 stream-K")


@pytest.mark.parametrize("M,G,N,K", [(1024, 2, 1024, 4096), (300, 3, 520, 4096)])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_PROMOTE])
def test_bmm_stream_k(M, G, N, K, kernel, path, stream_k):
    path(kernel)
    assert _sk_tiles(bs.OP_BMM, M, G, N, K) > 0
    d = wl.bmm_inputs(M, G, N, K, seed=980 + M + G)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    out = bmm_run(d, torch.float32)
    fp8_check(out, y, S, torch.float32, f"bmm stream-K {M}x{G}x{N}x{K} kernel={kernel}")
    assert torch.equal(out, bmm_run(d, torch.float32))


def test_int8_stream_k_equals_the_unsplit_plan(stream_k):
    d = wl.int8_inputs(4096, 4096, 4096, seed=990)
    assert _sk_tiles(bs.OP_INT_SCALED_MM, 4096, 1, 4096, 4096) > 0
    a = int8_run(d, torch.int32)
    stream_k()
    assert torch.equal(a, int8_run(d, torch.int32))


# ---------------------------------------------------------------------------
# edges of the input domain: extreme e8m0 bytes, the int32 limit, zero and
# subnormal fp32 block scales
# ---------------------------------------------------------------------------
# e8m0 bytes planted per batch g (the w bytes are shared by every row, so each
# batch holds one regime of w; the x bytes vary per row and K block):
#   g=0: w in {0,1,2} (2^-127 .. 2^-125, byte 0 an fp32 subnormal); rows of
#        the first half take x in {252,253,254}, so every block scale is
#        2^-2 .. 2^2; the second half x in {126,127,128}: tiny results
#        (2^-129 .. 2^-125 times the partials)
#   g=1: w in {252,253,254}; x in {0,1,2} (first half) or {30,31,32}
#   g=2: w in {126,127,128}; x drawn from {0,1,2,126,127,128,200,210,220}
#        per block, so huge and tiny blocks meet in one sum
#   g=3: w and x in {0,1,2}: every product underflows fp32 (2^-254 .. 2^-250)
#   g=4: w in {107,108,109}, x in {0,1,2}: block scales 2^-147 .. 2^-143,
#        results in the fp32 subnormal range
E8M0_EDGE_W = ((0, 1, 2), (252, 253, 254), (126, 127, 128), (0, 1, 2), (107, 108, 109))
E8M0_EDGE_X = (((252, 253, 254), (126, 127, 128)), ((0, 1, 2), (30, 31, 32)),
               ((0, 1, 2, 126, 127, 128, 200, 210, 220),) * 2, ((0, 1, 2),) * 2, ((0, 1, 2),) * 2)


def _bmm_edge_inputs(M, N, K, seed):
    G = len(E8M0_EDGE_W)
    d = wl.bmm_inputs(M, G, N, K, seed=seed)
    gen = torch.Generator().manual_seed(seed)
    xs, ws = d["x_scale"].clone(), d["w_scale"].clone()
    for g in range(G):
        wc = torch.tensor(E8M0_EDGE_W[g], dtype=torch.uint8)
        ws[g] = wc[torch.randint(0, len(wc), tuple(ws[g].shape), generator=gen)]
        for half, rows in enumerate((slice(0, M // 2), slice(M // 2, M))):
            xc = torch.tensor(E8M0_EDGE_X[g][half], dtype=torch.uint8)
            sub = xs[rows, g]
            xs[rows, g] = xc[torch.randint(0, len(xc), tuple(sub.shape), generator=gen)]
    d["x_scale"], d["w_scale"] = xs, ws
    return d


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_PROMOTE, bs.PATH_WIDE_SINGLE, bs.PATH_SKINNY])
def test_bmm_extreme_e8m0_bytes(kernel, out_dtype, path):
    """Scale bytes 0, 1, 2 and 252, 253, 254 (2^-127 .. 2^127) on every BMM path:
    the tensor core's block-scaled MMA decodes the byte itself, the promotion
    paths decode it in software; both must meet the bound, and products that
    underflow fp32 must give zero, not NaN."""
    M, N, K = 256, 384, 1024
    d = _bmm_edge_inputs(M, N, K, seed=901)
    y, S = oracle.bmm_blockscale(d["x"], d["w"], d["x_scale"], d["w_scale"])
    assert np.all(np.isfinite(y)) and float(np.abs(y).max()) < 2.0 ** 120  # finite in fp32 by construction
    path(kernel)
    fp8_check(bmm_run(d, out_dtype), y, S, out_dtype, f"bmm extreme e8m0 kernel={kernel}")


def test_int8_at_the_int32_limit():
    """K = 131071 (the largest the header allows, lda = 131072) with -128 / 127
    patterns: the accumulator reaches 16384 * 131071 = 2^31 - 16383 and
    -16256 * 131071; int32, fp32 and bf16 outputs bit-exact on both wide
    kernel variants."""
    M, N, K = 128, 128, 131071
    gen = torch.Generator().manual_seed(905)
    vals = torch.tensor([-128, 127, -127, 0, 1, -1], dtype=torch.int8)
    A = torch.zeros(M, K + 1, dtype=torch.int8)
    Bt = torch.zeros(N, K + 1, dtype=torch.int8)
    A[:, :K] = vals[torch.randint(0, len(vals), (M, K), generator=gen)]
    Bt[:, :K] = vals[torch.randint(0, len(vals), (N, K), generator=gen)]
    A[0, :K], A[1, :K], A[2, :K] = -128, 127, -128
    Bt[0, :K], Bt[1, :K] = -128, 127
    A[2, 1:K:2] = 127           # alternating row
    Bt[2, :K] = -128
    Bt[3, :K] = A[3, :K]         # a column equal to a random row: a large positive sum
    d = {"A": A[:, :K], "B_t": Bt[:, :K], "s_a": wl.log_uniform(M, 1e-3, 1e-1, 906),
         "s_b": wl.log_uniform(N, 1e-3, 1e-1, 907)}
    acc, _, _ = oracle.int_scaled_mm(d["A"], d["B_t"], None, None)
    assert acc[0, 0] == 16384 * K and acc[0, 1] == -16256 * K and acc[1, 0] == -16256 * K
    for kernel in (bs.PATH_WIDE, bs.PATH_WIDE_SINGLE):
        bs.set_path_override(kernel)
        try:
            Ad = A.to(DEV)[:, :K]
            Bd = Bt.to(DEV)[:, :K].t()
            assert Ad.stride(0) == K + 1
            for out_dtype in (torch.int32, torch.float32, torch.bfloat16):
                got = bs.int_scaled_mm(Ad, Bd, d["s_a"].to(DEV), d["s_b"].to(DEV), out_dtype=out_dtype)
                acc_r, y_r, bf_r = oracle.int_scaled_mm(d["A"], d["B_t"], d["s_a"], d["s_b"])
                if out_dtype == torch.int32:
                    np.testing.assert_array_equal(got.cpu().numpy(), acc_r)
                elif out_dtype == torch.float32:
                    np.testing.assert_array_equal(f32_bits(got), y_r.view(np.uint32))
                else:
                    np.testing.assert_array_equal(bf16_bits(got), bf_r)
        finally:
            bs.set_path_override(bs.PATH_AUTO)


def _blockwise_zero_and_subnormal_scales(M, N, K, seed):
    """Block scales with zeros and fp32 subnormals planted:
      scale_a row 3 all zero, row 4 zero at kb=2, rows 5..8 subnormal
      (2^-149, 1e-40, 2^-130, 3e-39) in every block, row 9 subnormal in the
      even blocks only; scale_b block (1, 0) zero, (2, 2) subnormal (1e-39);
      column block 1 of scale_b scaled by 2^24 so the subnormal scale_a
      entries meet a partner that lifts their product into the normal range."""
    d = wl.fp8_blockwise_inputs(M, N, K, seed=seed)
    sa, sb = d["scale_a"].clone(), d["scale_b"].clone()
    sa[3] = 0.0
    sa[4, 2] = 0.0
    for r, v in zip(range(5, 9), (2.0 ** -149, 1e-40, 2.0 ** -130, 3e-39)):
        sa[r] = v
    sa[9, 0::2] = 1e-40
    sb[1, 0] = 0.0
    sb[2, 2] = 1e-39
    sb[:, 1] *= 2.0 ** 24
    d["scale_a"], d["scale_b"] = sa, sb
    return d


@pytest.mark.parametrize("kernel", [bs.PATH_WIDE, bs.PATH_WIDE_SINGLE, bs.PATH_SKINNY])
def test_fp8_zero_and_subnormal_block_scales(kernel, path):
    """Zero and subnormal fp32 entries in scale_a and scale_b.  bf16 outputs
    meet the bound everywhere (its ulp floor covers the tiny results).  The
    kernels form each block-scale product scale_a * scale_b in fp32, where a
    subnormal product carries an absolute error of up to 2^-150; that is
    within 1e-3 of the product when it is at least 2^-140.  fp32 outputs are
    checked wherever every block's product is zero or at least 2^-140 (the
    domain the header states for fp32 outputs)."""
    M, N, K = 256, 384, 1024
    d = _blockwise_zero_and_subnormal_scales(M, N, K, seed=910)
    y, S = oracle_fp8(d)
    assert np.all(y[3] == 0.0)
    path(kernel)
    fp8_check(fp8_run(d, torch.bfloat16), y, S, torch.bfloat16, f"zero/subnormal scales bf16 kernel={kernel}")
    g = fp8_run(d, torch.float32)
    sa = d["scale_a"].double().numpy()
    sb = d["scale_b"].double().numpy()
    prod = np.abs(sa[:, :, None] * sb[None, :, :])                 # [M, KB, NB], exact in fp64
    ok_blk = (prod == 0.0) | (prod >= 2.0 ** -140)
    ok = np.repeat(ok_blk.all(axis=1), 128, axis=1)[:, :N]         # [M, N]: every block of (m, n) is safe
    assert ok[:10].sum() > 0 and (~ok).sum() > 0
    gf = to_f64(g)
    assert np.all(np.isfinite(gf))
    rows, cols = np.nonzero(ok)
    sub = torch.tensor(gf[rows, cols])
    fp8_check(sub, y[rows, cols], S[rows, cols], torch.float32, f"zero/subnormal scales f32 kernel={kernel}")

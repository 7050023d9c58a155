"""Host-side tests of the C-ABI library (no GPU needed).

The library must load and export every function include/bsgemm.h declares;
argument validation, planning and the persistent tile order are pure host
logic and are checked here.  No GEMM is computed without a GPU: a well-formed
call on a machine without an sm_100 device must fail with BS_ERR_DEVICE.
"""
from __future__ import annotations

import ctypes
import json
import os
import re
import subprocess

import pytest
import torch

import int8_gemm_b200 as bs
from int8_gemm_b200 import build as bsbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsgemm.h")
GOLDEN = os.path.join(ROOT, "tests", "golden")
HAS_GPU = torch.cuda.is_available()


@pytest.fixture(scope="module", autouse=True)
def built_library():
    bsbuild.build()
    return bs.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(bs_\w+|int_scaled_mm|bmm_a8w8_blockscale)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_the_entry_points():
    f = declared_functions()
    for name in ("bs_gemm_fp8_blockwise", "int_scaled_mm", "bmm_a8w8_blockscale", "bs_gemm_fp8_rowwise",
                 "bs_quantize_fp8_1x128", "bs_quantize_fp8_t", "bs_quantize_fp8_128x128"):
        assert name in f
    assert len(f) >= 14


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", bs.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert getattr(bs.lib(), f) is not None


def test_status_strings():
    names = ["BS_OK", "BS_ERR_NULL", "BS_ERR_SHAPE", "BS_ERR_LAYOUT", "BS_ERR_ALIGNMENT", "BS_ERR_DTYPE",
             "BS_ERR_DEVICE", "BS_ERR_CUDA", "BS_ERR_TIMEOUT"]
    for code, name in enumerate(names):
        assert bs.status_string(code) == name
    assert bs.status_string(99) == "BS_ERR_UNKNOWN"
    assert bs.version() == 200  # 0.2.0


def test_blockwise_scale_shape_rule_from_the_issue():
    g = json.load(open(os.path.join(GOLDEN, "scale_shapes_blockwise.json")))
    h = bs.lib()
    assert h.bs_check_blockwise_scale_shapes(g["M"], g["N"], g["K"], *g["scale_a"], *g["scale_b"]) == bs.BS_OK
    st = h.bs_check_blockwise_scale_shapes(g["M"], g["N"], g["K"], *g["rowwise_scale_a"], *g["rowwise_scale_b"])
    assert st == bs.BS_ERR_SHAPE
    msg = h.bs_last_error_message().decode()
    assert "(16640, 64)" in msg and "(64, 40)" in msg and "(16640, 1)" in msg
    # transposed scale_b is also rejected
    assert h.bs_check_blockwise_scale_shapes(g["M"], g["N"], g["K"], 16640, 64, 40, 64) == bs.BS_ERR_SHAPE


# ---------------------------------------------------------------------------
# planning
# ---------------------------------------------------------------------------
def test_plan_large_fp8_is_persistent_wide_on_cta_pairs():
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 16640, 1, 5120, 8192, 148)
    assert p == {"kernel": 1, "tile_m": 256, "tile_n": 256, "splits": 1, "ctas": 148, "cluster": 2, "launches": 1,
                 "sk_tiles": 0}
    prev = bs.set_path_override(bs.PATH_WIDE_SINGLE)
    try:
        p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 16640, 1, 5120, 8192, 148)
        assert p == {"kernel": 1, "tile_m": 128, "tile_n": 256, "splits": 1, "ctas": 148, "cluster": 1, "launches": 1,
                     "sk_tiles": 0}
    finally:
        bs.set_path_override(prev)
    # fewer tiles than CTA pairs and too few K blocks to spread: one pair per tile
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 300, 1, 512, 1024, 148)
    assert p["ctas"] == 2 * 2 * 2 and p["cluster"] == 2 and p["sk_tiles"] == 0
    # a badly filled last round: whole tiles by default; with stream-K enabled, split over every pair
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 1000, 1, 7168, 2048, 148)
    assert p["ctas"] == 148 and p["sk_tiles"] == 0
    prev = bs.set_stream_k(True)
    try:
        p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 1000, 1, 7168, 2048, 148)
        assert p["ctas"] == 148 and p["sk_tiles"] == 112 - 74
    finally:
        bs.set_stream_k(prev)


@pytest.mark.parametrize("M", [1, 8, 16, 17, 32, 127, 128, 129, 255, 256])
def test_plan_skinny_split_k(M):
    prev = bs.set_path_override(bs.PATH_SKINNY if M <= 8 else bs.PATH_AUTO)  # M <= 8 runs the small-M kernel
    try:
        p = bs.plan_for(bs.OP_FP8_BLOCKWISE, M, 1, 7168, 2048, 148)
    finally:
        bs.set_path_override(prev)
    assert p["kernel"] == 2 and p["launches"] == 1
    assert p["tile_m"] in (16, 32, 64, 128) and p["tile_m"] >= min(M, 128)
    assert p["splits"] in (1, 2, 4, 8) and p["splits"] <= 2048 // 128
    assert p["cluster"] == p["splits"]
    m_tiles = -(-M // p["tile_m"])
    assert p["ctas"] == m_tiles * (7168 // 128) * p["splits"]


@pytest.mark.parametrize("M", [1, 5, 8])
def test_plan_small_m_weight_stream(M):
    # M <= 8: the warp-MMA weight stream, 16 output columns per CTA, one CTA per (16 columns, batch)
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, M, 1, 7168, 2048, 148)
    assert (p["kernel"], p["tile_m"], p["tile_n"], p["ctas"], p["cluster"]) == (4, 8, 16, 448, 1)
    b = bs.plan_for(bs.OP_BMM, M, 8, 1000, 4096, 148)
    assert b["kernel"] == 4 and b["ctas"] == 63 * 8
    assert bs.plan_for(bs.OP_INT_SCALED_MM, M, 1, 7168, 2048, 148)["kernel"] == 1  # no small-M INT8 kernel
    prev = bs.set_path_override(bs.PATH_GEMV)
    try:
        assert bs.plan_for(bs.OP_FP8_BLOCKWISE, M, 1, 256, 128, 148)["kernel"] == 4
    finally:
        bs.set_path_override(prev)


@pytest.mark.parametrize("M", [9, 16, 17])
def test_plan_small_m_beyond_weight_stream(M):
    # 9 to 16 rows: the tcgen05 skinny kernel (faster there), also under the small-M override
    assert bs.plan_for(bs.OP_FP8_BLOCKWISE, M, 1, 7168, 2048, 148)["kernel"] == 2
    assert bs.plan_for(bs.OP_BMM, M, 8, 1000, 4096, 148)["kernel"] == 2
    prev = bs.set_path_override(bs.PATH_GEMV)
    try:
        assert bs.plan_for(bs.OP_FP8_BLOCKWISE, M, 1, 256, 128, 148)["kernel"] != 4  # beyond its M limit
    finally:
        bs.set_path_override(prev)


def test_plan_skinny_long_k_prefers_two_ctas_per_sm():
    # 32 or more K blocks: 32-row activation tiles (two CTAs per SM) when that grid is one wave
    b = bs.plan_for(bs.OP_BMM, 128, 8, 1024, 4096, 148)
    assert (b["tile_m"], b["splits"], b["ctas"]) == (32, 1, 4 * 8 * 8)
    b = bs.plan_for(bs.OP_BMM, 128, 2, 1024, 4096, 148)
    assert (b["tile_m"], b["splits"], b["ctas"]) == (32, 4, 4 * 8 * 2 * 4)
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 70, 1, 640, 4096, 148)
    assert (p["tile_m"], p["splits"], p["cluster"]) == (32, 8, 8)
    # 16 K blocks, or a grid of 32-row tiles beyond one wave: the widest tile that covers M
    assert bs.plan_for(bs.OP_FP8_BLOCKWISE, 127, 1, 7168, 2048, 148)["tile_m"] == 128
    assert bs.plan_for(bs.OP_BMM, 255, 8, 1024, 4096, 148)["tile_m"] == 128


def test_plan_int8_and_edges():
    assert bs.plan_for(bs.OP_INT_SCALED_MM, 4096, 1, 4096, 4096, 148)["kernel"] == 1
    assert bs.plan_for(bs.OP_INT_SCALED_MM, 1, 1, 4096, 4096, 148)["kernel"] == 1  # no skinny INT8 kernel
    assert bs.plan_for(bs.OP_FP8_BLOCKWISE, 0, 1, 5120, 8192, 148)["launches"] == 0
    assert bs.plan_for(bs.OP_FP8_BLOCKWISE, 16, 1, 0, 8192, 148)["launches"] == 0
    p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 16, 1, 512, 0, 148)
    assert p["kernel"] == 3 and p["launches"] == 1
    b = bs.plan_for(bs.OP_BMM, 16384, 8, 1024, 4096, 148)
    assert b["kernel"] == 1 and b["ctas"] == 148 and b["tile_m"] == 256
    b = bs.plan_for(bs.OP_BMM, 1, 8, 1024, 4096, 148)
    assert b["kernel"] == 4 and b["ctas"] == (1024 // 16) * 8
    b = bs.plan_for(bs.OP_BMM, 17, 8, 1024, 4096, 148)
    assert b["kernel"] == 2 and b["ctas"] == 8 * 8 * b["splits"]


def test_path_override_forces_kernels():
    prev = bs.set_path_override(bs.PATH_WIDE)
    try:
        assert bs.plan_for(bs.OP_FP8_BLOCKWISE, 1, 1, 7168, 2048, 148)["kernel"] == 1
        bs.set_path_override(bs.PATH_SKINNY)
        p = bs.plan_for(bs.OP_FP8_BLOCKWISE, 1000, 1, 7168, 2048, 148)
        assert p["kernel"] == 2 and p["tile_m"] == 128
        assert bs.plan_for(bs.OP_INT_SCALED_MM, 1, 1, 4096, 4096, 148)["kernel"] == 1
    finally:
        bs.set_path_override(prev)
    assert bs.plan_for(bs.OP_FP8_BLOCKWISE, 1, 1, 7168, 2048, 148)["kernel"] == 4
    assert bs.plan_for(bs.OP_FP8_BLOCKWISE, 32, 1, 7168, 2048, 148)["kernel"] == 2


# ---------------------------------------------------------------------------
# persistent tile order
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("gm,gn,G,group", [(130, 20, 1, 16), (7, 3, 2, 4), (33, 28, 1, 16), (1, 5, 3, 16), (17, 1, 1, 8)])
def test_tile_order_is_a_bijection_with_grouped_sweep(gm, gn, G, group):
    order = bs.tile_order(gm, gn, G, group)
    assert sorted(order) == sorted((g, m, n) for g in range(G) for m in range(gm) for n in range(gn))
    per = gm * gn
    for t, (g, m, n) in enumerate(order):
        assert g == t // per
        # tiles of one group share a band of `group` tile rows
        local = t % per
        first = (local // (group * gn)) * group
        assert first <= m < first + group


def test_tile_order_columns_sweep_inside_group():
    order = bs.tile_order(32, 4, 1, 16)
    assert order[:17] == [(0, m, 0) for m in range(16)] + [(0, 0, 1)]


# ---------------------------------------------------------------------------
# argument validation (host-only; returns before touching a device)
# ---------------------------------------------------------------------------
P16 = 1 << 20  # a fake, 16-byte aligned "device" address: never dereferenced


def _fp8(**kw):
    a = dict(A=P16, lda=256, B=P16, ldb=256, sa=P16, sa_sm=2, sa_sk=1, sb=P16, sb_sk=2, sb_sn=1, out=P16, ldo=256,
             dt=bs.BS_OUT_BF16, M=64, N=256, K=256)
    a.update(kw)
    v = ctypes.c_void_p
    return bs.lib().bs_gemm_fp8_blockwise(v(a["A"]), a["lda"], v(a["B"]), a["ldb"], v(a["sa"]), a["sa_sm"], a["sa_sk"],
                                          v(a["sb"]), a["sb_sk"], a["sb_sn"], v(a["out"]), a["ldo"], a["dt"],
                                          a["M"], a["N"], a["K"], None)


def test_fp8_validation_codes():
    assert _fp8(K=200) == bs.BS_ERR_SHAPE
    assert _fp8(M=-1) == bs.BS_ERR_SHAPE
    assert _fp8(dt=bs.BS_OUT_I32) == bs.BS_ERR_DTYPE
    assert _fp8(out=0) == bs.BS_ERR_NULL
    assert _fp8(A=0) == bs.BS_ERR_NULL
    assert _fp8(lda=128) == bs.BS_ERR_LAYOUT
    assert _fp8(ldo=100) == bs.BS_ERR_LAYOUT
    assert _fp8(A=P16 + 8) == bs.BS_ERR_ALIGNMENT
    assert _fp8(lda=264) == bs.BS_ERR_ALIGNMENT
    assert _fp8(ldo=260) == bs.BS_ERR_ALIGNMENT  # 260 * 2 bytes is not a multiple of 16
    assert _fp8(M=0) == bs.BS_OK and _fp8(N=0) == bs.BS_OK  # empty problem: no-op, no device needed


def _rw(**kw):
    a = dict(A=P16, lda=256, B=P16, ldb=256, sa=P16, sas=1, sb=P16, sbs=1, bias=None, sres=None, out=P16, ldo=256,
             dt=bs.BS_OUT_BF16, M=64, N=256, K=200)
    a.update(kw)
    v = ctypes.c_void_p
    return bs.lib().bs_gemm_fp8_rowwise(v(a["A"]), a["lda"], v(a["B"]), a["ldb"], v(a["sa"]), a["sas"], v(a["sb"]),
                                        a["sbs"], v(a["bias"]), v(a["sres"]), v(a["out"]), a["ldo"], a["dt"], a["M"],
                                        a["N"], a["K"], None)


def test_fp8_rowwise_validation_codes():
    # the issue's rule: both scales tensorwise (scalars) or both rowwise ((M, 1) and (1, N))
    assert _rw(sas=0, sbs=1) == bs.BS_ERR_SHAPE and _rw(sas=1, sbs=0) == bs.BS_ERR_SHAPE
    assert _rw(sas=2, sbs=2) == bs.BS_ERR_SHAPE
    assert _rw(M=-1) == bs.BS_ERR_SHAPE
    assert _rw(dt=bs.BS_OUT_I32) == bs.BS_ERR_DTYPE
    assert _rw(out=0) == bs.BS_ERR_NULL and _rw(sa=0) == bs.BS_ERR_NULL and _rw(sb=0) == bs.BS_ERR_NULL
    assert _rw(lda=128) == bs.BS_ERR_LAYOUT and _rw(ldo=100) == bs.BS_ERR_LAYOUT
    assert _rw(lda=264) == bs.BS_ERR_ALIGNMENT and _rw(bias=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _rw(M=0) == bs.BS_OK and _rw(N=0) == bs.BS_OK
    # e4m3 output: an optional output scale, rows of N bytes on 16-byte boundaries
    e8 = bs.BS_OUT_E4M3
    assert _rw(sres=P16) == bs.BS_ERR_DTYPE and _rw(dt=bs.BS_OUT_F32, sres=P16) == bs.BS_ERR_DTYPE
    assert _rw(dt=e8, sres=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _rw(dt=e8, N=200, ldo=200) == bs.BS_ERR_ALIGNMENT and _rw(dt=e8, ldo=100) == bs.BS_ERR_LAYOUT
    assert _rw(dt=e8, sres=P16, N=0) == bs.BS_OK
    if not HAS_GPU:  # well-formed calls reach the device check (never launched with fake pointers on a GPU)
        # K need not be a multiple of 128 here (scales are constant along K)
        assert _rw(K=200) == bs.BS_ERR_DEVICE and _rw(sas=0, sbs=0, K=48) == bs.BS_ERR_DEVICE
        assert _rw(dt=e8, sres=P16, N=200, ldo=208) == bs.BS_ERR_DEVICE and _rw(dt=e8, K=0) == bs.BS_ERR_DEVICE


def test_plan_fp8_rowwise_is_the_wide_kernel_for_every_m():
    for M in (1, 16, 300, 16640):
        p = bs.plan_for(bs.OP_FP8_ROWWISE, M, 1, 5120, 8192, 148)
        assert p["kernel"] == 1 and p["tile_n"] == 256 and p["cluster"] == 2
    assert bs.plan_for(bs.OP_FP8_ROWWISE, 16, 1, 512, 0, 148)["kernel"] == 3  # K = 0: bias (or zero) fill


@pytest.mark.parametrize("entry", ["int_scaled_mm", "bs_int_scaled_mm_noalloc"])
def test_int8_and_bmm_validation_codes(entry):
    h, v = bs.lib(), ctypes.c_void_p
    fn = getattr(h, entry)
    call = lambda **k: fn(v(k.get("A", P16)), k.get("lda", 128), v(k.get("B", P16)), k.get("ldb", 128),
                          v(P16), v(P16), v(k.get("out", P16)), k.get("ldo", 64), k.get("dt", bs.BS_OUT_F32),
                          k.get("M", 8), 64, k.get("K", 128), None)
    assert call(K=131072) == bs.BS_ERR_SHAPE
    assert call(dt=7) == bs.BS_ERR_DTYPE
    assert call(dt=bs.BS_OUT_E4M3) == bs.BS_ERR_DTYPE
    assert call(B=0) == bs.BS_ERR_NULL
    assert call(ldb=64) == bs.BS_ERR_LAYOUT
    assert call(lda=136) == bs.BS_ERR_ALIGNMENT
    assert call(M=0) == bs.BS_OK
    if not HAS_GPU:
        assert call() == bs.BS_ERR_DEVICE
    bmm = lambda **k: h.bmm_a8w8_blockscale(v(P16), k.get("x_sm", 1024), 128, v(P16), 128 * 256, 128, v(P16), v(P16),
                                            v(P16), 2048, 256, bs.BS_OUT_BF16, 4, 8, 256, k.get("K", 128), None)
    assert bmm(K=64) == bs.BS_ERR_SHAPE
    assert bmm(x_sm=1000) == bs.BS_ERR_ALIGNMENT


@pytest.mark.skipif(HAS_GPU, reason="checks the no-device path")
def test_well_formed_call_without_gpu_fails_loudly():
    assert _fp8() == bs.BS_ERR_DEVICE
    assert "device" in bs.lib().bs_last_error_message().decode().lower()


def test_binding_rejects_cpu_tensors():
    A = torch.zeros(128, 256, dtype=torch.uint8)
    with pytest.raises(bs.BsgemmError):
        bs.bs_gemm_fp8_blockwise(A, A.t(), torch.ones(128, 2), torch.ones(2, 1))
    with pytest.raises(bs.BsgemmError):
        bs.int_scaled_mm(A.to(torch.int8), A.to(torch.int8).t(), None)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("N", [1, 7, 8, 130, 259, 4099, 7168])
def test_default_output_rows_start_on_16_byte_boundaries(N, dtype):
    """The binding's own output allocation satisfies the 16-byte row-stride rule
    of the C ABI for any N (padding lives in memory, not in the shape)."""
    out = bs._empty_out((5,), N, dtype, "cpu")
    assert out.shape == (5, N) and out.stride(1) == 1
    assert (out.stride(0) * out.element_size()) % 16 == 0 and out.stride(0) - N < 16 // out.element_size()
    out3 = bs._empty_out((3, 4), N, dtype, "cpu")
    assert out3.shape == (3, 4, N)
    assert all((s * out3.element_size()) % 16 == 0 for s in out3.stride()[:2])


def _qz(**kw):
    a = dict(x=P16, dt=0, M=64, K=300, ldx=304, q=P16, ldq=304, s=P16, fmt=0, lds=3)
    a.update(kw)
    v = ctypes.c_void_p
    return bs.lib().bs_quantize_fp8_1x128(v(a["x"]), a["dt"], a["M"], a["K"], a["ldx"], v(a["q"]), a["ldq"],
                                          v(a["s"]), a["fmt"], a["lds"], None)


def test_quantize_validation_codes():
    assert _qz(M=-1) == bs.BS_ERR_SHAPE and _qz(K=-5) == bs.BS_ERR_SHAPE
    assert _qz(M=1 << 31) == bs.BS_ERR_SHAPE
    assert _qz(dt=2) == bs.BS_ERR_DTYPE and _qz(fmt=2) == bs.BS_ERR_DTYPE
    assert _qz(x=0) == bs.BS_ERR_NULL and _qz(q=0) == bs.BS_ERR_NULL and _qz(s=0) == bs.BS_ERR_NULL
    assert _qz(ldx=200) == bs.BS_ERR_LAYOUT and _qz(ldq=299) == bs.BS_ERR_LAYOUT
    assert _qz(lds=2) == bs.BS_ERR_LAYOUT  # ceil(300 / 128) = 3 scales per row
    assert _qz(x=P16 + 1) == bs.BS_ERR_ALIGNMENT and _qz(dt=1, x=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _qz(s=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _qz(M=0) == bs.BS_OK and _qz(K=0) == bs.BS_OK
    if not HAS_GPU:  # well-formed calls reach the device check (never launched with fake pointers on a GPU)
        for kw in ({}, {"x": P16 + 2}, {"q": P16 + 1}, {"ldx": 300}, {"ldq": 301}, {"fmt": 1, "s": P16 + 3}):
            assert _qz(**kw) == bs.BS_ERR_DEVICE, kw


def _qt(**kw):
    a = dict(x=P16, dt=0, R=300, C=200, ldx=208, q=P16, ldq=304, s=P16, fmt=0, grp=0, lds=3)
    a.update(kw)
    v = ctypes.c_void_p
    return bs.lib().bs_quantize_fp8_t(v(a["x"]), a["dt"], a["R"], a["C"], a["ldx"], v(a["q"]), a["ldq"], v(a["s"]),
                                      a["fmt"], a["grp"], a["lds"], None)


def test_quantize_t_validation_codes():
    assert _qt(R=-1) == bs.BS_ERR_SHAPE and _qt(C=-5) == bs.BS_ERR_SHAPE and _qt(R=1 << 31) == bs.BS_ERR_SHAPE
    assert _qt(grp=2) == bs.BS_ERR_SHAPE
    assert _qt(R=1 << 30, C=1 << 30, ldx=1 << 30, ldq=1 << 30, lds=1 << 23) == bs.BS_ERR_SHAPE  # 2^46 tiles
    assert _qt(dt=2) == bs.BS_ERR_DTYPE and _qt(fmt=2) == bs.BS_ERR_DTYPE
    assert _qt(x=0) == bs.BS_ERR_NULL and _qt(q=0) == bs.BS_ERR_NULL and _qt(s=0) == bs.BS_ERR_NULL
    assert _qt(ldx=199) == bs.BS_ERR_LAYOUT and _qt(ldq=299) == bs.BS_ERR_LAYOUT
    assert _qt(lds=2) == bs.BS_ERR_LAYOUT               # 128x1: ceil(300 / 128) = 3 scales per column
    assert _qt(grp=1, lds=1) == bs.BS_ERR_LAYOUT        # 128x128: ceil(200 / 128) = 2 scales per block row
    assert _qt(x=P16 + 1) == bs.BS_ERR_ALIGNMENT and _qt(dt=1, x=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _qt(s=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _qt(R=0) == bs.BS_OK and _qt(C=0) == bs.BS_OK
    if not HAS_GPU:  # well-formed calls reach the device check (never launched with fake pointers on a GPU)
        for kw in ({}, {"grp": 1, "lds": 2}, {"x": P16 + 2}, {"q": P16 + 1}, {"ldx": 201}, {"fmt": 1, "s": P16 + 3}):
            assert _qt(**kw) == bs.BS_ERR_DEVICE, kw


def _qb(**kw):
    a = dict(x=P16, dt=0, R=300, C=200, ldx=208, q=P16, ldq=208, s=P16, fmt=0, srb=1, scb=3)
    a.update(kw)
    v = ctypes.c_void_p
    return bs.lib().bs_quantize_fp8_128x128(v(a["x"]), a["dt"], a["R"], a["C"], a["ldx"], v(a["q"]), a["ldq"],
                                            v(a["s"]), a["fmt"], a["srb"], a["scb"], None)


def test_quantize_128x128_validation_codes():
    assert _qb(R=-1) == bs.BS_ERR_SHAPE and _qb(C=-5) == bs.BS_ERR_SHAPE and _qb(R=1 << 31) == bs.BS_ERR_SHAPE
    assert _qb(R=1 << 30, C=1 << 30, ldx=1 << 30, ldq=1 << 30) == bs.BS_ERR_SHAPE  # 2^46 blocks
    assert _qb(dt=2) == bs.BS_ERR_DTYPE and _qb(fmt=2) == bs.BS_ERR_DTYPE
    assert _qb(x=0) == bs.BS_ERR_NULL and _qb(q=0) == bs.BS_ERR_NULL and _qb(s=0) == bs.BS_ERR_NULL
    assert _qb(ldx=199) == bs.BS_ERR_LAYOUT and _qb(ldq=199) == bs.BS_ERR_LAYOUT
    assert _qb(srb=-1) == bs.BS_ERR_LAYOUT and _qb(scb=0) == bs.BS_ERR_LAYOUT  # 2 column blocks need a stride
    assert _qb(srb=0) == bs.BS_ERR_LAYOUT                                        # 3 row blocks too
    assert _qb(x=P16 + 1) == bs.BS_ERR_ALIGNMENT and _qb(dt=1, x=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _qb(s=P16 + 2) == bs.BS_ERR_ALIGNMENT
    assert _qb(R=0) == bs.BS_OK and _qb(C=0) == bs.BS_OK
    if not HAS_GPU:  # well-formed calls reach the device check (never launched with fake pointers on a GPU)
        for kw in ({}, {"R": 100, "srb": 0}, {"C": 100, "scb": 0}, {"x": P16 + 2}, {"q": P16 + 1}, {"ldx": 201},
                   {"fmt": 1, "s": P16 + 3}):
            assert _qb(**kw) == bs.BS_ERR_DEVICE, kw


@pytest.fixture
def stream_k_on():
    prev = bs.set_stream_k(True)
    yield
    bs.set_stream_k(prev)


@pytest.mark.parametrize("M,N,K,G,op", [(4096, 4096, 4096, 1, 2), (1000, 7168, 2048, 1, 1), (1024, 1024, 4096, 2, 3),
                                        (1024, 1024, 4096, 8, 3), (300, 1024, 2048, 1, 1), (1024, 1024, 4096, 1, 2),
                                        (16640, 5120, 8192, 1, 1)])
@pytest.mark.parametrize("sms", [148, 132])
def test_stream_k_split_covers_every_k_block_once(M, N, K, G, op, sms, stream_k_on):
    """The host copy of the wide kernel's decomposition: every (tile, K block) is computed by exactly one
    unit; each split tile has one head (the unit holding its first block, where that block is the last
    item of the unit); the other pieces are the first split item of their units, so each unit hands over
    at most one partial and finishes at most one split tile."""
    p = bs.plan_for(op, M, G, N, K, sms)
    assert p["kernel"] == 1
    units = p["ctas"] // p["cluster"]
    tiles = -(-M // 256) * -(-N // 256) * G
    KB = -(-K // 128)
    sk_tiles = p["sk_tiles"]
    dp = tiles - sk_tiles
    cover = {}
    heads, givers = {}, {}
    for u in range(units):
        items = bs.work_items(tiles, dp, sk_tiles * KB, KB, units, u)
        split = [it for it in items if it[0] >= dp]
        for n_it, (t, k0, k1) in enumerate(items):
            assert 0 <= k0 < k1 <= KB and 0 <= t < tiles
            for kb in range(k0, k1):
                assert (t, kb) not in cover
                cover[(t, kb)] = u
            if (k0, k1) != (0, KB):
                assert t >= dp
                if k0 == 0:
                    heads.setdefault(t, []).append(u)
                    assert (t, k0, k1) == split[-1], "a head is the last item of its unit"
                else:
                    givers.setdefault(t, []).append(u)
                    assert (t, k0, k1) == split[0], "a hand-over is the first split item of its unit"
        assert sum(1 for it in split if it[1] > 0) <= 1
    assert len(cover) == tiles * KB
    for t in givers:
        assert len(heads[t]) == 1 and all(g > heads[t][0] for g in givers[t])
    if sk_tiles:
        assert set(heads) == set(givers) and len(heads) > 0
        assert p["ctas"] == p["cluster"] * (sms // p["cluster"])


def test_workspace_size_and_registration_checks():
    assert bs.workspace_size(148) >= 148 * 128 * 1024 and bs.workspace_size(0) == 0
    assert bs.workspace_size(148) % 256 == 0
    if not HAS_GPU:  # registration needs a device
        assert bs.lib().bs_set_workspace(ctypes.c_void_p(P16), 1 << 30) == bs.BS_ERR_DEVICE
    assert bs.status_string(bs.BS_ERR_WORKSPACE) == "BS_ERR_WORKSPACE"

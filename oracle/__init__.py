"""CPU oracle for the scaled low-precision GEMMs -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never loads it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module compiles it with gcc on first use and marshals numpy arrays through
ctypes.  See ``oracle.c`` for the definitions and the passages they follow.

Parity status of each function (what pins it in ``tests/test_oracle_pins.py``):
  e4m3_table        -- exhaustive comparison with torch's float8_e4m3fn decode
  round_bf16        -- exact rational rounding (fractions) incl. ties, subnormals, overflow
  fp8_blockwise     -- exact-rational brute force, integer special case, fp64
                       library matmul of dequantised operands, power-of-two
                       linearity, one-hot scale_b orientation
  int_scaled_mm     -- bit-exact against torch._int_mm and torch fp32 ops on CPU
  bmm_blockscale    -- fp64 einsum of bf16-dequantised operands, per-g agreement
                       with fp8_blockwise, one-hot w_scale orientation
  e4m3_encode       -- round trip of every finite code, midpoints (ties to the
                       even code), saturation; torch's float8_e4m3fn cast
  quantize_1x128    -- torch's float8_e4m3fn cast of x / scale (the library
                       routine the recipe reduces to), amax -> +-448, zero
                       groups, e8m0 exponent at and around 448 * 2^e, ragged K,
                       scales that underflow take the zero group's scale
  quantize_t        -- 128x1 groups = the 1x128 quantiser of the transpose;
                       torch's cast of x over its 128x128 block scale; one-hot
                       orientation and block isolation; a block's scale is its
                       largest column scale; the backward GEMMs of the
                       quantised operands approximate the exact gradients
  quantize_128x128  -- torch's cast of x over its block scale; the transposed
                       quantiser's 128x128 codes, transposed back; one-hot block
                       isolation and orientation; the forward GEMM of the
                       quantised weight approximates the exact product
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-shared", "-fPIC", "-Wall"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc); returns the library path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, p = ctypes.c_int64, ctypes.c_void_p
            lib.orc_e4m3_table.argtypes = [p]
            lib.orc_num_threads.restype = ctypes.c_int
            lib.orc_round_bf16.argtypes = [p, p, i64]
            lib.orc_round_f32.argtypes = [p, p, i64]
            lib.orc_fp8_blockwise.argtypes = [p, i64, p, i64, p, i64, i64, p, i64, i64,
                                              i64, i64, i64, p, i64, p, p]
            lib.orc_bmm_blockscale.argtypes = [p, i64, i64, p, i64, i64, p, p,
                                               i64, i64, i64, i64, p, i64, p, p]
            lib.orc_int_scaled_mm.argtypes = [p, i64, p, i64, p, p, i64, i64, i64, p, i64, p, p, p]
            lib.orc_fp8_rowwise.argtypes = [p, i64, p, i64, p, i64, p, i64, p, i64, i64, i64, p, i64, p, p]
            lib.orc_e4m3_encode.argtypes = [p, p, i64]
            lib.orc_quantize_1x128.argtypes = [p, i64, i64, i64, ctypes.c_int, p, i64, p, p]
            lib.orc_quantize_t.argtypes = [p, i64, i64, i64, ctypes.c_int, ctypes.c_int, p, i64, p, p]
            lib.orc_quantize_128x128.argtypes = [p, i64, i64, i64, ctypes.c_int, p, i64, p, p]
            for f in (lib.orc_fp8_blockwise, lib.orc_bmm_blockscale, lib.orc_int_scaled_mm, lib.orc_fp8_rowwise,
                      lib.orc_quantize_1x128, lib.orc_quantize_t, lib.orc_quantize_128x128):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _np(t):
    """Accept numpy arrays or CPU torch tensors."""
    if hasattr(t, "numpy") and not isinstance(t, np.ndarray):
        return t.detach().cpu().numpy()
    return np.asarray(t)


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _estride(a, axis):
    return a.strides[axis] // a.itemsize


def _rows(rows, M):
    if rows is None:
        return None, M
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, len(r)


def num_threads() -> int:
    return _load().orc_num_threads()


def e4m3_table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _load().orc_e4m3_table(_ptr(out))
    return out


def round_bf16(y) -> np.ndarray:
    """fp64 -> bf16 bit patterns (uint16), RNE directly from fp64."""
    y = np.ascontiguousarray(_np(y), dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    _load().orc_round_bf16(_ptr(y), _ptr(out), y.size)
    return out


def round_f32(y) -> np.ndarray:
    y = np.ascontiguousarray(_np(y), dtype=np.float64)
    out = np.empty(y.shape, dtype=np.float32)
    _load().orc_round_f32(_ptr(y), _ptr(out), y.size)
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(_np(bits)).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _row_major_u8(a):
    a = _np(a)
    assert a.dtype in (np.uint8, np.int8) and a.ndim == 2 and a.strides[1] == 1
    return a


def fp8_blockwise(A, B_t, scale_a, scale_b, rows=None):
    """Operation 1.  A uint8 [M,K] e4m3 codes (row stride arbitrary, unit K
    stride); B_t uint8 [N,K] codes of B[K,N]; scale_a fp32 [M,K/128];
    scale_b fp32 [K/128, ceil(N/128)] (any element strides).

    Returns (y, S): fp64 [R, N] exact-order results and the |a*b| magnitude
    sums for the listed rows (all rows when ``rows`` is None)."""
    A, B_t = _row_major_u8(A), _row_major_u8(B_t)
    sa = _np(scale_a).astype(np.float32, copy=False)
    sb = _np(scale_b).astype(np.float32, copy=False)
    M, K = A.shape
    N = B_t.shape[0]
    assert B_t.shape[1] == K and sa.shape == (M, K // 128) and sb.shape == (K // 128, (N + 127) // 128)
    r, R = _rows(rows, M)
    y = np.empty((R, N), dtype=np.float64)
    S = np.empty((R, N), dtype=np.float64)
    rc = _load().orc_fp8_blockwise(
        _ptr(A), _estride(A, 0), _ptr(B_t), _estride(B_t, 0),
        _ptr(sa), _estride(sa, 0), _estride(sa, 1), _ptr(sb), _estride(sb, 0), _estride(sb, 1),
        M, N, K, _ptr(r), R, _ptr(y), _ptr(S))
    if rc != 0:
        raise ValueError(f"oracle fp8_blockwise failed with code {rc}")
    return y, S


def bmm_blockscale(x, w, x_scale, w_scale, rows=None):
    """Operation 3.  x uint8 [M,G,K] (strides (x_sm, x_sg, 1)), w uint8 [G,N,K]
    (unit K stride), x_scale uint8 [M,G,K/128], w_scale uint8 [G,ceil(N/128),K/128].

    Returns (y, S): fp64 [R, G, N]."""
    x, w = _np(x), _np(w)
    xs = np.ascontiguousarray(_np(x_scale), dtype=np.uint8)
    ws = np.ascontiguousarray(_np(w_scale), dtype=np.uint8)
    M, G, K = x.shape
    N = w.shape[1]
    assert x.strides[2] == 1 and w.strides[2] == 1 and w.shape == (G, N, K)
    assert xs.shape == (M, G, K // 128) and ws.shape == (G, (N + 127) // 128, K // 128)
    r, R = _rows(rows, M)
    y = np.empty((R, G, N), dtype=np.float64)
    S = np.empty((R, G, N), dtype=np.float64)
    rc = _load().orc_bmm_blockscale(
        _ptr(x), _estride(x, 0), _estride(x, 1), _ptr(w), _estride(w, 0), _estride(w, 1),
        _ptr(xs), _ptr(ws), M, G, N, K, _ptr(r), R, _ptr(y), _ptr(S))
    if rc != 0:
        raise ValueError(f"oracle bmm_blockscale failed with code {rc}")
    return y, S


def int_scaled_mm(A, B_t, s_a, s_b, rows=None):
    """Operation 2.  A int8 [M,K], B_t int8 [N,K] (codes of B[K,N]), s_a fp32 [M]
    or None, s_b fp32 [N] or None.

    Returns (acc int32 [R,N], y fp32 [R,N], bf16 bits uint16 [R,N])."""
    A, B_t = _row_major_u8(A), _row_major_u8(B_t)
    M, K = A.shape
    N = B_t.shape[0]
    sa = None if s_a is None else np.ascontiguousarray(_np(s_a), dtype=np.float32).reshape(-1)
    sb = None if s_b is None else np.ascontiguousarray(_np(s_b), dtype=np.float32).reshape(-1)
    assert sa is None or sa.size == M
    assert sb is None or sb.size == N
    r, R = _rows(rows, M)
    acc = np.empty((R, N), dtype=np.int32)
    y = np.empty((R, N), dtype=np.float32)
    bf = np.empty((R, N), dtype=np.uint16)
    rc = _load().orc_int_scaled_mm(
        _ptr(A), _estride(A, 0), _ptr(B_t), _estride(B_t, 0), _ptr(sa), _ptr(sb),
        M, N, K, _ptr(r), R, _ptr(acc), _ptr(y), _ptr(bf))
    if rc != 0:
        raise ValueError(f"oracle int_scaled_mm failed with code {rc} (2 = int32 overflow)")
    return acc, y, bf


def fp8_rowwise(A, B_t, scale_a, scale_b, bias=None, rows=None):
    """FP8 GEMM with tensorwise or rowwise scales.  A uint8 [M,K] e4m3 codes, B_t uint8 [N,K] codes of
    B[K,N]; scale_a fp32 scalar (tensorwise) or [M] / [M,1] (rowwise); scale_b fp32 scalar or [N] / [1,N]
    (the same kind as scale_a); bias fp32 [N] or None.

    Returns (y, S): fp64 [R, N] results and |a*b| magnitude sums times |scale_a*scale_b|."""
    A, B_t = _row_major_u8(A), _row_major_u8(B_t)
    M, K = A.shape
    N = B_t.shape[0]
    assert B_t.shape[1] == K
    sa = np.ascontiguousarray(_np(scale_a), dtype=np.float32).reshape(-1)
    sb = np.ascontiguousarray(_np(scale_b), dtype=np.float32).reshape(-1)
    assert (sa.size, sb.size) in ((1, 1), (M, N))
    rowwise = (sa.size, sb.size) == (M, N) and (M, N) != (1, 1)
    bias_a = None if bias is None else np.ascontiguousarray(_np(bias), dtype=np.float32).reshape(-1)
    assert bias_a is None or bias_a.size == N
    r, R = _rows(rows, M)
    y = np.empty((R, N), dtype=np.float64)
    S = np.empty((R, N), dtype=np.float64)
    st = 1 if rowwise else 0
    rc = _load().orc_fp8_rowwise(_ptr(A), _estride(A, 0), _ptr(B_t), _estride(B_t, 0), _ptr(sa), st, _ptr(sb), st,
                                 _ptr(bias_a), M, N, K, _ptr(r), R, _ptr(y), _ptr(S))
    if rc != 0:
        raise ValueError(f"oracle fp8_rowwise failed with code {rc}")
    return y, S


def e4m3_encode(v) -> np.ndarray:
    """fp64 values -> e4m3 codes (uint8): round to nearest, ties to the even
    code, |v| >= 448 saturates to +-448, NaN -> 0x7F."""
    v = np.ascontiguousarray(_np(v), dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().orc_e4m3_encode(_ptr(v), _ptr(out), v.size)
    return out


def quantize_1x128(x, fmt: int = 0):
    """1x128 group quantisation of x [M, K] (fp32 or bf16, any row stride).

    fmt 0: returns (codes uint8 [M, K], scale fp32 [M, ceil(K/128)]), scale = amax / 448;
    fmt 1: returns (codes, e8m0 bytes uint8 [M, ceil(K/128)]).  See orc_quantize_1x128."""
    xt = _np(x.float() if hasattr(x, "float") and not isinstance(x, np.ndarray) else x)
    xt = np.ascontiguousarray(xt, dtype=np.float32)
    assert xt.ndim == 2
    M, K = xt.shape
    KB = -(-K // 128)
    q = np.empty((M, K), dtype=np.uint8)
    sf = np.empty((M, KB), dtype=np.float32) if fmt == 0 else None
    se = np.empty((M, KB), dtype=np.uint8) if fmt == 1 else None
    rc = _load().orc_quantize_1x128(_ptr(xt), M, K, K, fmt, _ptr(q), K, _ptr(sf), _ptr(se))
    if rc != 0:
        raise ValueError(f"orc_quantize_1x128 failed ({rc})")
    return q, (sf if fmt == 0 else se)


def quantize_t(x, group: int = 0, fmt: int = 0):
    """Transposed-output quantisation of x [R, C] (fp32 or bf16) for the backward GEMMs.

    Returns (codes uint8 [C, R], q_t[c, r] the code of x[r, c]; scales).  group 0 (128x1 groups along
    the rows): scales [C, ceil(R/128)]; group 1 (128x128 blocks): scales [ceil(R/128), ceil(C/128)].
    fmt 0: fp32 scales (amax / 448); fmt 1: e8m0 bytes.  See orc_quantize_t."""
    xt = _np(x.float() if hasattr(x, "float") and not isinstance(x, np.ndarray) else x)
    xt = np.ascontiguousarray(xt, dtype=np.float32)
    assert xt.ndim == 2
    R, C = xt.shape
    RB, CB = -(-R // 128), -(-C // 128)
    sshape = (C, RB) if group == 0 else (RB, CB)
    q = np.empty((C, R), dtype=np.uint8)
    sf = np.empty(sshape, dtype=np.float32) if fmt == 0 else None
    se = np.empty(sshape, dtype=np.uint8) if fmt == 1 else None
    rc = _load().orc_quantize_t(_ptr(xt), R, C, C, group, fmt, _ptr(q), R, _ptr(sf), _ptr(se))
    if rc != 0:
        raise ValueError(f"orc_quantize_t failed ({rc})")
    return q, (sf if fmt == 0 else se)


def quantize_128x128(x, fmt: int = 0):
    """128x128 block quantisation of x [R, C] (fp32 or bf16) keeping its orientation (a weight W [N, K]
    becomes the B_t codes of the forward GEMM).

    Returns (codes uint8 [R, C], q[r, c] the code of x[r, c]; scales [ceil(R/128), ceil(C/128)], fp32 for
    fmt 0 or e8m0 bytes for fmt 1).  The transpose of the scales is scale_b [K/128, N/128] for x = W [N, K].
    See orc_quantize_128x128."""
    xt = _np(x.float() if hasattr(x, "float") and not isinstance(x, np.ndarray) else x)
    xt = np.ascontiguousarray(xt, dtype=np.float32)
    assert xt.ndim == 2
    R, C = xt.shape
    RB, CB = -(-R // 128), -(-C // 128)
    q = np.empty((R, C), dtype=np.uint8)
    sf = np.empty((RB, CB), dtype=np.float32) if fmt == 0 else None
    se = np.empty((RB, CB), dtype=np.uint8) if fmt == 1 else None
    rc = _load().orc_quantize_128x128(_ptr(xt), R, C, C, fmt, _ptr(q), C, _ptr(sf), _ptr(se))
    if rc != 0:
        raise ValueError(f"orc_quantize_128x128 failed ({rc})")
    return q, (sf if fmt == 0 else se)

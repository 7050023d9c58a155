"""bsgemm: scaled low-precision GEMMs with fused dequantisation for NVIDIA B200.

Thin Python binding over ``libbsgemm.so`` (C ABI, ``include/bsgemm.h``).  The
functions below only check and marshal arguments -- pointers, strides, the
current CUDA stream -- and allocate ``out`` when it is not given; every
arithmetic step runs in the library's sm_100a kernels.  There is no CPU
fallback: if the library is missing or the device is not an sm_100 GPU the
calls raise.

    bs_gemm_fp8_blockwise(A, B, scale_a, scale_b, out_dtype=torch.bfloat16)
    int_scaled_mm(A, B, s_a, s_b=None, out_dtype=torch.float32)
    bmm_a8w8_blockscale(x, w, x_scale, w_scale, out_dtype=torch.bfloat16)
    bs_gemm_fp8_rowwise(A, B, scale_a, scale_b, bias=None, out_dtype=torch.bfloat16, scale_result=None)
    bs_quantize_fp8_1x128(x, scale_format="f32")            -> (q, scale)
    bs_quantize_fp8_t(x, group="128x1", scale_format="f32")  -> (q_t, scale)
    bs_quantize_fp8_128x128(w, scale_format="f32")           -> (q, scale_b)

The quantisers are also available as ``quantize_fp8_1x128``, ``quantize_fp8_t`` and ``quantize_fp8_128x128``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsgemm.so")

BS_OK, BS_ERR_NULL, BS_ERR_SHAPE, BS_ERR_LAYOUT, BS_ERR_ALIGNMENT = 0, 1, 2, 3, 4
BS_ERR_DTYPE, BS_ERR_DEVICE, BS_ERR_CUDA, BS_ERR_TIMEOUT, BS_ERR_WORKSPACE = 5, 6, 7, 8, 9
BS_OUT_BF16, BS_OUT_F32, BS_OUT_I32, BS_OUT_E4M3 = 0, 1, 2, 3

PATH_AUTO, PATH_WIDE, PATH_SKINNY, PATH_WIDE_SINGLE, PATH_WIDE_PROMOTE, PATH_GEMV = 0, 1, 2, 3, 4, 5

_OUT_CODE = {torch.bfloat16: BS_OUT_BF16, torch.float32: BS_OUT_F32, torch.int32: BS_OUT_I32,
             torch.float8_e4m3fn: BS_OUT_E4M3}


class BsgemmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class Plan(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("tile_m", ctypes.c_int32), ("tile_n", ctypes.c_int32),
                ("splits", ctypes.c_int32), ("ctas", ctypes.c_int32), ("cluster", ctypes.c_int32),
                ("launches", ctypes.c_int32), ("sk_tiles", ctypes.c_int32)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


_lock = threading.Lock()
_handle = None


def lib() -> ctypes.CDLL:
    """Load libbsgemm.so (raises if it has not been built)."""
    global _handle
    with _lock:
        if _handle is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m int8_gemm_b200.build`")
            h = ctypes.CDLL(LIB_PATH)
            i64, p, i32, u32p = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)
            h.bs_gemm_fp8_blockwise.argtypes = [p, i64, p, i64, p, i64, i64, p, i64, i64, p, i64, ctypes.c_int,
                                                i64, i64, i64, p]
            h.int_scaled_mm.argtypes = [p, i64, p, i64, p, p, p, i64, ctypes.c_int, i64, i64, i64, p]
            h.bs_int_scaled_mm_noalloc.argtypes = h.int_scaled_mm.argtypes
            h.bs_gemm_fp8_rowwise.argtypes = [p, i64, p, i64, p, i64, p, i64, p, p, p, i64, ctypes.c_int,
                                              i64, i64, i64, p]
            h.bmm_a8w8_blockscale.argtypes = [p, i64, i64, p, i64, i64, p, p, p, i64, i64, ctypes.c_int,
                                              i64, i64, i64, i64, p]
            h.bs_quantize_fp8_1x128.argtypes = [p, ctypes.c_int, i64, i64, i64, p, i64, p, ctypes.c_int, i64, p]
            h.bs_quantize_fp8_t.argtypes = [p, ctypes.c_int, i64, i64, i64, p, i64, p, ctypes.c_int, ctypes.c_int,
                                            i64, p]
            h.bs_quantize_fp8_128x128.argtypes = [p, ctypes.c_int, i64, i64, i64, p, i64, p, ctypes.c_int, i64, i64,
                                                  p]
            for f in (h.bs_gemm_fp8_blockwise, h.int_scaled_mm, h.bs_int_scaled_mm_noalloc, h.bmm_a8w8_blockscale,
                      h.bs_gemm_fp8_rowwise, h.bs_quantize_fp8_1x128, h.bs_quantize_fp8_t,
                      h.bs_quantize_fp8_128x128):
                f.restype = ctypes.c_int
            h.bs_status_string.argtypes = [ctypes.c_int]
            h.bs_status_string.restype = ctypes.c_char_p
            h.bs_last_error_message.argtypes = []
            h.bs_last_error_message.restype = ctypes.c_char_p
            h.bs_check_blockwise_scale_shapes.argtypes = [i64] * 7
            h.bs_check_blockwise_scale_shapes.restype = ctypes.c_int
            h.bs_plan_for.argtypes = [i32, i64, i64, i64, i64, i32, ctypes.POINTER(Plan)]
            h.bs_plan_for.restype = ctypes.c_int
            h.bs_set_path_override.argtypes = [i32]
            h.bs_set_path_override.restype = i32
            h.bs_tile_order.argtypes = [i32, i32, i32, i32, ctypes.POINTER(ctypes.c_int32), i64]
            h.bs_tile_order.restype = ctypes.c_int
            h.bs_get_device_error.argtypes = [p, u32p]
            h.bs_get_device_error.restype = ctypes.c_int
            h.bs_version.restype = i32
            h.bs_workspace_size.argtypes = [i32]
            h.bs_workspace_size.restype = ctypes.c_size_t
            h.bs_set_workspace.argtypes = [p, ctypes.c_size_t]
            h.bs_set_workspace.restype = ctypes.c_int
            h.bs_set_split_override.argtypes = [i32]
            h.bs_set_split_override.restype = i32
            h.bs_set_stream_k.argtypes = [i32]
            h.bs_set_stream_k.restype = i32
            h.bs_work_items.argtypes = [i32, i32, i64, i32, i32, i32, ctypes.POINTER(ctypes.c_int32), i32]
            h.bs_work_items.restype = i32
            _handle = h
    return _handle


def _check(status: int):
    if status != BS_OK:
        h = lib()
        name = h.bs_status_string(status).decode()
        msg = h.bs_last_error_message().decode()
        raise BsgemmError(status, f"{name}: {msg}")


def status_string(status: int) -> str:
    return lib().bs_status_string(status).decode()


_workspaces = {}  # device index -> the zero-filled stream-K workspace registered with the library
_stream_k_on = False  # mirrors bs_set_stream_k: a workspace is registered only while the split is enabled


def _ensure_workspace(device) -> None:
    """Registers a stream-K workspace for `device` on its first GEMM call (bs_set_workspace): allocated
    from torch's caching allocator, zero-filled, and waited for once so that calls on any stream see it
    zeroed.  Inside a CUDA-graph capture nothing is registered (the calls run whole tiles) until a later
    call outside a capture."""
    idx = torch.device(device).index
    idx = torch.cuda.current_device() if idx is None else idx
    if not _stream_k_on or idx in _workspaces:
        return
    with torch.cuda.device(idx):
        if torch.cuda.is_current_stream_capturing():
            return
        n = lib().bs_workspace_size(torch.cuda.get_device_properties(idx).multi_processor_count)
        ws = torch.zeros(n + 256, dtype=torch.uint8, device=f"cuda:{idx}")
        torch.cuda.current_stream().synchronize()
        off = (-ws.data_ptr()) % 256
        _check(lib().bs_set_workspace(ctypes.c_void_p(ws.data_ptr() + off), n))
    _workspaces[idx] = ws


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _cuda(t, name):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise BsgemmError(BS_ERR_DEVICE, f"{name} must be a CUDA tensor (there is no CPU path)")


def _bytes8(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype in (torch.float8_e4m3fn, torch.uint8, torch.int8):
        return t
    raise BsgemmError(BS_ERR_DTYPE, f"{name} must be float8_e4m3fn (or its uint8 bytes), got {t.dtype}")


def _empty_out(lead: tuple, N: int, dtype: torch.dtype, device) -> torch.Tensor:
    """Output [*lead, N] whose rows start on 16-byte boundaries (the kernels'
    store alignment): the last dimension is padded in memory, not in shape."""
    per16 = 16 // torch.empty((), dtype=dtype).element_size()
    Np = -(-N // per16) * per16
    return torch.empty((*lead, Np), dtype=dtype, device=device)[..., :N]


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def bs_gemm_fp8_blockwise(A: torch.Tensor, B: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
                          out_dtype: torch.dtype = torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """FP8 block-scaled GEMM: out = (A . expand(scale_a)) @ (B . expand(scale_b)).

    A       e4m3 [M, K] row-major (A.stride(1) == 1)
    B       e4m3 [K, N] column-major (B.stride(0) == 1), e.g. ``B_t.t()`` for B_t [N, K]
    scale_a fp32 [M, K/128] (1x128 groups, any strides)
    scale_b fp32 [K/128, N/128] (128x128 blocks, any strides)
    """
    for t, n in ((A, "A"), (B, "B"), (scale_a, "scale_a"), (scale_b, "scale_b")):
        _cuda(t, n)
    _bytes8(A, "A"), _bytes8(B, "B")
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise BsgemmError(BS_ERR_SHAPE, f"A [M,K] and B [K,N] expected, got {tuple(A.shape)} and {tuple(B.shape)}")
    M, K = A.shape
    N = B.shape[1]
    if scale_a.dtype != torch.float32 or scale_b.dtype != torch.float32:
        raise BsgemmError(BS_ERR_DTYPE, "scale_a and scale_b must be float32")
    if scale_a.dim() != 2 or scale_b.dim() != 2:
        raise BsgemmError(BS_ERR_SHAPE, "scale_a and scale_b must be 2-D")
    _check(lib().bs_check_blockwise_scale_shapes(M, N, K, *scale_a.shape, *scale_b.shape))
    if A.stride(1) != 1 and M > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"A must be row-major, got strides {A.stride()}")
    if B.stride(0) != 1 and N > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"B must be column-major, got strides {B.stride()}")
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise BsgemmError(BS_ERR_DTYPE, f"out_dtype must be bfloat16 or float32, got {out_dtype}")
    if out is None:
        out = _empty_out((M,), N, out_dtype, A.device)
    elif out.dtype != out_dtype or tuple(out.shape) != (M, N) or out.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "out must be a row-major [M, N] tensor of out_dtype")
    _ensure_workspace(A.device)
    with torch.cuda.device(A.device):
        _check(lib().bs_gemm_fp8_blockwise(
            _ptr(A), A.stride(0), _ptr(B), B.stride(1), _ptr(scale_a), scale_a.stride(0), scale_a.stride(1),
            _ptr(scale_b), scale_b.stride(0), scale_b.stride(1), _ptr(out), out.stride(0), _OUT_CODE[out_dtype],
            M, N, K, _stream(A.device)))
    return out


def bs_gemm_fp8_rowwise(A: torch.Tensor, B: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
                        bias: torch.Tensor | None = None, out_dtype: torch.dtype = torch.bfloat16,
                        out: torch.Tensor | None = None, scale_result: torch.Tensor | None = None,
                        use_fast_accum: bool = False) -> torch.Tensor:
    """FP8 GEMM with tensorwise or rowwise scales: out = (A @ B) * (scale_a * scale_b) + bias.

    A       e4m3 [M, K] row-major;  B e4m3 [K, N] column-major (``B_t.t()`` for B_t [N, K])
    scale_a fp32 scalar (tensorwise) or [M] / [M, 1] (rowwise)
    scale_b fp32 scalar (tensorwise) or [N] / [1, N] (rowwise), the same kind as scale_a
    bias    fp32 [N] or None
    out_dtype bfloat16, float32 or float8_e4m3fn (saturating round-to-nearest-even cast)
    scale_result fp32 scalar or None: an e4m3 result is scale_result * (the above) before
            its cast (the output scale of _scaled_mm); only with out_dtype float8_e4m3fn
    use_fast_accum accepted for _scaled_mm's signature; the tensor cores accumulate in fp32
            over all of K either way, so it changes nothing
    """
    del use_fast_accum
    for t, n in ((A, "A"), (B, "B"), (scale_a, "scale_a"), (scale_b, "scale_b")):
        _cuda(t, n)
    _bytes8(A, "A"), _bytes8(B, "B")
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise BsgemmError(BS_ERR_SHAPE, f"A [M,K] and B [K,N] expected, got {tuple(A.shape)} and {tuple(B.shape)}")
    M, K = A.shape
    N = B.shape[1]
    if scale_a.dtype != torch.float32 or scale_b.dtype != torch.float32:
        raise BsgemmError(BS_ERR_DTYPE, "scale_a and scale_b must be float32")
    tensorwise = scale_a.numel() == 1 and scale_b.numel() == 1 and scale_a.dim() in (0, 1) and scale_b.dim() in (0, 1)
    rowwise = tuple(scale_a.shape) in ((M,), (M, 1)) and tuple(scale_b.shape) in ((N,), (1, N))
    if not (tensorwise or rowwise):
        raise BsgemmError(BS_ERR_SHAPE, "tensorwise scales are scalars; rowwise scale_a is (M, 1) and scale_b (1, N); "
                                        f"got {tuple(scale_a.shape)} and {tuple(scale_b.shape)}")
    stride = 0 if tensorwise and not rowwise else 1
    if stride == 1:
        scale_a, scale_b = scale_a.reshape(-1).contiguous(), scale_b.reshape(-1).contiguous()
    if bias is not None:
        _cuda(bias, "bias")
        if bias.dtype != torch.float32 or bias.numel() != N:
            raise BsgemmError(BS_ERR_SHAPE, "bias must be float32 [N]")
        bias = bias.reshape(-1).contiguous()
    if scale_result is not None:
        _cuda(scale_result, "scale_result")
        if scale_result.dtype != torch.float32 or scale_result.numel() != 1:
            raise BsgemmError(BS_ERR_SHAPE, "scale_result must be a float32 scalar")
        scale_result = scale_result.reshape(-1).contiguous()
    if A.stride(1) != 1 and M > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"A must be row-major, got strides {A.stride()}")
    if B.stride(0) != 1 and N > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"B must be column-major, got strides {B.stride()}")
    if out_dtype not in (torch.bfloat16, torch.float32, torch.float8_e4m3fn):
        raise BsgemmError(BS_ERR_DTYPE, f"out_dtype must be bfloat16, float32 or float8_e4m3fn, got {out_dtype}")
    if out is None:
        out = _empty_out((M,), N, out_dtype, A.device)
    elif out.dtype != out_dtype or tuple(out.shape) != (M, N) or out.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "out must be a row-major [M, N] tensor of out_dtype")
    _ensure_workspace(A.device)
    with torch.cuda.device(A.device):
        _check(lib().bs_gemm_fp8_rowwise(
            _ptr(A), A.stride(0), _ptr(B), B.stride(1), _ptr(scale_a), stride, _ptr(scale_b), stride, _ptr(bias),
            _ptr(scale_result), _ptr(out), out.stride(0), _OUT_CODE[out_dtype], M, N, K, _stream(A.device)))
    return out


def int_scaled_mm(A: torch.Tensor, B: torch.Tensor, s_a: torch.Tensor | None, s_b: torch.Tensor | None = None,
                  out_dtype: torch.dtype = torch.float32, out: torch.Tensor | None = None) -> torch.Tensor:
    """INT8 GEMM with fused (float(acc) * s_a[m]) * s_b[n].

    A int8 [M, K] row-major; B int8 [K, N] column-major; s_a fp32 [M] / [M, 1] or None;
    s_b fp32 [N] / [1, N] or None.  out_dtype float32, bfloat16 or int32 (raw accumulator).
    """
    _cuda(A, "A"), _cuda(B, "B")
    if A.dtype != torch.int8 or B.dtype != torch.int8:
        raise BsgemmError(BS_ERR_DTYPE, "A and B must be int8")
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise BsgemmError(BS_ERR_SHAPE, f"A [M,K] and B [K,N] expected, got {tuple(A.shape)} and {tuple(B.shape)}")
    M, K = A.shape
    N = B.shape[1]
    sa = sb = None
    if s_a is not None:
        _cuda(s_a, "s_a")
        if s_a.dtype != torch.float32 or s_a.numel() != M:
            raise BsgemmError(BS_ERR_SHAPE, f"s_a must be float32 with M={M} elements")
        sa = s_a.reshape(M).contiguous()
    if s_b is not None:
        _cuda(s_b, "s_b")
        if s_b.dtype != torch.float32 or s_b.numel() != N:
            raise BsgemmError(BS_ERR_SHAPE, f"s_b must be float32 with N={N} elements")
        sb = s_b.reshape(N).contiguous()
    if A.stride(1) != 1 and M > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"A must be row-major, got strides {A.stride()}")
    if B.stride(0) != 1 and N > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"B must be column-major, got strides {B.stride()}")
    if out_dtype not in _OUT_CODE:
        raise BsgemmError(BS_ERR_DTYPE, f"out_dtype must be float32, bfloat16 or int32, got {out_dtype}")
    if out is None:
        out = _empty_out((M,), N, out_dtype, A.device)
    elif out.dtype != out_dtype or tuple(out.shape) != (M, N) or out.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "out must be a row-major [M, N] tensor of out_dtype")
    _ensure_workspace(A.device)
    with torch.cuda.device(A.device):
        _check(lib().int_scaled_mm(_ptr(A), A.stride(0), _ptr(B), B.stride(1), _ptr(sa), _ptr(sb), _ptr(out),
                                   out.stride(0), _OUT_CODE[out_dtype], M, N, K, _stream(A.device)))
    return out


def bs_int_scaled_mm_noalloc(A: torch.Tensor, B: torch.Tensor, s_a: torch.Tensor | None, s_b: torch.Tensor | None,
                             out: torch.Tensor) -> torch.Tensor:
    """int_scaled_mm through the entry point that allocates nothing (for callers that cannot allocate device
    memory): the wide kernel's stream-K split with the library's built-in scratch.  Results equal
    int_scaled_mm's.  Nothing is allocated here either: `out` (row-major [M, N], float32, bfloat16 or int32)
    must be given, and s_a / s_b must be contiguous float32 vectors or None.  The first call on a device sets
    up the scratch and belongs before any stream capture; calls that overlap on the GPU race on the scratch.
    """
    for t, name in ((A, "A"), (B, "B"), (out, "out")):
        _cuda(t, name)
    if A.dtype != torch.int8 or B.dtype != torch.int8:
        raise BsgemmError(BS_ERR_DTYPE, "A and B must be int8")
    if A.dim() != 2 or B.dim() != 2 or A.shape[1] != B.shape[0]:
        raise BsgemmError(BS_ERR_SHAPE, f"A [M,K] and B [K,N] expected, got {tuple(A.shape)} and {tuple(B.shape)}")
    M, K = A.shape
    N = B.shape[1]
    for s, n, name in ((s_a, M, "s_a"), (s_b, N, "s_b")):
        if s is not None:
            _cuda(s, name)
            if s.dtype != torch.float32 or s.numel() != n or not s.is_contiguous():
                raise BsgemmError(BS_ERR_SHAPE, f"{name} must be a contiguous float32 tensor of {n} elements")
    if A.stride(1) != 1 and M > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"A must be row-major, got strides {A.stride()}")
    if B.stride(0) != 1 and N > 1:
        raise BsgemmError(BS_ERR_LAYOUT, f"B must be column-major, got strides {B.stride()}")
    if out.dtype not in _OUT_CODE or tuple(out.shape) != (M, N) or out.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "out must be a row-major [M, N] float32, bfloat16 or int32 tensor")
    with torch.cuda.device(A.device):
        _check(lib().bs_int_scaled_mm_noalloc(_ptr(A), A.stride(0), _ptr(B), B.stride(1), _ptr(s_a), _ptr(s_b),
                                              _ptr(out), out.stride(0), _OUT_CODE[out.dtype], M, N, K,
                                              _stream(A.device)))
    return out


def _e8m0_bytes(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype == torch.uint8:
        return t
    if hasattr(torch, "float8_e8m0fnu") and t.dtype == torch.float8_e8m0fnu:
        return t.view(torch.uint8)
    raise BsgemmError(BS_ERR_DTYPE, f"{name} must hold e8m0 bytes (uint8 or float8_e8m0fnu), got {t.dtype}")


def bmm_a8w8_blockscale(x: torch.Tensor, w: torch.Tensor, x_scale: torch.Tensor, w_scale: torch.Tensor,
                        out_dtype: torch.dtype = torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """Batched FP8 GEMM with e8m0 block scales: out[m, g, :] = x[m, g, :] @ w[g]^T (dequantised).

    x        e4m3 [M, G, K] with x.stride(2) == 1 (m-major or batch-first storage)
    w        e4m3 [G, N, K] with w.stride(2) == 1
    x_scale  e8m0 [M, G, K/128] contiguous;  w_scale e8m0 [G, N/128, K/128] contiguous
    """
    for t, n in ((x, "x"), (w, "w"), (x_scale, "x_scale"), (w_scale, "w_scale")):
        _cuda(t, n)
    _bytes8(x, "x"), _bytes8(w, "w")
    xs, ws = _e8m0_bytes(x_scale, "x_scale"), _e8m0_bytes(w_scale, "w_scale")
    if x.dim() != 3 or w.dim() != 3 or x.shape[1] != w.shape[0] or x.shape[2] != w.shape[2]:
        raise BsgemmError(BS_ERR_SHAPE, f"x [M,G,K] and w [G,N,K] expected, got {tuple(x.shape)}, {tuple(w.shape)}")
    M, G, K = x.shape
    N = w.shape[1]
    KB, NB = -(-K // 128), -(-N // 128)
    if tuple(xs.shape) != (M, G, KB) or tuple(ws.shape) != (G, NB, KB):
        raise BsgemmError(BS_ERR_SHAPE, f"x_scale must be [{M},{G},{KB}] and w_scale [{G},{NB},{KB}], got "
                          f"{tuple(xs.shape)} and {tuple(ws.shape)}")
    if not xs.is_contiguous() or not ws.is_contiguous():
        raise BsgemmError(BS_ERR_LAYOUT, "x_scale and w_scale must be contiguous")
    if x.stride(2) != 1 or w.stride(2) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "x and w must have unit stride along K")
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise BsgemmError(BS_ERR_DTYPE, f"out_dtype must be bfloat16 or float32, got {out_dtype}")
    if out is None:
        out = _empty_out((M, G), N, out_dtype, x.device)
    elif out.dtype != out_dtype or tuple(out.shape) != (M, G, N) or out.stride(2) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "out must be [M, G, N] of out_dtype with unit stride along N")
    _ensure_workspace(x.device)
    with torch.cuda.device(x.device):
        _check(lib().bmm_a8w8_blockscale(
            _ptr(x), x.stride(0), x.stride(1), _ptr(w), w.stride(0), w.stride(1), _ptr(xs), _ptr(ws), _ptr(out),
            out.stride(0), out.stride(1), _OUT_CODE[out_dtype], M, G, N, K, _stream(x.device)))
    return out


# ---------------------------------------------------------------------------
# host-side helpers
# ---------------------------------------------------------------------------
OP_FP8_BLOCKWISE, OP_INT_SCALED_MM, OP_BMM, OP_FP8_ROWWISE = 1, 2, 3, 4


def bs_quantize_fp8_1x128(x: torch.Tensor, scale_format: str = "f32", q: torch.Tensor | None = None,
                          scale: torch.Tensor | None = None):
    """1x128 group quantisation of x [M, K] (bf16 or fp32, unit stride along K) to e4m3.

    scale_format "f32": scale fp32 [M, ceil(K/128)] = amax / 448 (1 for an all-zero group);
    scale_format "e8m0": scale uint8 [M, ceil(K/128)], the e8m0 byte of ceil(log2(amax / 448)).
    Returns (q, scale) with q as uint8 e4m3 codes [M, K] (rows padded to 16 bytes in memory).
    """
    _cuda(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "x must be [M, K] with unit stride along K")
    if x.dtype == torch.bfloat16:
        xd = 0
    elif x.dtype == torch.float32:
        xd = 1
    else:
        raise BsgemmError(BS_ERR_DTYPE, f"x must be bfloat16 or float32, got {x.dtype}")
    if scale_format not in ("f32", "e8m0"):
        raise BsgemmError(BS_ERR_DTYPE, f"unknown scale_format {scale_format!r}")
    M, K = x.shape
    KB = -(-K // 128)
    if q is None:
        q = _empty_out((M,), K, torch.uint8, x.device)
    if scale is None:
        scale = torch.empty((M, KB), dtype=torch.float32 if scale_format == "f32" else torch.uint8, device=x.device)
    _cuda(q, "q"), _cuda(scale, "scale")
    _check_quant_out(q, scale, scale_format)
    if q.shape != (M, K) or q.stride(1) != 1 or scale.shape != (M, KB) or scale.stride(1) != 1:
        raise BsgemmError(BS_ERR_SHAPE, "q must be [M, K] and scale [M, ceil(K/128)], unit stride along the last dim")
    _check(lib().bs_quantize_fp8_1x128(_ptr(x), xd, M, K, x.stride(0), _ptr(q), q.stride(0), _ptr(scale),
                                       0 if scale_format == "f32" else 1, scale.stride(0), _stream(x.device)))
    return q, scale


def _check_quant_out(q: torch.Tensor, scale: torch.Tensor, scale_format: str):
    if q.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise BsgemmError(BS_ERR_DTYPE, f"q must hold e4m3 bytes (uint8 or float8_e4m3fn), got {q.dtype}")
    want = torch.float32 if scale_format == "f32" else torch.uint8
    if scale.dtype != want:
        raise BsgemmError(BS_ERR_DTYPE, f"scale_format {scale_format!r} writes {want} scales, got {scale.dtype}")


def bs_quantize_fp8_t(x: torch.Tensor, group: str = "128x1", scale_format: str = "f32",
                      q_t: torch.Tensor | None = None, scale: torch.Tensor | None = None):
    """Transposed-output e4m3 quantisation of x [R, C] (bf16 or fp32, unit stride along C) for the
    backward GEMMs: q_t [C, R] (uint8 codes, rows padded to 16 bytes in memory), q_t[c, r] the code of x[r, c].

    group "128x1": one scale per column and 128-row block, scale [C, ceil(R/128)] (scale_a of A = q_t);
    group "128x128": one scale per 128 x 128 block, scale [ceil(R/128), ceil(C/128)] (scale_b of B_t = q_t).
    scale_format "f32" (amax / 448) or "e8m0" (uint8 bytes).  Returns (q_t, scale).
    """
    _cuda(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "x must be [R, C] with unit stride along C")
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise BsgemmError(BS_ERR_DTYPE, f"x must be bfloat16 or float32, got {x.dtype}")
    if scale_format not in ("f32", "e8m0"):
        raise BsgemmError(BS_ERR_DTYPE, f"unknown scale_format {scale_format!r}")
    if group not in ("128x1", "128x128"):
        raise BsgemmError(BS_ERR_SHAPE, f"unknown group {group!r}")
    R, C = x.shape
    RB, CB = -(-R // 128), -(-C // 128)
    sshape = (C, RB) if group == "128x1" else (RB, CB)
    if q_t is None:
        q_t = _empty_out((C,), R, torch.uint8, x.device)
    if scale is None:
        scale = torch.empty(sshape, dtype=torch.float32 if scale_format == "f32" else torch.uint8, device=x.device)
    _cuda(q_t, "q_t"), _cuda(scale, "scale")
    _check_quant_out(q_t, scale, scale_format)
    if q_t.shape != (C, R) or q_t.stride(1) != 1 or scale.shape != sshape or scale.stride(1) != 1:
        raise BsgemmError(BS_ERR_SHAPE, f"q_t must be [C, R] and scale {list(sshape)}, unit stride along the last dim")
    _check(lib().bs_quantize_fp8_t(_ptr(x), 0 if x.dtype == torch.bfloat16 else 1, R, C, x.stride(0), _ptr(q_t),
                                   q_t.stride(0), _ptr(scale), 0 if scale_format == "f32" else 1,
                                   0 if group == "128x1" else 1, scale.stride(0), _stream(x.device)))
    return q_t, scale


def bs_quantize_fp8_128x128(x: torch.Tensor, scale_format: str = "f32", q: torch.Tensor | None = None,
                            scale: torch.Tensor | None = None):
    """128x128 block quantisation of a weight x = W [R, C] (bf16 or fp32, unit stride along C) to e4m3 codes in
    its own orientation: q [R, C] (uint8, rows padded to 16 bytes in memory), q[r, c] the code of x[r, c].

    The scales come back as [ceil(C/128), ceil(R/128)]: for W [N, K] that is the scale_b [K/128, N/128] of
    bs_gemm_fp8_blockwise with B = q.t() (no transpose copy).  A ``scale`` passed in may have any strides;
    element (cb, rb) is the scale of the block of rows 128rb.. and columns 128cb..
    scale_format "f32" (amax / 448) or "e8m0" (uint8 bytes).  Returns (q, scale).
    """
    _cuda(x, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise BsgemmError(BS_ERR_LAYOUT, "x must be [R, C] with unit stride along C")
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise BsgemmError(BS_ERR_DTYPE, f"x must be bfloat16 or float32, got {x.dtype}")
    if scale_format not in ("f32", "e8m0"):
        raise BsgemmError(BS_ERR_DTYPE, f"unknown scale_format {scale_format!r}")
    R, C = x.shape
    RB, CB = -(-R // 128), -(-C // 128)
    if q is None:
        q = _empty_out((R,), C, torch.uint8, x.device)
    if scale is None:
        scale = torch.empty((CB, RB), dtype=torch.float32 if scale_format == "f32" else torch.uint8, device=x.device)
    _cuda(q, "q"), _cuda(scale, "scale")
    _check_quant_out(q, scale, scale_format)
    if q.shape != (R, C) or q.stride(1) != 1 or scale.shape != (CB, RB):
        raise BsgemmError(BS_ERR_SHAPE, f"q must be [R, C] with unit stride along C and scale [{CB}, {RB}]")
    with torch.cuda.device(x.device):
        _check(lib().bs_quantize_fp8_128x128(_ptr(x), 0 if x.dtype == torch.bfloat16 else 1, R, C, x.stride(0),
                                             _ptr(q), q.stride(0), _ptr(scale), 0 if scale_format == "f32" else 1,
                                             scale.stride(1), scale.stride(0), _stream(x.device)))
    return q, scale


quantize_fp8_1x128 = bs_quantize_fp8_1x128
quantize_fp8_t = bs_quantize_fp8_t
quantize_fp8_128x128 = bs_quantize_fp8_128x128


def plan_for(op: int, M: int, G: int, N: int, K: int, num_sms: int = 148) -> dict:
    p = Plan()
    _check(lib().bs_plan_for(op, M, G, N, K, num_sms, ctypes.byref(p)))
    return p.as_dict()


def set_split_override(splits: int) -> int:
    """Forces the skinny kernel's split-K factor (1, 2, 4, 8; 0 = automatic); returns the previous value."""
    return lib().bs_set_split_override(splits)


def set_stream_k(enable: bool) -> bool:
    """Enables or disables the stream-K split of the wide kernel's last wave (off by default: it measured
    slower than whole tiles on every shape tried); returns the previous setting.  While enabled, the
    first GEMM call on a device registers a workspace for it."""
    global _stream_k_on
    prev = bool(lib().bs_set_stream_k(1 if enable else 0))
    _stream_k_on = bool(enable)
    return prev


def workspace_size(num_sms: int) -> int:
    return int(lib().bs_workspace_size(num_sms))


def work_items(num_tiles: int, dp_tiles: int, sk_iters: int, kb: int, units: int, unit: int):
    """Host copy of the wide kernel's work decomposition: the (tile, kb0, kb1) items of one unit, in order."""
    n = lib().bs_work_items(num_tiles, dp_tiles, sk_iters, kb, units, unit, None, 0)
    if n < 0:
        raise BsgemmError(BS_ERR_SHAPE, "inconsistent work split")
    buf = (ctypes.c_int32 * (3 * max(n, 1)))()
    lib().bs_work_items(num_tiles, dp_tiles, sk_iters, kb, units, unit, buf, n)
    return [tuple(buf[3 * i:3 * i + 3]) for i in range(n)]


def set_path_override(path: int) -> int:
    return lib().bs_set_path_override(path)


def tile_order(grid_m: int, grid_n: int, batches: int = 1, group_m: int = 16):
    n = grid_m * grid_n * batches
    buf = (ctypes.c_int32 * (3 * n))()
    _check(lib().bs_tile_order(grid_m, grid_n, batches, group_m, buf, n))
    return [(buf[3 * i], buf[3 * i + 1], buf[3 * i + 2]) for i in range(n)]


def device_error(stream: torch.cuda.Stream | None = None) -> int:
    """Synchronise and read/clear the device error word (0 = no kernel timed out)."""
    code = ctypes.c_uint32(0)
    s = ctypes.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)
    st = lib().bs_get_device_error(s, ctypes.byref(code))
    if st not in (BS_OK, BS_ERR_TIMEOUT):
        _check(st)
    return code.value


def version() -> int:
    return lib().bs_version()

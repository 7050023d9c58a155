"""Seeded synthetic inputs for the scaled low-precision GEMMs.

This module only *makes inputs*: random values, their quantisation to the
low-precision storage formats and the scale tensors that go with them.  It
holds none of the GEMM arithmetic.  Both the CUDA path (tests, benchmark,
smoke run) and the CPU oracle consume what it returns, so that the two sides
see byte-identical operands.

Value recipe (shared by every workload):

* FP8 operands start as fp32 N(0, 1) draws; 1 % of the entries (chosen by an
  independent U[0, 1) < 0.01 draw) are multiplied by 20 to plant outliers.
* Activations A[M, K] are quantised per 1x128 group along K with
  ``scale = amax / 448`` (fp32), weights B[K, N] per 128x128 block.  The
  quantised code is ``e4m3_rne(clamp(x / scale, -448, 448))``; the clamp is
  the "saturation" of the recipe (``x / scale`` can land one ulp above 448
  and the plain fp32 -> e4m3fn cast would then give NaN).  A group whose amax
  is 0 gets scale 1.
* Batched-GEMM scales are e8m0 powers of two: ``e = ceil(log2(amax / 448))``
  taken exactly through frexp, stored as the byte ``e + 127`` clamped to
  [0, 254]; the operand code is ``e4m3_rne(x * 2**-e)``.
* INT8 operands are uniform integers in [-127, 127]; the row / column scales
  are ``10 ** (-3 + 2u)`` with u ~ U[0, 1) drawn in fp64 and cast to fp32.

Every tensor draws from its own CPU ``torch.Generator`` seeded with
``1000 * config + sweep_index + 10 * tensor_id``; inside one tensor the
order is ``randn`` then ``rand`` (outlier mask).  Weights are returned in the
K-major ("column-major B") storage the kernels read: ``B_t[N, K]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

E4M3_MAX = 448.0
GROUP = 128  # quantisation group / block edge along K (and N for weights)


# ---------------------------------------------------------------------------
# workload table (shapes of the five parity / benchmark configurations)
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    # "fp8_blockwise" | "int_scaled_mm" | "bmm_a8w8_blockscale" | "fp8_rowwise" | "quantize_1x128" | "quantize_t"
    # | "quantize_128x128"
    op: str
    M: int
    N: int
    K: int
    G: int = 1
    seed: int = 0  # configuration index; tensors seed from 1000 * seed
    extra: dict = field(default_factory=dict, compare=False, hash=False)


WORKLOADS = {
    "fp8_tiny_256x256x512": Workload("fp8_tiny_256x256x512", "fp8_blockwise", 256, 256, 512, seed=0),
    "int8_4096x4096x4096": Workload("int8_4096x4096x4096", "int_scaled_mm", 4096, 4096, 4096, seed=1),
    "fp8_16640x5120x8192": Workload("fp8_16640x5120x8192", "fp8_blockwise", 16640, 5120, 8192, seed=2),
    # the rowwise-scaled form of the same shape (the mode the blockwise issue's error message names)
    "fp8_rowwise_16640x5120x8192": Workload("fp8_rowwise_16640x5120x8192", "fp8_rowwise", 16640, 5120, 8192, seed=5),
    # the same, with an e4m3 result: output scale 448 / 4096 (a result amax of 4096, just above this data's)
    "fp8_rowwise_e4m3out_16640x5120x8192": Workload("fp8_rowwise_e4m3out_16640x5120x8192", "fp8_rowwise", 16640, 5120,
                                                    8192, seed=5, extra={"out": "e4m3", "scale_result": 0.109375}),
    # the activations of the 16640x5120x8192 shape, bf16, quantised to e4m3 per 1x128 group (fp32 scales)
    "quant_1x128_16640x8192_bf16": Workload("quant_1x128_16640x8192_bf16", "quantize_1x128", 16640, 0, 8192, seed=6),
    # the backward operands of the same layer, quantised transposed: the output gradient dy [16640, 5120] in
    # 128x1 groups (A of the weight gradient) and the activations x [16640, 8192] in 128x128 blocks (its B)
    "quant_t_128x1_16640x5120_bf16": Workload("quant_t_128x1_16640x5120_bf16", "quantize_t", 16640, 0, 5120, seed=7,
                                              extra={"group": "128x1"}),
    "quant_t_128x128_16640x8192_bf16": Workload("quant_t_128x128_16640x8192_bf16", "quantize_t", 16640, 0, 8192,
                                                seed=8, extra={"group": "128x128"}),
    # the weight W [5120, 8192] of the same layer, bf16, quantised to the forward GEMM's B_t in 128x128 blocks
    "quant_128x128_5120x8192_bf16": Workload("quant_128x128_5120x8192_bf16", "quantize_128x128", 5120, 0, 8192,
                                             seed=9),
}
BMM_M_SWEEP = (1, 16, 128, 1024, 16384)
BMM_G = (8, 2)
BMM_N, BMM_K = 1024, 4096
SKINNY_M_SWEEP = (1, 8, 32, 127, 255, 1000, 16383)
SKINNY_N, SKINNY_K = 7168, 2048

for _i, _m in enumerate(BMM_M_SWEEP):
    for _g in BMM_G:
        WORKLOADS[f"bmm_g{_g}_m{_m}"] = Workload(f"bmm_g{_g}_m{_m}", "bmm_a8w8_blockscale",
                                                 _m, BMM_N, BMM_K, G=_g, seed=3)
for _i, _m in enumerate(SKINNY_M_SWEEP):
    WORKLOADS[f"fp8_skinny_m{_m}"] = Workload(f"fp8_skinny_m{_m}", "fp8_blockwise",
                                              _m, SKINNY_N, SKINNY_K, seed=4)


def sweep_index(values, v) -> int:
    return list(values).index(v)


# ---------------------------------------------------------------------------
# primitive draws
# ---------------------------------------------------------------------------
def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_with_outliers(shape, seed: int) -> torch.Tensor:
    """fp32 N(0,1) with 1 % of the entries multiplied by 20."""
    g = _gen(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    mask = torch.rand(shape, generator=g, dtype=torch.float32) < 0.01
    x[mask] *= 20.0
    return x


def to_e4m3_bytes(x: torch.Tensor) -> torch.Tensor:
    """Saturating round-to-nearest-even cast to e4m3 (OCP fp8 E4M3), as raw bytes."""
    y = x.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return y.view(torch.uint8)


# ---------------------------------------------------------------------------
# FP8 blockwise: 1x128 activation groups, 128x128 weight blocks, fp32 scales
# ---------------------------------------------------------------------------
def quantize_groups_1x128(x: torch.Tensor):
    """x[R, K] fp32 -> (codes uint8 [R, K], scale fp32 [R, ceil(K/128)])."""
    R, K = x.shape
    KB = -(-K // GROUP)
    xp = torch.zeros(R, KB * GROUP, dtype=torch.float32)
    xp[:, :K] = x
    amax = xp.view(R, KB, GROUP).abs().amax(dim=-1)
    scale = amax / E4M3_MAX
    scale[scale == 0] = 1.0  # all-zero groups (and quotients that underflow)
    q = to_e4m3_bytes(xp / scale.repeat_interleave(GROUP, dim=1))
    return q[:, :K].contiguous(), scale.contiguous()


def quantize_blocks_128x128(w_kn: torch.Tensor):
    """w[K, N] fp32 -> (codes uint8 [K, N], scale fp32 [ceil(K/128), ceil(N/128)])."""
    K, N = w_kn.shape
    KB, NB = -(-K // GROUP), -(-N // GROUP)
    wp = torch.zeros(KB * GROUP, NB * GROUP, dtype=torch.float32)
    wp[:K, :N] = w_kn
    amax = wp.view(KB, GROUP, NB, GROUP).abs().amax(dim=(1, 3))
    scale = amax / E4M3_MAX
    scale[scale == 0] = 1.0  # all-zero groups (and quotients that underflow)
    full = scale.repeat_interleave(GROUP, dim=0).repeat_interleave(GROUP, dim=1)
    q = to_e4m3_bytes(wp / full)
    return q[:K, :N].contiguous(), scale.contiguous()


def fp8_blockwise_inputs(M: int, N: int, K: int, seed: int):
    """Inputs of ``bs_gemm_fp8_blockwise``.

    Returns a dict of CPU tensors:
      A       uint8 [M, K]    e4m3 codes, row-major
      B_t     uint8 [N, K]    e4m3 codes of B[K, N], stored K-major (column-major B)
      scale_a fp32  [M, K/128]
      scale_b fp32  [K/128, N/128]
    """
    a = normal_with_outliers((M, K), seed + 10 * 1)
    b = normal_with_outliers((K, N), seed + 10 * 2)
    A, sa = quantize_groups_1x128(a)
    Bkn, sb = quantize_blocks_128x128(b)
    return {"A": A, "B_t": Bkn.t().contiguous(), "scale_a": sa, "scale_b": sb}


def fp8_rowwise_inputs(M: int, N: int, K: int, seed: int, tensorwise: bool = False, bias: bool = True):
    """Inputs of ``bs_gemm_fp8_rowwise``: the same N(0,1)-with-outliers data quantised with one scale per
    row of A and per column of B (amax / 448), or one per operand when ``tensorwise``.

    Returns CPU tensors: A uint8 [M, K], B_t uint8 [N, K], scale_a fp32 [M, 1] or [], scale_b fp32 [1, N] or [],
    bias fp32 [N] (N(0,1)) or None."""
    a = normal_with_outliers((M, K), seed + 10 * 1)
    b = normal_with_outliers((N, K), seed + 10 * 2)

    def quant(x, per_row):
        amax = x.abs().amax(dim=1, keepdim=True) if per_row else x.abs().amax().reshape(1, 1)
        scale = amax / E4M3_MAX
        scale[scale == 0] = 1.0  # all-zero groups (and quotients that underflow)
        return to_e4m3_bytes(x / scale), scale

    A, sa = quant(a, not tensorwise)
    B_t, sb = quant(b, not tensorwise)
    if tensorwise:
        sa, sb = sa.reshape(()), sb.reshape(())
    else:
        sb = sb.reshape(1, N)
    out = {"A": A.contiguous(), "B_t": B_t.contiguous(), "scale_a": sa.contiguous(), "scale_b": sb.contiguous(),
           "bias": None}
    if bias:
        out["bias"] = torch.randn(N, generator=_gen(seed + 10 * 7), dtype=torch.float32)
    return out


# ---------------------------------------------------------------------------
# INT8 row/column scaled
# ---------------------------------------------------------------------------
def log_uniform(n: int, lo: float, hi: float, seed: int) -> torch.Tensor:
    g = _gen(seed)
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return torch.pow(10.0, math.log10(lo) + (math.log10(hi) - math.log10(lo)) * u).to(torch.float32)


def int8_inputs(M: int, N: int, K: int, seed: int):
    """Inputs of ``int_scaled_mm``: A int8 [M,K], B_t int8 [N,K], s_a fp32 [M], s_b fp32 [N]."""
    A = torch.randint(-127, 128, (M, K), generator=_gen(seed + 10 * 1), dtype=torch.int8)
    B = torch.randint(-127, 128, (K, N), generator=_gen(seed + 10 * 2), dtype=torch.int8)
    s_a = log_uniform(M, 1e-3, 1e-1, seed + 10 * 3)
    s_b = log_uniform(N, 1e-3, 1e-1, seed + 10 * 4)
    return {"A": A, "B_t": B.t().contiguous(), "s_a": s_a, "s_b": s_b}


# ---------------------------------------------------------------------------
# batched GEMM with e8m0 (power-of-two) block scales
# ---------------------------------------------------------------------------
def e8m0_exponent(amax: torch.Tensor) -> torch.Tensor:
    """ceil(log2(amax / 448)) computed exactly (fp64 + frexp); amax == 0 -> 0."""
    r = amax.to(torch.float64) / E4M3_MAX
    mant, ex = torch.frexp(r)
    e = torch.where(mant == 0.5, ex - 1, ex).to(torch.int64)
    return torch.where(amax == 0, torch.zeros_like(e), e)


def e8m0_bytes(e: torch.Tensor) -> torch.Tensor:
    return (e + 127).clamp(0, 254).to(torch.uint8)


def bmm_inputs(M: int, G: int, N: int, K: int, seed: int, batch_first: bool = False):
    """Inputs of ``bmm_a8w8_blockscale``.

    Returns CPU tensors:
      x        uint8 [M, G, K] e4m3 codes.  m-major storage (strides G*K, K, 1), or
               with ``batch_first`` a [G, M, K] buffer viewed as [M, G, K]
               (strides K, M*K, 1).
      w        uint8 [G, N, K] e4m3 codes (contiguous)
      x_scale  uint8 [M, G, K/128] e8m0 bytes
      w_scale  uint8 [G, N/128, K/128] e8m0 bytes
    """
    KB, NB = -(-K // GROUP), -(-N // GROUP)
    x = normal_with_outliers((M, G, K), seed + 10 * 5)
    w = normal_with_outliers((G, N, K), seed + 10 * 6)
    xp = torch.zeros(M, G, KB * GROUP)
    xp[..., :K] = x
    xe = e8m0_exponent(xp.view(M, G, KB, GROUP).abs().amax(-1))          # [M,G,KB]
    xe_b = e8m0_bytes(xe)
    xq = to_e4m3_bytes(xp * torch.pow(2.0, -(xe_b.to(torch.float64) - 127)).to(torch.float32)
                       .repeat_interleave(GROUP, dim=-1))[..., :K]
    wp = torch.zeros(G, NB * GROUP, KB * GROUP)
    wp[:, :N, :K] = w
    we = e8m0_exponent(wp.view(G, NB, GROUP, KB, GROUP).abs().amax(dim=(2, 4)))  # [G,NB,KB]
    we_b = e8m0_bytes(we)
    wfull = torch.pow(2.0, -(we_b.to(torch.float64) - 127)).to(torch.float32)
    wfull = wfull.repeat_interleave(GROUP, dim=1).repeat_interleave(GROUP, dim=2)
    wq = to_e4m3_bytes(wp * wfull)[:, :N, :K].contiguous()
    if batch_first:
        xs = xq.permute(1, 0, 2).contiguous().permute(1, 0, 2)  # storage [G, M, K]
    else:
        xs = xq.contiguous()
    return {"x": xs, "w": wq, "x_scale": xe_b.contiguous(), "w_scale": we_b.contiguous()}


def workload_inputs(w: Workload, sweep: int = 0, batch_first: bool = False):
    """Inputs for a named workload (seed = 1000*config + sweep)."""
    base = 1000 * w.seed + sweep
    if w.op == "fp8_blockwise":
        return fp8_blockwise_inputs(w.M, w.N, w.K, base)
    if w.op == "int_scaled_mm":
        return int8_inputs(w.M, w.N, w.K, base)
    if w.op == "fp8_rowwise":
        return fp8_rowwise_inputs(w.M, w.N, w.K, base)
    if w.op in ("quantize_1x128", "quantize_t", "quantize_128x128"):
        return {"x": normal_with_outliers((w.M, w.K), base + 10 * 7).to(torch.bfloat16)}
    return bmm_inputs(w.M, w.G, w.N, w.K, base, batch_first=batch_first)

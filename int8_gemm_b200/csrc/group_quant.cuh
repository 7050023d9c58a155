// Group-scale and e4m3 code arithmetic shared by the quantiser kernels.
//
// For a group with largest magnitude amax:
//   fp32 scale:  s = amax / 448 (1 when that quotient is 0), code = e4m3(x / s)
//   e8m0 scale:  byte = clamp(ceil(log2(amax / 448)) + 127, 0, 254) (127 when
//                amax == 0), code = e4m3(x * 2^-(byte - 127))
// with e4m3() rounding to nearest even and saturating at +-448, the largest
// finite e4m3 magnitude (pytorch issue "torch._scaled_mm with blockwise
// scaling doesn't work with torch.compile": one fp32 scale per group; ROCm/
// aiter PR "Add opus fp8 mxscale BMM kernels for gfx950": power-of-two scales).
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace bsg {

// Two saturating round-to-nearest-even e4m3 codes (first value in the low byte).
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// amax / 448, or 1 where that fp32 quotient is zero: an all-zero group, or a
// group whose amax is below 448 * 2^-150 so that the quotient underflows.
// The correctly rounded quotient comes from Markstein's correction step (see
// quotient_rn) with r = RN(1/448) = 0x1.24924ap-9 for every amax in
// [2^-116, FLT_MAX] -- an exhaustive check of those 2.05e9 fp32 values against
// the exactly rounded quotient found no difference -- and from an IEEE
// division below that range (and for inf or NaN).
__device__ __forceinline__ float group_scale_f32(float amax) {
  float s;
  if (amax >= 0x1p-116f && amax <= 3.40282347e38f) {
    constexpr float r = 0x1.24924ap-9f;
    const float q1 = __fmul_rn(amax, r);
    s = __fmaf_rn(__fmaf_rn(-q1, 448.f, amax), r, q1);
  } else {
    s = __fdiv_rn(amax, 448.f);
  }
  return s == 0.f ? 1.f : s;
}

// fp32(v / s) without an fp32 division per element: v times the fp64
// reciprocal of s (rinv = __drcp_rn(s)), rounded to fp32.  The fp64 product is
// within 2^-52 (relative) of v / s, while a quotient of two 24-bit-significand
// numbers is never an fp32 rounding midpoint and, when it is not exactly
// representable, lies at least 2^-49 (relative) away from every midpoint, so
// both round to the same fp32 value.  Quotients in the fp32 subnormal range
// map to e4m3 zero either way.
__device__ __forceinline__ float over_scale(float v, double rinv) {
  return __double2float_rn(__dmul_rn(static_cast<double>(v), rinv));
}

// fp32(v / s), correctly rounded, from fp32 operations on the FMA pipe.  With
// r = RN(1/s) and q1 = RN(v * r), the residual v - q1 * s is exact (one fma)
// and RN(q1 + residual * r) is the correctly rounded quotient -- Markstein's
// correction step (P. Markstein, IBM J. Res. Dev. 34(1), 1990) -- provided the
// residual does not underflow.  For a group scale s >= 2^-90 that holds for
// every quotient of magnitude >= 2^-11; smaller quotients give the e4m3 code
// zero with v's sign either way, and copysign keeps the sign of a zero v.  A
// CPU check over 1.3e9 (v, s) pairs, many of them chosen with quotients next to
// fp32 rounding midpoints, found no difference from the exact quotient.  Groups
// with smaller or non-finite scales take the fp64 path of over_scale.  (The
// fp64 path spends three fp32/fp64 conversions per element on the conversion
// pipe, which bounded the quantisers' throughput.)
__device__ __forceinline__ float quotient_rn(float v, float s, float r) {
  const float q1 = __fmul_rn(v, r);
  const float rem = __fmaf_rn(-q1, s, v);
  return copysignf(__fmaf_rn(rem, r, q1), v);
}

// Whether a group scale lies in quotient_rn's range.
__device__ __forceinline__ bool quotient_fast_range(float s) { return s >= 0x1p-90f && s <= 3.40282347e38f; }

// y[i] = fp32(v[i] / s) for the N elements of one group held by this thread.
// The fp32 path runs when every active lane of the warp has a scale in its
// range (a branch the warp takes together, so the fp64 conversions are not
// issued); otherwise the lanes take the fp64 path.
template <int N>
__device__ __forceinline__ void code_quotients(const float (&v)[N], float s, float (&y)[N]) {
  if (__all_sync(__activemask(), quotient_fast_range(s))) {
    const float r = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < N; ++i) y[i] = quotient_rn(v[i], s, r);
  } else {
    const double rinv = __drcp_rn(static_cast<double>(s));
#pragma unroll
    for (int i = 0; i < N; ++i) y[i] = over_scale(v[i], rinv);
  }
}

// y[i] = (fp32(v[i].x / s.x), fp32(v[i].y / s.y)) for N elements of two groups
// side by side (scales s.x and s.y): quotient_rn on both lanes of the packed
// two-wide fp32 operations when `fast` -- true on every lane of the warp or on
// none, and then r = (RN(1 / s.x), RN(1 / s.y)) -- else the fp64 path.  (-q1 * s
// and q1 * -s are the same exact product, so the residual is quotient_rn's.)
// Callers that code several runs of elements with one pair of scales compute
// `fast` and r once.
template <int N>
__device__ __forceinline__ void code_quotients2(const float2 (&v)[N], float2 s, float2 r, bool fast, float2 (&y)[N]) {
  if (fast) {
    const float2 ns = make_float2(-s.x, -s.y);
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float2 q1 = __fmul2_rn(v[i], r);
      const float2 rem = __ffma2_rn(q1, ns, v[i]);
      const float2 q = __ffma2_rn(rem, r, q1);
      y[i] = make_float2(copysignf(q.x, v[i].x), copysignf(q.y, v[i].y));
    }
  } else {
    const double r0 = __drcp_rn(static_cast<double>(s.x)), r1 = __drcp_rn(static_cast<double>(s.y));
#pragma unroll
    for (int i = 0; i < N; ++i) y[i] = make_float2(over_scale(v[i].x, r0), over_scale(v[i].y, r1));
  }
}

// The same with the range test (warp-uniform, over the active lanes) and the
// reciprocals worked out here.
template <int N>
__device__ __forceinline__ void code_quotients2(const float2 (&v)[N], float s0, float s1, float2 (&y)[N]) {
  const bool fast = __all_sync(__activemask(), quotient_fast_range(s0) && quotient_fast_range(s1));
  code_quotients2<N>(v, make_float2(s0, s1), make_float2(__frcp_rn(s0), __frcp_rn(s1)), fast, y);
}

// Lane-wise magnitude max of two bf16 pairs (exact: the result is one of the
// inputs' magnitudes); the result's sign bits are not meaningful, callers
// clear them.
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The e8m0 byte: ceil(log2(amax / 448)) from amax = f * 2^ex, f in [0.5, 1):
// with 448 = 0.875 * 2^9 it is ex - 9, plus one when f > 0.875.
__device__ __forceinline__ int group_e8m0(float amax) {
  int e = 0;
  if (amax != 0.f) {
    int ex;
    const float f = frexpf(amax, &ex);
    e = ex - 9 + (f > 0.875f ? 1 : 0);
  }
  return e + 127 < 0 ? 0 : (e + 127 > 254 ? 254 : e + 127);
}

}  // namespace bsg

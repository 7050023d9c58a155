// 1x128 activation-group quantisation to e4m3 for sm_100a (HBM-bound).
//
// For row m and group g (elements 128g .. min(128g + 128, K) - 1 of the row):
//   amax = max |x|
//   fp32 scales: scale = amax / 448 (1 when amax == 0), q = e4m3(x / scale)
//   e8m0 scales: byte = clamp(ceil(log2(amax / 448)) + 127, 0, 254) (127 when
//                amax == 0), q = e4m3(x * 2^-(byte - 127))
// with the e4m3 conversion rounding to nearest even and saturating at 448.
// These are the quantisation steps the blockwise operation's 1x128 activation
// groups (fp32 scale_a [M, K/128]) and the batched operation's e8m0 group
// scales presuppose (pytorch issue "torch._scaled_mm with blockwise scaling
// doesn't work with torch.compile"; ROCm/aiter PR "Add opus fp8 mxscale BMM
// kernels for gfx950"); 448 is the largest finite e4m3 magnitude.
//
// Eight lanes quantise one group: lane j holds elements 16j .. 16j + 15 (16-
// byte loads where the row's alignment allows, else element loads), three
// shuffle steps give the eight lanes the group's amax, and each lane writes
// its 16 codes as one 16-byte store, so a warp covers four consecutive groups
// of a row per pass, reading and writing them contiguously.  The per-group
// work (amax, scale, reciprocal) is shared by four groups per instruction.  A
// warp takes chunks of eight groups (two passes) and keeps all their loads in
// flight before it reduces any of them, then asks L2 for its next chunk while
// it quantises this one.  This kernel serves layouts the tensor copies cannot
// take; where x and q have 16-byte bases and row strides and K is a multiple of
// 16, the TMA-fed kernel of quant_ring.cuh runs instead.
#include <cuda_bf16.h>

#include "group_quant.cuh"
#include "quant_ring.cuh"
#include "quantize.h"

namespace bsg {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kLanesPerGroup = 8;                       // one 128-element group: 16 elements per lane
constexpr int kGroupsPerPass = 32 / kLanesPerGroup;     // groups one warp covers per pass
constexpr int kPasses = 2;                              // passes whose loads are in flight together
constexpr int kGroupsPerChunk = kGroupsPerPass * kPasses;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// 16 consecutive elements starting at element k of `row`; elements at or
// beyond K read as 0 (they do not change amax and are not stored).  `vec`:
// all 16 are inside the row and 16-byte aligned, so vector loads.
template <typename InT>
__device__ __forceinline__ void load16(const InT* row, long long k, long long K, bool vec, float (&v)[16]) {
  if (vec) {
    if constexpr (sizeof(InT) == 4) {
      const float4* p = reinterpret_cast<const float4*>(row + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = __ldg(p + i);
        v[4 * i] = t.x;
        v[4 * i + 1] = t.y;
        v[4 * i + 2] = t.z;
        v[4 * i + 3] = t.w;
      }
    } else {
      const uint4* p = reinterpret_cast<const uint4*>(row + k);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 t = __ldg(p + i);
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
          v[8 * i + 2 * j] = __low2float(h);
          v[8 * i + 2 * j + 1] = __high2float(h);
        }
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = k + i < K ? to_f32(row[k + i]) : 0.f;
  }
}

template <typename InT, int FMT>
__global__ void __launch_bounds__(kQuantThreads, 4)
    quantize_1x128_kernel(const InT* __restrict__ x, int M, long long K, long long ldx, uint8_t* __restrict__ q,
                          long long ldq, void* __restrict__ scale, long long lds) {
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerGroup;  // which group of a pass
  const int j = lane % kLanesPerGroup;    // 16-element slice of that group
  const int KB = static_cast<int>((K + 127) / 128);
  // a warp takes chunks of kGroupsPerChunk consecutive groups of one row
  const unsigned cpr = static_cast<unsigned>((KB + kGroupsPerChunk - 1) / kGroupsPerChunk);  // chunks per row
  const unsigned chunks = static_cast<unsigned>(M) * cpr;  // the host keeps this below 2^31
  const unsigned warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const unsigned nwarps = (gridDim.x * blockDim.x) >> 5;
  for (unsigned c = warp; c < chunks; c += nwarps) {
    const unsigned m = c / cpr;
    const int g0 = static_cast<int>(c - m * cpr) * kGroupsPerChunk;
    const InT* row = x + static_cast<long long>(m) * ldx;
    uint8_t* qrow = q + static_cast<long long>(m) * ldq;
    float v[kPasses][16];
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) {
      const int g = g0 + ps * kGroupsPerPass + sub;
      const long long k0 = static_cast<long long>(g) * 128;
      const bool vec = k0 + 128 <= K && (reinterpret_cast<uintptr_t>(row + k0) & 15u) == 0;
      load16<InT>(row, k0 + 16 * j, g < KB ? K : 0, vec, v[ps]);  // groups past the row read zeros
    }
    {  // the next chunk of this warp into L2 while this one is quantised
      const unsigned cn = c + nwarps;
      if (cn < chunks) {
        const unsigned mn = cn / cpr;
        const int gn0 = static_cast<int>(cn - mn * cpr) * kGroupsPerChunk;
#pragma unroll
        for (int ps = 0; ps < kPasses; ++ps) {
          const int g = gn0 + ps * kGroupsPerPass + sub;
          const long long k = static_cast<long long>(g) * 128 + 16 * j;
          if (g < KB && k < K)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(x + static_cast<long long>(mn) * ldx + k));
        }
      }
    }
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) {
      const int g = g0 + ps * kGroupsPerPass + sub;
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[ps][i]));
#pragma unroll
      for (int off = kLanesPerGroup / 2; off > 0; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      float y[16];
      if constexpr (FMT == 0) {
        const float s = group_scale_f32(amax);
        code_quotients<16>(v[ps], s, y);
        if (j == 0 && g < KB) static_cast<float*>(scale)[static_cast<long long>(m) * lds + g] = s;
      } else {
        const int byte = group_e8m0(amax);
        const float mul = ldexpf(1.f, 127 - byte);  // exact power of two
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = v[ps][i] * mul;
        if (j == 0 && g < KB) static_cast<uint8_t*>(scale)[static_cast<long long>(m) * lds + g] = static_cast<uint8_t>(byte);
      }
      if (g >= KB) continue;
      uint4 codes;
      codes.x = e4m3x2(y[0], y[1]) | (e4m3x2(y[2], y[3]) << 16);
      codes.y = e4m3x2(y[4], y[5]) | (e4m3x2(y[6], y[7]) << 16);
      codes.z = e4m3x2(y[8], y[9]) | (e4m3x2(y[10], y[11]) << 16);
      codes.w = e4m3x2(y[12], y[13]) | (e4m3x2(y[14], y[15]) << 16);
      const long long k0 = static_cast<long long>(g) * 128;
      const long long k = k0 + 16 * j;
      if (k0 + 128 <= K && (reinterpret_cast<uintptr_t>(qrow + k0) & 15u) == 0) {
        *reinterpret_cast<uint4*>(qrow + k) = codes;
      } else {
        const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (k + i < K) qrow[k + i] = static_cast<uint8_t>(w[i / 4] >> (8 * (i % 4)));
      }
    }
  }
}

template <typename InT, int FMT>
cudaError_t launch_q(const void* x, long long M, long long K, long long ldx, uint8_t* q, long long ldq, void* scale,
                     long long lds, int sms, cudaStream_t stream) {
  const long long chunks = M * (((K + 127) / 128 + kGroupsPerChunk - 1) / kGroupsPerChunk);
  long long blocks = (chunks * 32 + kQuantThreads - 1) / kQuantThreads;
  const long long cap = static_cast<long long>(sms > 0 ? sms : 148) * 8;  // 8 resident blocks per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_1x128_kernel<InT, FMT><<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
      static_cast<const InT*>(x), static_cast<int>(M), K, ldx, q, ldq, scale, lds);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_1x128(const void* x, bool x_bf16, long long M, long long K, long long ldx, uint8_t* q,
                                  long long ldq, void* scale, bool e8m0, long long lds, int sms,
                                  const CUtensorMap* tmx, const CUtensorMap* tmq, uint32_t* err,
                                  cudaStream_t stream) {
  if (tmx && tmq) {
    if (x_bf16)
      return e8m0 ? ring::launch_ring<__nv_bfloat16, 1, true>(*tmx, *tmq, M, K, scale, lds, 1, sms, err, stream)
                  : ring::launch_ring<__nv_bfloat16, 0, true>(*tmx, *tmq, M, K, scale, lds, 1, sms, err, stream);
    return e8m0 ? ring::launch_ring<float, 1, true>(*tmx, *tmq, M, K, scale, lds, 1, sms, err, stream)
                : ring::launch_ring<float, 0, true>(*tmx, *tmq, M, K, scale, lds, 1, sms, err, stream);
  }
  if (x_bf16)
    return e8m0 ? launch_q<__nv_bfloat16, 1>(x, M, K, ldx, q, ldq, scale, lds, sms, stream)
                : launch_q<__nv_bfloat16, 0>(x, M, K, ldx, q, ldq, scale, lds, sms, stream);
  return e8m0 ? launch_q<float, 1>(x, M, K, ldx, q, ldq, scale, lds, sms, stream)
              : launch_q<float, 0>(x, M, K, ldx, q, ldq, scale, lds, sms, stream);
}

}  // namespace bsg

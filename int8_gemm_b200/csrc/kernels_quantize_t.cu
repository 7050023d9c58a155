// Transposed-output e4m3 quantisation for the backward GEMMs (HBM-bound).
//
// x is [R, C]; the codes go to q_t [C, R], q_t[c][r] the code of x[r][c], so
// the dimension the backward GEMMs contract over (the rows of x: the tokens
// of an activation or an output gradient, the output features of a weight)
// becomes the contiguous one that the GEMM operands need.  Groups:
//   128x1:   rows 128rb .. 128rb + 127 of one column c, scale [C, ceil(R/128)]
//   128x128: a 128 x 128 block, scale [ceil(R/128), ceil(C/128)]
// with the scale and code rules of group_quant.cuh.  The blockwise linear
// layer's forward and backward benchmark (pytorch issue "torch._scaled_mm with
// blockwise scaling doesn't work with torch.compile") fixes two group shapes,
// 1x128 activation groups and 128x128 weight blocks; the backward operands
// take them along their contraction dimension: the output gradient's 128x1
// groups are the 1x128 groups of its transpose (scale_a of the weight-gradient
// GEMM), and 128x128 blocks give its scale_b.
//
// One CTA quantises a 128 x 128 tile at a time (persistent over tiles).  The
// tile is read row by row with 16-byte loads and kept in shared memory in the
// input type; thread t then owns column t % 128, rows 64 (t / 128) .. + 63,
// reading them down the column (a warp reads 32 consecutive elements of one
// row per step, no bank conflicts) once for the amax and once to quantise, so
// few registers are live and several CTAs share an SM: while one quantises,
// the others' loads are in flight.  The column halves' amaxes meet in shared
// memory (128x1), or the whole tile's in a block reduction (128x128).  Each
// thread writes its 64 codes, contiguous in q_t, as four 16-byte stores.
#include <cuda_bf16.h>

#include <cstring>

#include "group_quant.cuh"
#include "quantize.h"

namespace bsg {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
// CTAs per SM the register budget is sized for: four bf16 tiles (32 KB each),
// three fp32 tiles (64 KB each, which also hold twice the loads in flight)
template <typename InT>
constexpr int kMinBlocks = sizeof(InT) == 2 ? 4 : 3;

template <typename InT>
struct TileSmem {
  InT v[kTile][kTile];   // the tile, [row][column]
  float part[2][kTile];  // per-column amax of the two row halves
  float wmax[kThreads / 32];
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Tile rows are read as 16-byte vectors: 8 bf16 or 4 fp32 elements.
template <typename InT>
struct Vec {
  static constexpr int kElems = 16 / sizeof(InT);
  static constexpr int kPerRow = kTile / kElems;
  static constexpr int kPerThread = kTile * kPerRow / kThreads;
};

// GROUP 0: 128x1 groups; GROUP 1: 128x128 blocks.  FMT 0: fp32 scales; 1: e8m0.
// vec_x: x and its row stride allow 16-byte loads; vec_q: q_t and its row
// stride allow 16-byte stores.
template <typename InT, int FMT, int GROUP>
__global__ void __launch_bounds__(kThreads, kMinBlocks<InT>)
    quantize_t_kernel(const InT* __restrict__ x, long long R, long long C, long long ldx, uint8_t* __restrict__ q,
                      long long ldq, void* __restrict__ scale, long long lds, long long ctiles, long long ntiles,
                      bool vec_x, bool vec_q) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TileSmem<InT>& sm = *reinterpret_cast<TileSmem<InT>*>(smem_raw);
  using V = Vec<InT>;
  const int t = threadIdx.x;
  const int col = t % kTile;   // this thread's column in the compute phase
  const int half = t / kTile;  // and its half of the rows
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long rb = tile / ctiles, cb = tile - rb * ctiles;
    const long long r0 = rb * kTile, c0 = cb * kTile;
    __syncthreads();  // the previous tile's readers are done with the shared tile
    // load: vector i of the tile is row i / kPerRow, elements kElems * (i % kPerRow) ..
    uint4 raw[V::kPerThread];
#pragma unroll
    for (int k = 0; k < V::kPerThread; ++k) {
      const int i = k * kThreads + t;
      const long long r = r0 + i / V::kPerRow, c = c0 + (i % V::kPerRow) * V::kElems;
      const InT* src = x + r * ldx + c;
      if (vec_x && r < R && c + V::kElems <= C) {
        raw[k] = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        alignas(16) InT e[V::kElems];
#pragma unroll
        for (int j = 0; j < V::kElems; ++j) e[j] = (r < R && c + j < C) ? src[j] : InT(0.f);
        memcpy(&raw[k], e, sizeof(e));
      }
    }
#pragma unroll
    for (int k = 0; k < V::kPerThread; ++k) {
      const int i = k * kThreads + t;
      *reinterpret_cast<uint4*>(&sm.v[i / V::kPerRow][(i % V::kPerRow) * V::kElems]) = raw[k];
    }
    __syncthreads();
    // the amax of this thread's 64 values, down its column
    const InT* colp = &sm.v[64 * half][col];
    float amax = 0.f;
#pragma unroll 16
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(to_f32(colp[i * kTile])));
    if constexpr (GROUP == 0) {
      sm.part[half][col] = amax;
      __syncthreads();
      amax = fmaxf(sm.part[0][col], sm.part[1][col]);
    } else {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if ((t & 31) == 0) sm.wmax[t / 32] = amax;
      __syncthreads();
      amax = sm.wmax[0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, sm.wmax[w]);
    }
    const long long c = c0 + col;
    float s = 1.f;
    int byte = 127;
    if constexpr (FMT == 0) {
      s = group_scale_f32(amax);
    } else {
      byte = group_e8m0(amax);
    }
    const float mul = ldexpf(1.f, 127 - byte);  // exact power of two (e8m0)
    const bool owner = GROUP == 0 ? (half == 0 && c < C) : t == 0;
    if (owner) {
      const long long si = GROUP == 0 ? c * lds + rb : rb * lds + cb;
      if constexpr (FMT == 0) {
        static_cast<float*>(scale)[si] = s;
      } else {
        static_cast<uint8_t*>(scale)[si] = static_cast<uint8_t>(byte);
      }
    }
    if (c >= C) continue;  // a column past the matrix: nothing to store
    uint8_t* dst = q + c * ldq + r0 + 64 * half;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float e[16], y[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) e[j] = to_f32(colp[(16 * k + j) * kTile]);
      if constexpr (FMT == 0) {
        code_quotients<16>(e, s, y);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) y[j] = e[j] * mul;
      }
      uint4 codes;
      codes.x = e4m3x2(y[0], y[1]) | (e4m3x2(y[2], y[3]) << 16);
      codes.y = e4m3x2(y[4], y[5]) | (e4m3x2(y[6], y[7]) << 16);
      codes.z = e4m3x2(y[8], y[9]) | (e4m3x2(y[10], y[11]) << 16);
      codes.w = e4m3x2(y[12], y[13]) | (e4m3x2(y[14], y[15]) << 16);
      const long long r = r0 + 64 * half + 16 * k;
      if (vec_q && r + 16 <= R) {
        *reinterpret_cast<uint4*>(dst + 16 * k) = codes;
      } else {
        const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (r + j < R) dst[16 * k + j] = static_cast<uint8_t>(w[j / 4] >> (8 * (j % 4)));
      }
    }
  }
}

template <typename InT, int FMT, int GROUP>
cudaError_t launch_t(const void* x, long long R, long long C, long long ldx, uint8_t* q, long long ldq, void* scale,
                     long long lds, int sms, cudaStream_t stream) {
  const long long ctiles = (C + kTile - 1) / kTile;
  const long long ntiles = ((R + kTile - 1) / kTile) * ctiles;
  const size_t smem = sizeof(TileSmem<InT>);
  cudaError_t e = cudaFuncSetAttribute(quantize_t_kernel<InT, FMT, GROUP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;  // resident CTAs per SM (shared memory and registers): one wave, no stragglers
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_t_kernel<InT, FMT, GROUP>, kThreads, smem);
  if (e != cudaSuccess) return e;
  long long blocks = static_cast<long long>(sms > 0 ? sms : 148) * (per_sm > 0 ? per_sm : 1);
  if (blocks > ntiles) blocks = ntiles;
  if (blocks < 1) blocks = 1;
  const bool vec_x = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (ldx * static_cast<long long>(sizeof(InT))) % 16 == 0;
  const bool vec_q = (reinterpret_cast<uintptr_t>(q) & 15u) == 0 && ldq % 16 == 0;
  quantize_t_kernel<InT, FMT, GROUP><<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(
      static_cast<const InT*>(x), R, C, ldx, q, ldq, scale, lds, ctiles, ntiles, vec_x, vec_q);
  return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_t_fmt(const void* x, long long R, long long C, long long ldx, uint8_t* q, long long ldq,
                         void* scale, bool e8m0, bool block, long long lds, int sms, cudaStream_t stream) {
  if (block)
    return e8m0 ? launch_t<InT, 1, 1>(x, R, C, ldx, q, ldq, scale, lds, sms, stream)
                : launch_t<InT, 0, 1>(x, R, C, ldx, q, ldq, scale, lds, sms, stream);
  return e8m0 ? launch_t<InT, 1, 0>(x, R, C, ldx, q, ldq, scale, lds, sms, stream)
              : launch_t<InT, 0, 0>(x, R, C, ldx, q, ldq, scale, lds, sms, stream);
}

}  // namespace

cudaError_t launch_quantize_t(const void* x, bool x_bf16, long long R, long long C, long long ldx, uint8_t* q_t,
                              long long ldq, void* scale, bool e8m0, bool block128, long long lds, int sms,
                              cudaStream_t stream) {
  return x_bf16 ? launch_t_fmt<__nv_bfloat16>(x, R, C, ldx, q_t, ldq, scale, e8m0, block128, lds, sms, stream)
                : launch_t_fmt<float>(x, R, C, ldx, q_t, ldq, scale, e8m0, block128, lds, sms, stream);
}

}  // namespace bsg

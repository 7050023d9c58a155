// TMA-fed quantisation of 128 x 128 tiles in the input's own orientation, for
// 1x128 row groups (the activation quantiser) and 128x128 blocks (the forward
// weight quantiser); HBM-bound.
//
// Persistent CTAs (two of 256 threads per SM for bf16 input, one of 512 for
// fp32).  One thread keeps a ring of input tiles in flight with 2-D tensor
// copies (rows and columns past
// the matrix arrive as zeros) and writes each tile's codes back with one
// tensor store that clips at the matrix edge, so no thread spends
// instructions or registers on global loads or stores.  Eight threads
// share a tile row, 16 elements each, reading it from shared memory as
// 16-byte pieces (the eight threads of a row take 128 contiguous bytes per
// load); the amax of a row group comes from those eight threads, the amax of a
// block from a warp then block reduction (bf16: one packed magnitude max per
// element pair), so each thread's scale arithmetic serves 16 or 32 elements;
// each piece's 8 (bf16) or 4 (fp32) codes go to the same place of a shared
// code tile.  Scale and code rules: group_quant.cuh.
//
// The caller guarantees 16-byte bases and row strides for x and q and a
// column count that is a multiple of 16, so that every row of either ends on
// a 16-byte boundary.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "group_quant.cuh"
#include "quantize.h"
#include "sm100.cuh"
#include "tile_ring.cuh"

namespace bsg {
namespace ring {

constexpr int kTile = 128;

// bf16: two CTAs of 256 threads per SM, each with two input and two code
// tiles (96 KB), so that one CTA's reductions and barriers overlap the other's
// work; fp32: one CTA of 512 threads with three input tiles and one code tile
// (208 KB).
template <typename InT>
struct Ring {
  static constexpr bool kPair = sizeof(InT) == 2;
  static constexpr int kThreads = kPair ? 256 : 512;
  static constexpr int kCtasPerSm = kPair ? 2 : 1;
  static constexpr int kStages = kPair ? 2 : 3;                // input tiles (32 or 64 KB each)
  static constexpr int kCodeBufs = kPair ? 2 : 1;              // code tiles (16 KB each)
  static constexpr int kElems = 16 / sizeof(InT);             // elements per 16-byte piece
  static constexpr int kRowThreads = 8;                       // threads sharing a tile row
  static constexpr int kPieces = kTile / kElems / kRowThreads;  // a thread's pieces of a row (16 elements)
  static constexpr int kRowsPerPass = kThreads / kRowThreads;
  static constexpr int kPasses = kTile / kRowsPerPass;          // rows per thread
};

template <typename InT>
struct Smem {
  alignas(1024) InT v[Ring<InT>::kStages][kTile][kTile];          // input tiles, [row][column]
  alignas(1024) uint8_t codes[Ring<InT>::kCodeBufs][kTile][kTile];  // code tiles, [row][column], 128-byte swizzle
  float wmax[Ring<InT>::kThreads / 32];
  uint64_t full[Ring<InT>::kStages];
  int abort;
};

// The amax of a piece's elements.
__device__ __forceinline__ float piece_amax(const uint4& v, __nv_bfloat16) {
  const uint32_t m = max_abs_bf16x2(max_abs_bf16x2(v.x, v.y), max_abs_bf16x2(v.z, v.w));
  return fmaxf(__uint_as_float((m << 16) & 0x7FFFFFFFu), __uint_as_float(m & 0x7FFF0000u));
}
__device__ __forceinline__ float piece_amax(const uint4& v, float) {
  return fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
               fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
}

// A piece's elements as fp32 pairs (exact widening for bf16).
__device__ __forceinline__ void piece_pairs(const uint4& v, float2 (&e)[4]) {  // bf16: 8 elements
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) e[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}
__device__ __forceinline__ void piece_pairs(const uint4& v, float2 (&e)[2]) {  // fp32: 4 elements
  e[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
  e[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}

// FMT 0: fp32 scales, 1: e8m0 bytes.  ROWS: one scale per row and 128-column
// block (1x128 groups), at scale[row * s_r + column block * s_c]; otherwise
// one per 128 x 128 block, at scale[row block * s_r + column block * s_c].
template <typename InT, int FMT, bool ROWS>
__global__ void __launch_bounds__(Ring<InT>::kThreads, Ring<InT>::kCtasPerSm)
    quantize_ring_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmq, long long R,
                         void* __restrict__ scale, long long s_r, long long s_c, long long ctiles, long long ntiles,
                         uint32_t* err) {
  using G = Ring<InT>;
  using S = Smem<InT>;
  constexpr uint32_t kTileBytes = kTile * kTile * sizeof(InT);
  constexpr int kPairs = G::kElems / 2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + sizeof(S) > dynamic_smem_bytes()) {  // never touch memory the launch did not provide
    if (threadIdx.x == 0) record_error(err, kErrSmemTooSmall);
    return;
  }
  S& sm = *reinterpret_cast<S*>(smem_raw + pad);
  const int t = threadIdx.x;
  // Thread t holds pieces j8 + 8 i (i < kPieces) of rows row0 + kRowsPerPass k,
  // j8 = t % 8.  A warp's four row slots take rows r, r + 4, r + 8, r + 12 so
  // that under the code tile's 128-byte swizzle (16-byte piece c of row r at
  // c ^ (r % 8)) the warp's code stores fall on every bank equally.
  const int j8 = t % G::kRowThreads;
  const int w = t / 32, slot = (t % 32) / G::kRowThreads;
  const int row0 = (w / 4) * 16 + (w % 4) + 4 * slot;
  const TileRing<G::kStages, G::kCodeBufs> ring{sm.full, &sm.abort, &tmx, reinterpret_cast<uint8_t*>(&sm.v[0][0][0]),
                                                kTileBytes, ctiles, ntiles};
  if (t == 0) ring.init(&tmq);
  __syncthreads();
  // x may come from the previous kernel in the stream, which may also still read
  // q and the scales: every global access comes after this wait
  grid_dependency_wait();
  grid_launch_dependents();
  if (t == 0) ring.start();
  int it = 0;
  bool ok = true;
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int st = it % G::kStages, cbuf = it % G::kCodeBufs;
    const long long rb = tile / ctiles, cb = tile - rb * ctiles;
    const bool got = ring.wait(it, err);
    uint4 v[G::kPasses][G::kPieces];
#pragma unroll
    for (int k = 0; k < G::kPasses; ++k)
#pragma unroll
      for (int i = 0; i < G::kPieces; ++i)
        v[k][i] = *reinterpret_cast<const uint4*>(
            &sm.v[st][row0 + k * G::kRowsPerPass][(j8 + G::kRowThreads * i) * G::kElems]);
    float amax[G::kPasses];  // ROWS: the amax of each of this thread's rows; else of the tile
#pragma unroll
    for (int k = 0; k < G::kPasses; ++k) {
      amax[k] = piece_amax(v[k][0], InT());
#pragma unroll
      for (int i = 1; i < G::kPieces; ++i) amax[k] = fmaxf(amax[k], piece_amax(v[k][i], InT()));
    }
    if constexpr (ROWS) {
#pragma unroll
      for (int k = 0; k < G::kPasses; ++k)
#pragma unroll
        for (int off = G::kRowThreads / 2; off > 0; off >>= 1)
          amax[k] = fmaxf(amax[k], __shfl_xor_sync(0xffffffffu, amax[k], off));
    } else {
      float a = amax[0];
#pragma unroll
      for (int k = 1; k < G::kPasses; ++k) a = fmaxf(a, amax[k]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if ((t & 31) == 0) sm.wmax[t / 32] = a;
    }
    if (t == 0) ring.code_tile_free();
    // every thread holds its pieces: the stage can be refilled
    ok = __syncthreads_and(got) != 0;
    if (!ok) break;
    if (t == 0) ring.refill(tile, it);
    if constexpr (!ROWS) {
      float a = sm.wmax[0];
#pragma unroll
      for (int w = 1; w < G::kThreads / 32; ++w) a = fmaxf(a, sm.wmax[w]);
#pragma unroll
      for (int k = 0; k < G::kPasses; ++k) amax[k] = a;
    }
#pragma unroll
    for (int k = 0; k < G::kPasses; ++k) {
      const int row = row0 + k * G::kRowsPerPass;
      // the group's scale, written once: by each row's first thread (ROWS) or the tile's first thread
      const bool writer = ROWS ? (j8 == 0 && rb * kTile + row < R) : (t == 0 && k == 0);
      const long long si = (ROWS ? rb * kTile + row : rb) * s_r + cb * s_c;
      float s = 1.f, mul = 1.f, r = 1.f;
      bool fast = true;
      if constexpr (FMT == 0) {
        s = group_scale_f32(amax[k]);
        if (writer) static_cast<float*>(scale)[si] = s;
        fast = __all_sync(0xffffffffu, quotient_fast_range(s));  // every thread of the CTA is here
        r = __frcp_rn(s);
      } else {
        const int byte = group_e8m0(amax[k]);
        if (writer) static_cast<uint8_t*>(scale)[si] = static_cast<uint8_t>(byte);
        mul = ldexpf(1.f, 127 - byte);  // exact power of two
      }
#pragma unroll
      for (int i = 0; i < G::kPieces; ++i) {
        float2 e[kPairs], y[kPairs];
        piece_pairs(v[k][i], e);
        if constexpr (FMT == 0) {
          code_quotients2<kPairs>(e, make_float2(s, s), make_float2(r, r), fast, y);
        } else {
#pragma unroll
          for (int h = 0; h < kPairs; ++h) y[h] = __fmul2_rn(e[h], make_float2(mul, mul));
        }
        // byte offset of the piece's codes in the row, then the swizzled 16-byte piece
        const int b = (j8 + G::kRowThreads * i) * G::kElems;
        uint8_t* dst = &sm.codes[cbuf][row][(((b >> 4) ^ (row & 7)) << 4) | (b & 15)];
        if constexpr (kPairs == 4) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(e4m3x2(y[0].x, y[0].y) | (e4m3x2(y[1].x, y[1].y) << 16),
                                                      e4m3x2(y[2].x, y[2].y) | (e4m3x2(y[3].x, y[3].y) << 16));
        } else {
          *reinterpret_cast<uint32_t*>(dst) = e4m3x2(y[0].x, y[0].y) | (e4m3x2(y[1].x, y[1].y) << 16);
        }
      }
    }
    fence_proxy_async_smem();  // the code tile, before the tensor store reads it
    __syncthreads();
    if (t == 0) ring.store(&tmq, &sm.codes[cbuf][0][0], cb * kTile, rb * kTile);
  }
  if (t == 0) ring.finish(ok, it);
}

// tmx / tmq: x and q [R, C] as tensors of 128 x 128 boxes, x without swizzle,
// q with the 128-byte swizzle.
template <typename InT, int FMT, bool ROWS>
cudaError_t launch_ring(const CUtensorMap& tmx, const CUtensorMap& tmq, long long R, long long C, void* scale,
                        long long s_r, long long s_c, int sms, uint32_t* err, cudaStream_t stream) {
  const long long ctiles = (C + kTile - 1) / kTile;
  const long long ntiles = ((R + kTile - 1) / kTile) * ctiles;
  const size_t smem = sizeof(Smem<InT>) + 1024;
  int per_sm = 1;
  const cudaError_t e = ctas_per_sm_once<quantize_ring_kernel<InT, FMT, ROWS>>(Ring<InT>::kThreads, smem, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm > Ring<InT>::kCtasPerSm) per_sm = Ring<InT>::kCtasPerSm;
  long long blocks = static_cast<long long>(sms > 0 ? sms : 148) * per_sm;
  if (blocks > ntiles) blocks = ntiles;
  cudaLaunchAttribute attr[1];
  // programmatic dependent launch: the set-up may overlap the previous kernel in the stream
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(Ring<InT>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_ring_kernel<InT, FMT, ROWS>, tmx, tmq, R, scale, s_r, s_c, ctiles, ntiles,
                            err);
}

}  // namespace ring
}  // namespace bsg

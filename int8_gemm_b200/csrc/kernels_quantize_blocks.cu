// 128x128 block quantisation in the input's own orientation (HBM-bound): the
// weight operand of the forward GEMM.  A weight W [N, K] becomes the codes
// B_t [N, K] that bs_gemm_fp8_blockwise reads as its column-major B, with one
// scale per 128 x 128 block; the block scale matrix, indexed (n-block,
// k-block), is the transpose of that GEMM's scale_b [K/128, N/128] (pytorch
// issue "torch._scaled_mm with blockwise scaling doesn't work with
// torch.compile": 128x128 weight blocks, scale_b (64, 40) for K = 8192,
// N = 5120).  Scale and code rules: group_quant.cuh.
//
// One CTA of 256 threads quantises a 128 x 128 tile at a time (persistent over
// tiles, one wave of CTAs).  Consecutive threads read consecutive 16-byte
// pieces of a tile row, so every warp load is a contiguous run of the row;
// each thread keeps its pieces in registers (8 of bf16 or 16 of fp32), the
// tile amax comes from a warp then block reduction, and each piece is written
// back as its 8 (bf16) or 4 (fp32) codes at the same place in q.  Several
// CTAs share an SM, so one CTA's loads are in flight while another reduces.
// This kernel serves layouts the tensor copies cannot take; where x and q have
// 16-byte bases and row strides and C is a multiple of 16, the TMA-fed kernel
// of quant_ring.cuh runs instead.
#include <cuda_bf16.h>

#include <cstring>

#include "group_quant.cuh"
#include "quant_ring.cuh"
#include "quantize.h"

namespace bsg {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;

template <typename InT>
struct Pieces {
  static constexpr int kElems = 16 / sizeof(InT);          // elements per 16-byte piece
  static constexpr int kPerRow = kTile / kElems;           // pieces per tile row
  static constexpr int kRowsPerPass = kThreads / kPerRow;  // tile rows one pass of the CTA covers
  static constexpr int kPasses = kTile / kRowsPerPass;     // pieces per thread
};

// Element j of a 16-byte piece, widened to fp32 (exact for bf16).
template <typename InT>
__device__ __forceinline__ float piece_elem(const uint4& v, int j) {
  const uint32_t w = (&v.x)[j * static_cast<int>(sizeof(InT)) / 4];
  if constexpr (sizeof(InT) == 2) {
    return __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
  } else {
    return __uint_as_float(w);
  }
}

// FMT 0: fp32 scales; 1: e8m0 bytes.  vec_x: x and its row stride allow
// 16-byte loads; vec_q: q and its row stride allow the 8-byte (bf16) or
// 4-byte (fp32) code stores.
// Three bf16 CTAs (two fp32) per SM: a register budget that keeps one CTA's
// tile loads in flight while the others reduce and store.
template <typename InT>
constexpr int kBlocksMinCtas = sizeof(InT) == 2 ? 3 : 2;

template <typename InT, int FMT>
__global__ void __launch_bounds__(kThreads, kBlocksMinCtas<InT>)
    quantize_blocks_kernel(const InT* __restrict__ x, long long R, long long C, long long ldx,
                           uint8_t* __restrict__ q, long long ldq, void* __restrict__ scale, long long s_rb,
                           long long s_cb, long long ctiles, long long ntiles, bool vec_x, bool vec_q) {
  using P = Pieces<InT>;
  __shared__ float wmax[2][kThreads / 32];  // per-warp amaxes, double-buffered across tiles
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int piece = t % P::kPerRow;  // this thread's piece within a row
  const int row0 = t / P::kPerRow;   // and its first row within the tile
  int parity = 0;
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, parity ^= 1) {
    const long long rb = tile / ctiles, cb = tile - rb * ctiles;
    const long long c = cb * kTile + piece * P::kElems;  // first column of this thread's pieces
    uint4 v[P::kPasses];
#pragma unroll
    for (int k = 0; k < P::kPasses; ++k) {
      const long long r = rb * kTile + row0 + k * P::kRowsPerPass;
      const InT* src = x + r * ldx + c;
      if (vec_x && r < R && c + P::kElems <= C) {
        v[k] = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        alignas(16) InT e[P::kElems];
#pragma unroll
        for (int j = 0; j < P::kElems; ++j) e[j] = (r < R && c + j < C) ? src[j] : InT(0.f);
        memcpy(&v[k], e, sizeof(e));
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < P::kPasses; ++k)
#pragma unroll
      for (int j = 0; j < P::kElems; ++j) amax = fmaxf(amax, fabsf(piece_elem<InT>(v[k], j)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) wmax[parity][warp] = amax;
    __syncthreads();
    amax = wmax[parity][0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, wmax[parity][w]);
    float s = 1.f;
    int byte = 127;
    if constexpr (FMT == 0) {
      s = group_scale_f32(amax);
    } else {
      byte = group_e8m0(amax);
    }
    const float mul = ldexpf(1.f, 127 - byte);  // exact power of two (e8m0)
    if (t == 0) {
      const long long si = rb * s_rb + cb * s_cb;
      if constexpr (FMT == 0) {
        static_cast<float*>(scale)[si] = s;
      } else {
        static_cast<uint8_t*>(scale)[si] = static_cast<uint8_t>(byte);
      }
    }
#pragma unroll
    for (int k = 0; k < P::kPasses; ++k) {
      const long long r = rb * kTile + row0 + k * P::kRowsPerPass;
      if (r >= R) continue;
      float e[P::kElems], y[P::kElems];
#pragma unroll
      for (int j = 0; j < P::kElems; ++j) e[j] = piece_elem<InT>(v[k], j);
      if constexpr (FMT == 0) {
        code_quotients<P::kElems>(e, s, y);
      } else {
#pragma unroll
        for (int j = 0; j < P::kElems; ++j) y[j] = e[j] * mul;
      }
      uint32_t w[P::kElems / 4];
#pragma unroll
      for (int i = 0; i < P::kElems / 4; ++i)
        w[i] = e4m3x2(y[4 * i], y[4 * i + 1]) | (e4m3x2(y[4 * i + 2], y[4 * i + 3]) << 16);
      uint8_t* dst = q + r * ldq + c;
      if (vec_q && c + P::kElems <= C) {
        if constexpr (P::kElems == 8) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        } else {
          *reinterpret_cast<uint32_t*>(dst) = w[0];
        }
      } else {
#pragma unroll
        for (int j = 0; j < P::kElems; ++j)
          if (c + j < C) dst[j] = static_cast<uint8_t>(w[j / 4] >> (8 * (j % 4)));
      }
    }
  }
}

template <typename InT, int FMT>
cudaError_t launch_blocks(const void* x, long long R, long long C, long long ldx, uint8_t* q, long long ldq,
                          void* scale, long long s_rb, long long s_cb, int sms, cudaStream_t stream) {
  const long long ctiles = (C + kTile - 1) / kTile;
  const long long ntiles = ((R + kTile - 1) / kTile) * ctiles;
  int per_sm = 1;  // resident CTAs per SM: one wave of persistent CTAs
  const cudaError_t e = ctas_per_sm_once<quantize_blocks_kernel<InT, FMT>>(kThreads, 0, &per_sm);
  if (e != cudaSuccess) return e;
  long long blocks = static_cast<long long>(sms > 0 ? sms : 148) * per_sm;
  if (blocks > ntiles) blocks = ntiles;
  if (blocks < 1) blocks = 1;
  constexpr long long kStoreBytes = 16 / static_cast<long long>(sizeof(InT));  // codes per piece
  const bool vec_x = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (ldx * static_cast<long long>(sizeof(InT))) % 16 == 0;
  const bool vec_q = (reinterpret_cast<uintptr_t>(q) % kStoreBytes) == 0 && ldq % kStoreBytes == 0;
  quantize_blocks_kernel<InT, FMT><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const InT*>(x), R, C, ldx, q, ldq, scale, s_rb, s_cb, ctiles, ntiles, vec_x, vec_q);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_blocks(const void* x, bool x_bf16, long long R, long long C, long long ldx, uint8_t* q,
                                   long long ldq, void* scale, bool e8m0, long long s_rb, long long s_cb, int sms,
                                   const CUtensorMap* tmx, const CUtensorMap* tmq, uint32_t* err,
                                   cudaStream_t stream) {
  if (tmx && tmq) {
    if (x_bf16)
      return e8m0 ? ring::launch_ring<__nv_bfloat16, 1, false>(*tmx, *tmq, R, C, scale, s_rb, s_cb, sms, err, stream)
                  : ring::launch_ring<__nv_bfloat16, 0, false>(*tmx, *tmq, R, C, scale, s_rb, s_cb, sms, err, stream);
    return e8m0 ? ring::launch_ring<float, 1, false>(*tmx, *tmq, R, C, scale, s_rb, s_cb, sms, err, stream)
                : ring::launch_ring<float, 0, false>(*tmx, *tmq, R, C, scale, s_rb, s_cb, sms, err, stream);
  }
  if (x_bf16)
    return e8m0 ? launch_blocks<__nv_bfloat16, 1>(x, R, C, ldx, q, ldq, scale, s_rb, s_cb, sms, stream)
                : launch_blocks<__nv_bfloat16, 0>(x, R, C, ldx, q, ldq, scale, s_rb, s_cb, sms, stream);
  return e8m0 ? launch_blocks<float, 1>(x, R, C, ldx, q, ldq, scale, s_rb, s_cb, sms, stream)
              : launch_blocks<float, 0>(x, R, C, ldx, q, ldq, scale, s_rb, s_cb, sms, stream);
}

}  // namespace bsg

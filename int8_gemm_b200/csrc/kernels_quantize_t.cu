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
// input type; thread t then owns the column pair 2 (t % 64), 2 (t % 64) + 1
// and rows 32 (t / 64) .. + 31, reading both columns with one 4-byte (bf16)
// or 8-byte (fp32) shared load per row (a warp reads 64 consecutive elements
// of one row per step, no bank conflicts), once for the amax and once to
// quantise, so few registers are live and several CTAs share an SM: while one
// quantises, the others' loads are in flight.  The four row quarters' column
// amaxes meet in shared memory (128x1), or the whole tile's in a block
// reduction (128x128).  Each thread writes its 2 x 32 codes, contiguous in two
// rows of q_t, as 16-byte stores.
#include <cuda_bf16.h>

#include <cstring>
#include <type_traits>

#include "group_quant.cuh"
#include "quantize.h"
#include "sm100.cuh"
#include "tile_ring.cuh"

namespace bsg {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
// CTAs per SM the register budget is sized for: four bf16 tiles (32 KB each),
// three fp32 tiles (64 KB each, which also hold twice the loads in flight)
template <typename InT>
constexpr int kMinBlocks = sizeof(InT) == 2 ? 4 : 3;

constexpr int kQuarters = kThreads / (kTile / 2);  // row quarters: threads per column pair
constexpr int kRowsPerThread = kTile / kQuarters;

template <typename InT>
struct TileSmem {
  InT v[kTile][kTile];          // the tile, [row][column]
  float part[kQuarters][kTile];  // per-column amax of the row quarters
  float wmax[kThreads / 32];
};

// Elements (row, 2p) and (row, 2p + 1) of the shared tile, widened to fp32
// (exact for bf16), with one shared load.
__device__ __forceinline__ void pair_at(const TileSmem<__nv_bfloat16>& sm, int row, int p, float& a, float& b) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(&sm.v[row][2 * p]);
  a = __uint_as_float(w << 16);
  b = __uint_as_float(w & 0xFFFF0000u);
}
__device__ __forceinline__ void pair_at(const TileSmem<float>& sm, int row, int p, float& a, float& b) {
  const float2 w = *reinterpret_cast<const float2*>(&sm.v[row][2 * p]);
  a = w.x;
  b = w.y;
}

// 16 codes of one column to q_t row `dst` (rows r .. r + 15 of x), a 16-byte
// store where alignment and the row count allow.
__device__ __forceinline__ void store16(uint8_t* dst, const float (&y)[16], long long r, long long R, bool vec_q) {
  uint4 codes;
  codes.x = e4m3x2(y[0], y[1]) | (e4m3x2(y[2], y[3]) << 16);
  codes.y = e4m3x2(y[4], y[5]) | (e4m3x2(y[6], y[7]) << 16);
  codes.z = e4m3x2(y[8], y[9]) | (e4m3x2(y[10], y[11]) << 16);
  codes.w = e4m3x2(y[12], y[13]) | (e4m3x2(y[14], y[15]) << 16);
  if (vec_q && r + 16 <= R) {
    *reinterpret_cast<uint4*>(dst) = codes;
  } else {
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (r + j < R) dst[j] = static_cast<uint8_t>(w[j / 4] >> (8 * (j % 4)));
  }
}

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
  const int cp = t % (kTile / 2);  // this thread's column pair in the compute phase
  const int qr = t / (kTile / 2);  // and its quarter of the rows
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
    // the amaxes of this thread's two columns, down its quarter of the rows
    const int rq = kRowsPerThread * qr;
    float amax0 = 0.f, amax1 = 0.f;
#pragma unroll 8
    for (int i = 0; i < kRowsPerThread; ++i) {
      float a, b;
      pair_at(sm, rq + i, cp, a, b);
      amax0 = fmaxf(amax0, fabsf(a));
      amax1 = fmaxf(amax1, fabsf(b));
    }
    if constexpr (GROUP == 0) {
      sm.part[qr][2 * cp] = amax0;
      sm.part[qr][2 * cp + 1] = amax1;
      __syncthreads();
#pragma unroll
      for (int k = 1; k < kQuarters; ++k) {
        amax0 = fmaxf(amax0, sm.part[(qr + k) % kQuarters][2 * cp]);
        amax1 = fmaxf(amax1, sm.part[(qr + k) % kQuarters][2 * cp + 1]);
      }
    } else {
      float amax = fmaxf(amax0, amax1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if ((t & 31) == 0) sm.wmax[t / 32] = amax;
      __syncthreads();
      amax = sm.wmax[0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, sm.wmax[w]);
      amax0 = amax1 = amax;
    }
    const long long ca = c0 + 2 * cp, cbn = ca + 1;  // this thread's two columns of x
    float s0 = 1.f, s1 = 1.f;
    int byte0 = 127, byte1 = 127;
    if constexpr (FMT == 0) {
      s0 = group_scale_f32(amax0);
      s1 = group_scale_f32(amax1);
    } else {
      byte0 = group_e8m0(amax0);
      byte1 = group_e8m0(amax1);
    }
    const float mul0 = ldexpf(1.f, 127 - byte0), mul1 = ldexpf(1.f, 127 - byte1);  // exact powers of two
    if constexpr (GROUP == 0) {
      if (qr == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const long long c = ca + h;
          if (c >= C) continue;
          if constexpr (FMT == 0) {
            static_cast<float*>(scale)[c * lds + rb] = h ? s1 : s0;
          } else {
            static_cast<uint8_t*>(scale)[c * lds + rb] = static_cast<uint8_t>(h ? byte1 : byte0);
          }
        }
      }
    } else if (t == 0) {
      if constexpr (FMT == 0) {
        static_cast<float*>(scale)[rb * lds + cb] = s0;
      } else {
        static_cast<uint8_t*>(scale)[rb * lds + cb] = static_cast<uint8_t>(byte0);
      }
    }
    if (ca >= C) continue;  // both columns past the matrix: nothing to store
#pragma unroll
    for (int k = 0; k < kRowsPerThread / 16; ++k) {
      const long long r = r0 + rq + 16 * k;
      float e0[16], e1[16], y[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) pair_at(sm, rq + 16 * k + j, cp, e0[j], e1[j]);
      if constexpr (FMT == 0) {
        code_quotients<16>(e0, s0, y);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) y[j] = e0[j] * mul0;
      }
      store16(q + ca * ldq + r, y, r, R, vec_q);
      if (cbn < C) {
        if constexpr (FMT == 0) {
          code_quotients<16>(e1, s1, y);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = e1[j] * mul1;
        }
        store16(q + cbn * ldq + r, y, r, R, vec_q);
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
  int per_sm = 1;  // resident CTAs per SM (shared memory and registers): one wave, no stragglers
  const cudaError_t e = ctas_per_sm_once<quantize_t_kernel<InT, FMT, GROUP>>(kThreads, smem, &per_sm);
  if (e != cudaSuccess) return e;
  long long blocks = static_cast<long long>(sms > 0 ? sms : 148) * per_sm;
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

// ---------------------------------------------------------------------------
// TMA-fed form (x and q_t with 16-byte bases and row strides, rows ending on
// 16-byte boundaries)
// ---------------------------------------------------------------------------
// Persistent CTAs (two of 256 threads per SM for bf16 input, each with two
// input and two code tiles, so that one CTA's reductions and barriers overlap
// the other's work; one of 512 threads for fp32, with three input tiles and one
// code tile).  One thread keeps the ring of input tiles in flight with 2-D
// tensor copies and writes the code tiles back with tensor stores (TileRing,
// tile_ring.cuh), so no thread spends instructions or registers on loads.
// Thread t owns the column
// pair 2 (t % 64), + 1 and kRows consecutive rows (32 for bf16, 16 for fp32):
// it reads its pairs from the tile once (one 4- or 8-byte shared load each, a
// warp reading 128 or 256 contiguous bytes), takes their amax in registers
// (bf16: one packed max of magnitudes per pair), and after the amaxes meet in
// shared memory quantises the values it still holds, 16 rows at a time.  Each
// run of 16 codes of a column goes as one 16-byte piece into a shared
// [column][row] code tile laid out in the 128-byte swizzle, which one thread
// then writes to q_t with a tensor store that clips at R and C.
template <typename InT>
struct TRing {
  static constexpr bool kPair = sizeof(InT) == 2;
  static constexpr int kThreads = kPair ? 256 : 512;
  static constexpr int kCtasPerSm = kPair ? 2 : 1;
  static constexpr int kStages = kPair ? 2 : 3;    // input tiles (32 or 64 KB each)
  static constexpr int kCodeBufs = kPair ? 2 : 1;  // code tiles (16 KB each)
  static constexpr int kParts = kThreads / (kTile / 2);  // row groups per column pair
  static constexpr int kRows = kTile / kParts;           // rows per thread
  static constexpr int kRuns = kRows / 16;               // 16-row runs: one 16-byte code piece per column each
  using Held = typename std::conditional<kPair, uint32_t, float2>::type;  // one row of the column pair
};

template <typename InT>
struct TmaSmem {
  alignas(1024) InT v[TRing<InT>::kStages][kTile][kTile];          // input tiles, [row][column]
  alignas(1024) uint8_t codes[TRing<InT>::kCodeBufs][kTile][kTile];  // [column][row], 128-byte swizzle
  float2 part[TRing<InT>::kParts][kTile / 2];  // amaxes of each row group's column pairs
  float wmax[TRing<InT>::kThreads / 32];
  uint64_t full[TRing<InT>::kStages];
  int abort;
};

// One held row of a column pair as fp32 (exact widening for bf16).
__device__ __forceinline__ float2 widen(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float2 widen(float2 v) { return v; }

// 16 codes of one column (lane h of y) as a 16-byte piece.
__device__ __forceinline__ uint4 pack_column(const float2 (&y)[16], int h) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float a = h ? y[4 * j].y : y[4 * j].x, b = h ? y[4 * j + 1].y : y[4 * j + 1].x;
    const float c = h ? y[4 * j + 2].y : y[4 * j + 2].x, d = h ? y[4 * j + 3].y : y[4 * j + 3].x;
    w[j] = e4m3x2(a, b) | (e4m3x2(c, d) << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename InT, int FMT, int GROUP>
__global__ void __launch_bounds__(TRing<InT>::kThreads, TRing<InT>::kCtasPerSm)
    quantize_t_tma_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmq, long long R,
                          long long C, void* __restrict__ scale, long long lds, long long ctiles, long long ntiles,
                          uint32_t* err) {
  using G = TRing<InT>;
  using S = TmaSmem<InT>;
  using Held = typename G::Held;
  constexpr uint32_t kTileBytes = kTile * kTile * sizeof(InT);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + sizeof(S) > dynamic_smem_bytes()) {  // never touch memory the launch did not provide
    if (threadIdx.x == 0) record_error(err, kErrSmemTooSmall);
    return;
  }
  S& sm = *reinterpret_cast<S*>(smem_raw + pad);
  const int t = threadIdx.x;
  const int cp = t % (kTile / 2);  // column pair
  const int qr = t / (kTile / 2);  // row group: rows kRows * qr ..
  const TileRing<G::kStages, G::kCodeBufs> ring{sm.full, &sm.abort, &tmx, reinterpret_cast<uint8_t*>(&sm.v[0][0][0]),
                                                kTileBytes, ctiles, ntiles};
  if (t == 0) {
    ring.init(&tmq);
    ring.start();
  }
  int it = 0;
  bool ok = true;
  __syncthreads();  // the mbarriers are initialised
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int st = it % G::kStages, cbuf = it % G::kCodeBufs;
    const long long rb = tile / ctiles, cb = tile - rb * ctiles;
    const bool got = ring.wait(it, err);
    Held h[G::kRows];
#pragma unroll
    for (int i = 0; i < G::kRows; ++i) h[i] = *reinterpret_cast<const Held*>(&sm.v[st][G::kRows * qr + i][2 * cp]);
    float amax0, amax1;
    if constexpr (G::kPair) {
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < G::kRows; ++i) m = max_abs_bf16x2(m, h[i]);
      amax0 = __uint_as_float((m << 16) & 0x7FFFFFFFu);
      amax1 = __uint_as_float(m & 0x7FFF0000u);
    } else {
      amax0 = amax1 = 0.f;
#pragma unroll
      for (int i = 0; i < G::kRows; ++i) {
        amax0 = fmaxf(amax0, fabsf(widen(h[i]).x));
        amax1 = fmaxf(amax1, fabsf(widen(h[i]).y));
      }
    }
    if constexpr (GROUP == 0) {
      sm.part[qr][cp] = make_float2(amax0, amax1);
    } else {
      float a = fmaxf(amax0, amax1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      if ((t & 31) == 0) sm.wmax[t / 32] = a;
    }
    if (t == 0) ring.code_tile_free();
    // every thread holds its values: the stage can be refilled
    ok = __syncthreads_and(got) != 0;
    if (!ok) break;
    if (t == 0) ring.refill(tile, it);
    if constexpr (GROUP == 0) {
#pragma unroll
      for (int k = 0; k < G::kParts; ++k) {
        const float2 pk = sm.part[k][cp];
        amax0 = fmaxf(amax0, pk.x);
        amax1 = fmaxf(amax1, pk.y);
      }
    } else {
      float a = sm.wmax[0];
#pragma unroll
      for (int w = 1; w < G::kThreads / 32; ++w) a = fmaxf(a, sm.wmax[w]);
      amax0 = amax1 = a;
    }
    const long long ca = cb * kTile + 2 * cp;  // this thread's first column of x
    float2 sc = make_float2(1.f, 1.f), rc = sc, mul = sc;
    bool fast = true;
    if constexpr (FMT == 0) {
      sc = make_float2(group_scale_f32(amax0), group_scale_f32(amax1));
      if constexpr (GROUP == 0) {
        if (qr == 0) {
          if (ca < C) static_cast<float*>(scale)[ca * lds + rb] = sc.x;
          if (ca + 1 < C) static_cast<float*>(scale)[(ca + 1) * lds + rb] = sc.y;
        }
      } else if (t == 0) {
        static_cast<float*>(scale)[rb * lds + cb] = sc.x;
      }
      fast = __all_sync(0xffffffffu, quotient_fast_range(sc.x) && quotient_fast_range(sc.y));
      rc = make_float2(__frcp_rn(sc.x), __frcp_rn(sc.y));
    } else {
      const int byte0 = group_e8m0(amax0), byte1 = group_e8m0(amax1);
      if constexpr (GROUP == 0) {
        if (qr == 0) {
          if (ca < C) static_cast<uint8_t*>(scale)[ca * lds + rb] = static_cast<uint8_t>(byte0);
          if (ca + 1 < C) static_cast<uint8_t*>(scale)[(ca + 1) * lds + rb] = static_cast<uint8_t>(byte1);
        }
      } else if (t == 0) {
        static_cast<uint8_t*>(scale)[rb * lds + cb] = static_cast<uint8_t>(byte0);
      }
      mul = make_float2(ldexpf(1.f, 127 - byte0), ldexpf(1.f, 127 - byte1));  // exact powers of two
    }
#pragma unroll
    for (int run = 0; run < G::kRuns; ++run) {
      float2 e[16], y[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) e[i] = widen(h[16 * run + i]);
      if constexpr (FMT == 0) {
        code_quotients2<16>(e, sc, rc, fast, y);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __fmul2_rn(e[i], mul);
      }
      // code tile rows 2 cp and 2 cp + 1, 16-byte piece kRuns qr + run (swizzled by the row)
      const int piece = G::kRuns * qr + run;
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int c = 2 * cp + hc;
        *reinterpret_cast<uint4*>(&sm.codes[cbuf][c][(piece ^ (c & 7)) * 16]) = pack_column(y, hc);
      }
    }
    fence_proxy_async_smem();  // the code tile, before the tensor store reads it
    __syncthreads();
    if (t == 0) ring.store(&tmq, &sm.codes[cbuf][0][0], rb * kTile, cb * kTile);
  }
  if (t == 0) ring.finish(ok, it);
}

template <typename InT, int FMT, int GROUP>
cudaError_t launch_t_tma(const CUtensorMap& tmx, const CUtensorMap& tmq, long long R, long long C, void* scale,
                         long long lds, int sms, uint32_t* err, cudaStream_t stream) {
  const long long ctiles = (C + kTile - 1) / kTile;
  const long long ntiles = ((R + kTile - 1) / kTile) * ctiles;
  const size_t smem = sizeof(TmaSmem<InT>) + 1024;
  int per_sm = 1;
  const cudaError_t e = ctas_per_sm_once<quantize_t_tma_kernel<InT, FMT, GROUP>>(TRing<InT>::kThreads, smem, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm > TRing<InT>::kCtasPerSm) per_sm = TRing<InT>::kCtasPerSm;
  long long blocks = static_cast<long long>(sms > 0 ? sms : 148) * per_sm;
  if (blocks > ntiles) blocks = ntiles;
  quantize_t_tma_kernel<InT, FMT, GROUP><<<static_cast<unsigned>(blocks), TRing<InT>::kThreads, smem, stream>>>(
      tmx, tmq, R, C, scale, lds, ctiles, ntiles, err);
  return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_t_tma_fmt(const CUtensorMap& tmx, const CUtensorMap& tmq, long long R, long long C, void* scale,
                             bool e8m0, bool block, long long lds, int sms, uint32_t* err, cudaStream_t stream) {
  if (block)
    return e8m0 ? launch_t_tma<InT, 1, 1>(tmx, tmq, R, C, scale, lds, sms, err, stream)
                : launch_t_tma<InT, 0, 1>(tmx, tmq, R, C, scale, lds, sms, err, stream);
  return e8m0 ? launch_t_tma<InT, 1, 0>(tmx, tmq, R, C, scale, lds, sms, err, stream)
              : launch_t_tma<InT, 0, 0>(tmx, tmq, R, C, scale, lds, sms, err, stream);
}

}  // namespace

cudaError_t launch_quantize_t(const void* x, bool x_bf16, long long R, long long C, long long ldx, uint8_t* q_t,
                              long long ldq, void* scale, bool e8m0, bool block128, long long lds, int sms,
                              const CUtensorMap* tmx, const CUtensorMap* tmq, uint32_t* err, cudaStream_t stream) {
  if (tmx && tmq)
    return x_bf16 ? launch_t_tma_fmt<__nv_bfloat16>(*tmx, *tmq, R, C, scale, e8m0, block128, lds, sms, err, stream)
                  : launch_t_tma_fmt<float>(*tmx, *tmq, R, C, scale, e8m0, block128, lds, sms, err, stream);
  return x_bf16 ? launch_t_fmt<__nv_bfloat16>(x, R, C, ldx, q_t, ldq, scale, e8m0, block128, lds, sms, stream)
                : launch_t_fmt<float>(x, R, C, ldx, q_t, ldq, scale, e8m0, block128, lds, sms, stream);
}

}  // namespace bsg

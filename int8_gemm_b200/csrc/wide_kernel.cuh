// Persistent, warp-specialised scaled-GEMM kernel for sm_100a ("wide" path:
// M large enough to fill 128-row tiles).
//
// One CTA per SM walks output tiles of 128 x BN.  Roles inside the CTA:
//   warp 0      TMA producer: A[128 x 128 B] and B[BN x 128 B] K-block tiles
//               into a STAGES-deep shared-memory ring (full/empty mbarriers).
//   warp 1      MMA issuer: four tcgen05.mma (K = 32 bytes each) per K block
//               into a TMEM accumulator; owns the TMEM allocation.
//   warps 2, 3  idle (they complete warpgroup 0 for the register split).
//   warps 4..11 consumers (warpgroups 1 and 2).  Warp w reads TMEM lanes
//               32*(w%4).. and one half (128 columns) of the tile.
// Launched with 384 threads x 168 registers; warpgroup 0 gives registers back
// (40 each) so the consumer warpgroups can hold 128 fp32 accumulators plus a
// 32-column TMEM slice (232 each): 128*40 + 256*232 = 384*168.
//
// FP8 modes (block scales vary along K):  every 128-deep K block lands in one
// of two TMEM buffers; the consumers pull the partial P_kb into registers and
// add s(m, kb, n) * P_kb to an fp32 register accumulator, then release the
// buffer, so the MMA of block kb+1 overlaps the promotion of block kb.  The
// scale s = scale_a[m, kb] * scale_b[kb, n/128] is one number per thread per
// block because each consumer's 128 columns form one 128-wide scale block.
//   Sources: pytorch issue "torch._scaled_mm with blockwise scaling doesn't
//   work with torch.compile" (1x128 / 128x128 scale shapes); ROCm/aiter PR
//   "Add opus fp8 mxscale BMM kernels for gfx950" (m-major batched layout,
//   e8m0 scales [M, G, K/128] and [G, N/128, K/128]).
// INT8 mode: s8 x s8 -> s32 accumulates over all of K in TMEM (double-buffered
// across tiles); the epilogue computes (float(acc) * s_a[m]) * s_b[n] with two
// round-to-nearest fp32 multiplies.
//   Sources: pytorch/ao PR "Remove int_scaled_mm's dependency on triton for
//   cpu" (int_scaled_matmul_cpu); pytorch/ao issue "Unify scaled INT8 matmul"
//   (cast acc_i32 to f32, then multiply by the fp32 scales).
// Epilogue: registers -> 128B-swizzled shared staging (4 KB per consumer warp)
// -> TMA store, which clips rows >= M and columns >= N (the masked store of
// mm_template in pytorch/torch/_inductor/kernel/mm.py).  Rows >= M of A are
// zero-filled by the TMA loads, so ragged M needs no padding copies.
#pragma once

#include <type_traits>

#include "sm100.cuh"
#include "tile_order.h"

namespace bsg {

enum class Mode : int { kFp8F32Scale = 0, kFp8E8M0 = 1, kInt8 = 2 };

struct GemmArgs {
  int M, N, K, G;
  int KB;  // number of 128-deep K blocks
  int NB;  // number of 128-wide scale blocks along N
  int grid_m, grid_n, num_tiles, group_m;
  int splits;  // split-K factor (skinny kernel only)
  // FP8, fp32 scales: scale_a[m * sa_sm + kb * sa_sk], scale_b[kb * sb_sk + nb * sb_sn]
  const float* sa;
  long long sa_sm, sa_sk;
  const float* sb;
  long long sb_sk, sb_sn;
  // FP8, e8m0 scales: xs[(m * G + g) * KB + kb], ws[(g * NB + nb) * KB + kb]
  const uint8_t* xs;
  const uint8_t* ws;
  // INT8 per-row / per-column scales, either may be null
  const float* s_row;
  const float* s_col;
  uint32_t* err;
};

template <int BN, int STAGES>
struct WideSmem {
  uint8_t a[STAGES][128 * 128];
  uint8_t b[STAGES][BN * 128];
  uint8_t stage_out[8][32 * 128];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Block scale for row m, K block kb, scale block nb along N; 0 outside the
// problem (the matching partials are zero-filled anyway).
template <Mode MODE>
__device__ __forceinline__ float block_scale(const GemmArgs& p, int g, int m, int kb, int nb) {
  if (m >= p.M || nb >= p.NB) return 0.f;
  if constexpr (MODE == Mode::kFp8F32Scale) {
    const float a = __ldg(p.sa + static_cast<long long>(m) * p.sa_sm + static_cast<long long>(kb) * p.sa_sk);
    const float b = __ldg(p.sb + static_cast<long long>(kb) * p.sb_sk + static_cast<long long>(nb) * p.sb_sn);
    return a * b;
  } else {
    const uint32_t ea = __ldg(p.xs + (static_cast<long long>(m) * p.G + g) * p.KB + kb);
    const uint32_t eb = __ldg(p.ws + (static_cast<long long>(g) * p.NB + nb) * p.KB + kb);
    return e8m0_to_f32(ea) * e8m0_to_f32(eb);
  }
}

// Write 32 output values of this lane's row into the 128B-swizzled staging
// row (row = lane, 16-byte unit u stored at u ^ (lane & 7)).
template <typename OutT>
__device__ __forceinline__ void stage_32(uint8_t* stg, int lane, int unit0, const float (&v)[32]) {
  uint8_t* row = stg + lane * 128;
  if constexpr (sizeof(OutT) == 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(v[q * 8 + 0], v[q * 8 + 1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(v[q * 8 + 2], v[q * 8 + 3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[q * 8 + 4], v[q * 8 + 5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(v[q * 8 + 6], v[q * 8 + 7]);
      w.x = *reinterpret_cast<uint32_t*>(&h0);
      w.y = *reinterpret_cast<uint32_t*>(&h1);
      w.z = *reinterpret_cast<uint32_t*>(&h2);
      w.w = *reinterpret_cast<uint32_t*>(&h3);
      *reinterpret_cast<uint4*>(row + (((unit0 + q) ^ (lane & 7)) << 4)) = w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint4 w = make_uint4(__float_as_uint(v[q * 4 + 0]), __float_as_uint(v[q * 4 + 1]),
                           __float_as_uint(v[q * 4 + 2]), __float_as_uint(v[q * 4 + 3]));
      *reinterpret_cast<uint4*>(row + (((unit0 + q) ^ (lane & 7)) << 4)) = w;
    }
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* err,
                                          uint32_t code) {
  const bool ok = wait_bounded(bar, parity, abort, err, code);
  return __all_sync(0xffffffffu, ok);
}

constexpr int kWideProducerRegs = 40;
constexpr int kWideConsumerRegs = 232;
static_assert(128 * kWideProducerRegs + 256 * kWideConsumerRegs <= 384 * 168, "register split exceeds launch budget");

template <Mode MODE, int BN, int STAGES, typename OutT>
__global__ void __launch_bounds__(384, 1)
    wide_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const GemmArgs p) {
  constexpr int BM = 128, BK = 128;
  constexpr uint32_t A_BYTES = BM * BK, B_BYTES = BN * BK;
  constexpr int CONSUMER_WARPS = 8;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr bool IS_INT8 = MODE == Mode::kInt8;
  constexpr uint32_t IDESC = IS_INT8 ? idesc_s8_s32<BM, BN>() : idesc_e4m3_f32<BM, BN>();
  constexpr int CPC = 128 / sizeof(OutT);  // output columns per 128-byte staging row
  static_assert(BN == 256, "consumer layout assumes two 128-column halves");
  using Smem = WideSmem<BN, STAGES>;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + pad);
  volatile int* abort = &sm.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], CONSUMER_WARPS);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
    regs_dec<kWideProducerRegs>();
    if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      uint32_t issued = 0, issued_phase = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, p.grid_m, p.grid_n, p.group_m);
        const int m0 = tc.pm * BM, n0 = tc.pn * BN;
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!wait_bounded(&sm.empty[stage], phase ^ 1u, abort, p.err,
                            kErrTimeout | kRoleProducer | kWaitStageEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[stage], A_BYTES + B_BYTES);
          tma_load_3d(sm.a[stage], &tmA, &sm.full[stage], kb * BK, m0, tc.g);
          tma_load_3d(sm.b[stage], &tmB, &sm.full[stage], kb * BK, n0, tc.g);
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let copies already in flight land before the CTA retires
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) wait_bounded(&sm.full[s], (issued_phase >> s) & 1u, &never, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        if constexpr (IS_INT8) {
          if (!wait_bounded(&sm.acc_empty[buf], bphase ^ 1u, abort, p.err, kErrTimeout | kRoleMma | kWaitAccEmpty)) {
            ok = false;
            break;
          }
        }
        for (int kb = 0; kb < p.KB; ++kb) {
          if constexpr (!IS_INT8) {
            if (!wait_bounded(&sm.acc_empty[buf], bphase ^ 1u, abort, p.err,
                              kErrTimeout | kRoleMma | kWaitAccEmpty)) {
              ok = false;
              break;
            }
          }
          if (!wait_bounded(&sm.full[stage], phase, abort, p.err, kErrTimeout | kRoleMma | kWaitStageFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
          const uint64_t ad = sdesc_k_sw128(smem_u32(sm.a[stage]));
          const uint64_t bd = sdesc_k_sw128(smem_u32(sm.b[stage]));
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            if constexpr (IS_INT8) {
              mma_i8(d, ad + 2 * k, bd + 2 * k, IDESC, (kb > 0 || k > 0) ? 1u : 0u);
            } else {
              mma_f8f6f4(d, ad + 2 * k, bd + 2 * k, IDESC, k > 0 ? 1u : 0u);
            }
          }
          mma_commit(&sm.empty[stage]);
          if constexpr (!IS_INT8) {
            mma_commit(&sm.acc_full[buf]);
            buf ^= 1;
            if (buf == 0) bphase ^= 1u;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if constexpr (IS_INT8) {
          if (ok) {
            mma_commit(&sm.acc_full[buf]);
            buf ^= 1;
            if (buf == 0) bphase ^= 1u;
          }
        }
      }
      if (!ok) {  // wait until every MMA already issued has finished with TMEM and smem
        mma_commit(&sm.drain);
        volatile int never = 0;
        wait_bounded(&sm.drain, 0, &never, nullptr, 0);
      }
    }
    __syncwarp();
    }
  } else {
    regs_inc<kWideConsumerRegs>();
    // ------------------------------------------------------------ consumers
    const int cw = warp - 4;
    const int lg = warp & 3;
    const int half = cw >> 2;
    const uint32_t t_lane = static_cast<uint32_t>(lg * 32) << 16;
    const int row = lg * 32 + lane;
    uint8_t* stg = sm.stage_out[cw];
    int buf = 0;
    uint32_t bphase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, p.grid_m, p.grid_n, p.group_m);
      const int m0 = tc.pm * BM, n0 = tc.pn * BN;
      const int m = m0 + row;
      const int ncol0 = n0 + half * 128;
      bool ok = true;
      if constexpr (!IS_INT8) {
        const int nb = ncol0 >> 7;
        float acc[128];
#pragma unroll
        for (int j = 0; j < 128; ++j) acc[j] = 0.f;
        float s_cur = block_scale<MODE>(p, tc.g, m, 0, nb);
        for (int kb = 0; kb < p.KB; ++kb) {
          const float s_next = (kb + 1 < p.KB) ? block_scale<MODE>(p, tc.g, m, kb + 1, nb) : 0.f;
          if (!warp_wait(&sm.acc_full[buf], bphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitAccFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tb = tmem + t_lane + static_cast<uint32_t>(buf * BN + half * 128);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tb + c * 32, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[c * 32 + j] = fmaf(s_cur, __uint_as_float(r[j]), acc[c * 32 + j]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
          buf ^= 1;
          if (buf == 0) bphase ^= 1u;
          s_cur = s_next;
        }
        if (!ok) break;
#pragma unroll
        for (int ch = 0; ch < 128 / CPC; ++ch) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int sub = 0; sub < CPC / 32; ++sub) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = acc[ch * CPC + sub * 32 + j];
            stage_32<OutT>(stg, lane, sub * (32 * static_cast<int>(sizeof(OutT)) / 16), v);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && m0 + lg * 32 < p.M && ncol0 + ch * CPC < p.N) {  // skip boxes wholly outside
            tma_store_3d(&tmD, stg, ncol0 + ch * CPC, m0 + lg * 32, tc.g);
            bulk_commit();
          }
        }
      } else {
        if (!warp_wait(&sm.acc_full[buf], bphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitAccFull)) break;
        tc_fence_after();
        const bool has_row = p.s_row != nullptr, has_col = p.s_col != nullptr;
        const float sr = (has_row && m < p.M) ? __ldg(p.s_row + m) : 1.f;
        const uint32_t tb = tmem + t_lane + static_cast<uint32_t>(buf * BN + half * 128);
#pragma unroll
        for (int ch = 0; ch < 128 / CPC; ++ch) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int sub = 0; sub < CPC / 32; ++sub) {
            const int c0 = ch * CPC + sub * 32;
            uint32_t r[32];
            tmem_ld32(tb + c0, r);
            float v[32];
            if constexpr (sizeof(OutT) == 4 && !std::is_same<OutT, float>::value) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);  // raw int32 accumulator
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                float f = __int2float_rn(static_cast<int>(r[j]));
                if (has_row) f = __fmul_rn(f, sr);
                if (has_col) {
                  const int n = ncol0 + c0 + j;
                  const float sc = n < p.N ? __ldg(p.s_col + n) : 0.f;
                  f = __fmul_rn(f, sc);
                }
                v[j] = f;
              }
            }
            stage_32<OutT>(stg, lane, sub * (32 * static_cast<int>(sizeof(OutT)) / 16), v);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && m0 + lg * 32 < p.M && ncol0 + ch * CPC < p.N) {  // skip boxes wholly outside
            tma_store_3d(&tmD, stg, ncol0 + ch * CPC, m0 + lg * 32, tc.g);
            bulk_commit();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
        buf ^= 1;
        if (buf == 0) bphase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace bsg

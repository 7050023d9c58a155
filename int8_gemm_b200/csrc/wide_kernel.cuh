// Persistent, warp-specialised scaled-GEMM kernel for sm_100a ("wide" path:
// M large enough to fill 128-row tiles).
//
// One CTA per SM walks output tiles of 128 x BN.  Roles inside the CTA:
//   warp 0      TMA producer: A[128 x 128 B] and B[BN x 128 B] K-block tiles
//               into a STAGES-deep shared-memory ring (full/empty mbarriers).
//   warp 1      MMA issuer: four tcgen05.mma (K = 32 bytes each) per K block
//               into a TMEM accumulator; owns the TMEM allocation.
//   warps 2, 3  FP8 modes: scale producer (stages the block scales of the
//               next K blocks in a shared ring; for kFp8Mx, the e8m0 scale
//               factors the tensor core reads); idle for INT8 and rowwise.
//   warps 4..11 consumers (warpgroups 1 and 2).  Warp w reads TMEM lanes
//               32*(w%4).. and one half (128 columns) of the tile.
// Launched with 384 threads x 168 registers; warpgroup 0 keeps 56 each and the
// consumer warpgroups take 224 each (128 fp32 accumulators plus two 32-column
// TMEM slices in flight): 128*56 + 256*224 = 384*168.
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
// kFp8Mx (the batched operation on CTA pairs): the e8m0 scales are powers of
// two, so the tensor core applies them itself -- per K block the MMA thread
// copies the scale factors of the pair's 256 rows and 256 columns from
// shared memory into TMEM (tcgen05.cp) and issues block-scaled MMAs that
// accumulate over all of K.  To leave room for the scale factors the two
// accumulator buffers overlap in 32 columns: the epilogue reads those first
// and releases them early, so it still overlaps the next tile's MMAs.  The
// power-of-two scales make every product exact, so this sums the same terms
// as the per-block promotion, in a different order.
// INT8 mode: s8 x s8 -> s32 accumulates over all of K in TMEM (double-buffered
// across tiles); the epilogue computes (float(acc) * s_a[m]) * s_b[n] with two
// round-to-nearest fp32 multiplies.
//   Sources: pytorch/ao PR "Remove int_scaled_mm's dependency on triton for
//   cpu" (int_scaled_matmul_cpu); pytorch/ao issue "Unify scaled INT8 matmul"
//   (cast acc_i32 to f32, then multiply by the fp32 scales).
// Epilogue: registers -> 64B-swizzled shared staging (2 KB per consumer warp,
// two such buffers for INT8 on CTA pairs)
// -> TMA store, which clips rows >= M and columns >= N (the masked store of
// mm_template in pytorch/torch/_inductor/kernel/mm.py).  Rows >= M of A are
// zero-filled by the TMA loads, so ragged M needs no padding copies.
#pragma once

#include <cuda_fp8.h>

#include <type_traits>

#include "sm100.cuh"
#include "tile_order.h"

namespace bsg {

// kFp8Rowwise: e4m3 with one scale per row of A and per column of B (or one
// per operand), constant along K, so the accumulator stays in TMEM for all of
// K as in the INT8 mode.
// kFp8Mx: the batched operation's e8m0 (power-of-two) block scales applied by
// the tensor core itself (tcgen05.mma kind::mxf8f6f4 with block scaling, one
// scale per 32 K elements, each 128-deep block's scale repeated four times),
// so the accumulator also stays in TMEM for all of K.  CTA pairs only.
enum class Mode : int { kFp8F32Scale = 0, kFp8E8M0 = 1, kInt8 = 2, kFp8Rowwise = 3, kFp8Mx = 4 };

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
  // INT8 and FP8-rowwise per-row / per-column scales.  INT8 reads s_row[m]
  // and s_col[n] and allows either to be null.  FP8 rowwise reads s_row[m]
  // when s_row_stride is 1 and s_row[0] when it is 0 (tensorwise), likewise
  // for s_col; the strides are 0 or 1 and are applied as a select.  bias:
  // fp32 [N] or null (FP8 rowwise).  s_result: fp32 scalar or null, the
  // factor an e4m3 output of FP8 rowwise takes before its cast.
  const float* s_row;
  const float* s_col;
  long long s_row_stride, s_col_stride;
  const float* bias;
  const float* s_result;
  uint32_t* err;
  // Stream-K split of the wide kernel (tile_order.h): tiles [0, dp_tiles)
  // whole, the sk_iters K blocks of the others cut evenly over the units
  // (sk_iters == 0: no split).  sk_ws: one partial-sum slot per unit and
  // CTA (kWsSlotWords words); sk_flags: one word per slot and consumer warp,
  // zero between launches.
  int dp_tiles;
  long long sk_iters;
  uint32_t* sk_ws;
  uint32_t* sk_flags;
};

// A stream-K partial-sum slot: the 128 x 256 accumulator of one CTA, laid out
// per consumer warp as [column / 4][lane][column % 4] (16-byte pieces, so a
// warp's stores and loads of four columns cover 512 contiguous bytes).
constexpr int kWsSlotWords = 8 * 128 * 32;
constexpr int kWsFlagsPerSlot = 8;

// Shared-memory layout of one CTA.  In the pair (cta_group::2) variant both
// CTAs use the same layout: the leader's MMA descriptors address the same
// offsets in the peer.
constexpr int kScaleRing = 16;  // K blocks of scales staged ahead of the consumers
constexpr int kScaleBatch = 8;  // K blocks whose scale loads are in flight together
constexpr int kSfRing = 5;      // kFp8Mx: scale-factor slots (four K blocks each) staged ahead of the MMA
// kFp8Mx TMEM columns: accumulator buffer 1 starts at kAcc1Col, so the two
// 256-column buffers share 32 columns and the scale factors fit behind them.
constexpr uint32_t kAcc1Col = 224, kSfaCol = 480, kSfbCol = 484;

// Output staging buffers per consumer warp: two for INT8 on CTA pairs (a
// chunk is staged while the previous chunk's TMA store still reads the
// other), with one operand stage fewer to make room.  Its epilogue has to
// hide behind the next tile's MMAs, and its fp32 and int32 outputs take eight
// chunks per warp; measured on 4096^3 with fp32 out, 62.3 -> 60.0 us.  The
// FP8 modes keep one buffer and the deeper ring (rowwise and the block-scaled
// MMA measured about 1 % slower with two), and so do single-CTA tiles, whose
// 48 KB stages leave no room for a second buffer.
template <Mode MODE, int CG>
__host__ __device__ constexpr int wide_stage_bufs() {
  return CG == 2 && MODE == Mode::kInt8 ? 2 : 1;
}
template <Mode MODE, int CG>
__host__ __device__ constexpr int wide_stages() {
  return CG == 2 ? (wide_stage_bufs<MODE, CG>() == 2 ? 5 : 6) : 4;
}

template <int BNL, int STAGES, int SBUFS>
struct WideSmem {
  static constexpr int kStageBufs = SBUFS;
  uint8_t a[STAGES][128 * 128];  // this CTA's 128 A rows of one K block
  uint8_t b[STAGES][BNL * 128];  // this CTA's BNL B rows (output columns) of one K block
  uint8_t stage_out[kStageBufs][8][32 * 64];  // per consumer warp: 32 rows x 64 bytes, 64-byte swizzle
  union {
    float sa[kScaleRing][128];  // scale_a of this CTA's rows, per K block
    // kFp8Mx, per four K blocks: three 512-byte scale-factor chunks (this
    // CTA's 128 rows of A; B columns 0-127; B columns 128-255), each 32 lanes
    // x 16 bytes as tcgen05.cp reads them: item i in the 32-bit word at byte
    // 16*(i%32) + 4*(i/32), byte j of that word for the slot's K block j (the
    // MMAs of K block kb select byte kb % 4 through the scale-factor ids)
    alignas(16) uint8_t sf[kSfRing][3][512];
  };
  float sb[kScaleRing][4];       // scale_b of the tile's two 128-column blocks, per K block
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];   // INT8: tile accumulator complete (FP8 uses the stage barriers)
  uint64_t acc_empty[2];  // accumulator buffer released by every consumer warp (of both CTAs)
  uint64_t ovl_empty[2];  // kFp8Mx: the buffer's 32 shared columns read by the warps holding them
  uint64_t sc_full[kScaleRing];
  uint64_t sc_empty[kScaleRing];
  uint64_t drain;
  uint64_t part_bar[8];  // consumer warps: a stream-K partial copied into the idle operand ring
  uint32_t tmem_base;
  int abort;
  long long sk_pos[8];  // consumer warps: position in the stream-K range (kept out of registers)
};

// Row and column-block factors of the block scale (0 outside the problem; the
// matching partials are zero-filled anyway).
template <Mode MODE>
__device__ __forceinline__ float scale_row(const GemmArgs& p, int g, int m, int kb) {
  if (m >= p.M) return 0.f;
  if constexpr (MODE == Mode::kFp8F32Scale) {
    return __ldg(p.sa + static_cast<long long>(m) * p.sa_sm + static_cast<long long>(kb) * p.sa_sk);
  } else {
    return e8m0_to_f32(__ldg(p.xs + (static_cast<long long>(m) * p.G + g) * p.KB + kb));
  }
}
template <Mode MODE>
__device__ __forceinline__ float scale_col(const GemmArgs& p, int g, int kb, int nb) {
  if (nb >= p.NB) return 0.f;
  if constexpr (MODE == Mode::kFp8F32Scale) {
    return __ldg(p.sb + static_cast<long long>(kb) * p.sb_sk + static_cast<long long>(nb) * p.sb_sn);
  } else {
    return e8m0_to_f32(__ldg(p.ws + (static_cast<long long>(g) * p.NB + nb) * p.KB + kb));
  }
}

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

// Write one 64-byte staging row (this lane's output row; CPC = 64 / sizeof(OutT)
// values) with the 64-byte swizzle of the output tensor map: 16-byte unit u of
// row r lives at unit u ^ ((r >> 1) & 3), which also keeps the 8 rows a
// quarter-warp writes at once on distinct banks.  One-byte outputs are e4m3
// codes, rounded to nearest even and saturated at +-448.
template <typename OutT, int CPC>
__device__ __forceinline__ void stage_row64(uint8_t* stg, int lane, const float (&v)[CPC]) {
  uint8_t* row = stg + lane * 64;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    if constexpr (sizeof(OutT) == 1) {
      uint32_t c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        c[i] = __nv_cvt_float2_to_fp8x2(make_float2(v[q * 16 + 2 * i], v[q * 16 + 2 * i + 1]), __NV_SATFINITE,
                                        __NV_E4M3);
      w = make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16), c[4] | (c[5] << 16), c[6] | (c[7] << 16));
    } else if constexpr (sizeof(OutT) == 2) {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(v[q * 8 + 0], v[q * 8 + 1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(v[q * 8 + 2], v[q * 8 + 3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[q * 8 + 4], v[q * 8 + 5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(v[q * 8 + 6], v[q * 8 + 7]);
      w.x = *reinterpret_cast<uint32_t*>(&h0);
      w.y = *reinterpret_cast<uint32_t*>(&h1);
      w.z = *reinterpret_cast<uint32_t*>(&h2);
      w.w = *reinterpret_cast<uint32_t*>(&h3);
    } else {
      w = make_uint4(__float_as_uint(v[q * 4 + 0]), __float_as_uint(v[q * 4 + 1]), __float_as_uint(v[q * 4 + 2]),
                     __float_as_uint(v[q * 4 + 3]));
    }
    *reinterpret_cast<uint4*>(row + ((q ^ sw) << 4)) = w;
  }
}

// acc[j] += s * partial[j] for 32 columns, two columns per packed FMA.
__device__ __forceinline__ void promote32(float* acc, float s, const uint32_t (&r)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 t = __ffma2_rn(make_float2(s, s), make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                                make_float2(acc[j], acc[j + 1]));
    acc[j] = t.x;
    acc[j + 1] = t.y;
  }
}

template <bool CLUSTER = false>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* err,
                                          uint32_t code) {
  const bool ok = wait_bounded<CLUSTER>(bar, parity, abort, err, code);
  return __all_sync(0xffffffffu, ok);
}

constexpr int kWideProducerRegs = 64;
constexpr int kWideConsumerRegs = 216;
static_assert(128 * kWideProducerRegs + 256 * kWideConsumerRegs <= 384 * 168, "register split exceeds launch budget");

// CG = 1: one CTA computes a 128 x 256 tile.  CG = 2: a cluster of two CTAs
// (a CTA pair) computes a 256 x 256 tile with tcgen05.mma.cta_group::2 issued
// by the even ("leader") CTA; each CTA loads its own 128 A rows and 128 of the
// 256 B rows, so per SM a K block costs 32 KB of shared memory instead of 48 KB
// and more stages fit.  Both CTAs' TMA loads signal the leader's full barrier;
// the leader's commits arrive on both CTAs' barriers; the peer's consumers
// release the leader's accumulator barrier remotely.
// SPLIT: the plan splits the last round of tiles (stream-K, tile_order.h); a
// separate instantiation, so the consumers of plans without a split keep
// their registers for the promotion loop.
template <Mode MODE, int CG, int STAGES, typename OutT, bool SPLIT>
__global__ void __launch_bounds__(384, 1)
    wide_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const GemmArgs p) {
  constexpr int BM = 128, BK = 128, BN = 256;
  constexpr int BNL = BN / CG;  // B rows loaded by one CTA
  constexpr uint32_t A_BYTES = BM * BK, B_BYTES = BNL * BK;
  constexpr uint32_t STAGE_TX = CG * (A_BYTES + B_BYTES);  // bytes the leader's full barrier waits for
  constexpr int CONSUMER_WARPS = 8;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr bool IS_INT8 = MODE == Mode::kInt8;
  constexpr bool MX = MODE == Mode::kFp8Mx;  // block scales applied by the tensor core
  constexpr bool FULL_K = IS_INT8 || MODE == Mode::kFp8Rowwise || MX;  // accumulate over all of K in TMEM
  constexpr int NACC = 2;  // accumulator buffers
  // first TMEM column of accumulator buffer b (kFp8Mx: the buffers overlap)
  auto acc_col = [](int b) -> uint32_t { return MX ? (b ? kAcc1Col : 0u) : static_cast<uint32_t>(b * BN); };
  constexpr uint32_t IDESC = IS_INT8 ? idesc_s8_s32<BM * CG, BN>()
                                     : (MX ? idesc_mx_e4m3_f32<BM * CG, BN>() : idesc_e4m3_f32<BM * CG, BN>());
  static_assert(!MX || CG == 2, "hardware block scaling is built for CTA pairs");
  constexpr int CPC = 64 / sizeof(OutT);  // output columns per 64-byte staging row
  static_assert(CG == 1 || CG == 2, "CTA group is 1 or 2");
  using Smem = WideSmem<BNL, STAGES, wide_stage_bufs<MODE, CG>()>;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + sizeof(Smem) > dynamic_smem_bytes()) {  // never touch memory the launch did not provide
    if (threadIdx.x == 0) record_error(p.err, kErrSmemTooSmall);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + pad);
  volatile int* abort = &sm.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = CG == 2 ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = rank == 0;
  const int unit = blockIdx.x / CG, units = gridDim.x / CG;  // pair (or CTA) index / count

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], CONSUMER_WARPS * CG);
      mbar_init(&sm.ovl_empty[b], (CONSUMER_WARPS / 2) * CG);  // the half holding the shared columns
    }
    for (int i = 0; i < kScaleRing; ++i) {
      // FP8 block scales: every thread of the two scale warps fills, the
      // consumer warps release.  kFp8Mx: one arrival per scale warp of both
      // CTAs on the leader's barrier, released by the MMA's commit.
      mbar_init(&sm.sc_full[i], MX ? 2 * CG : 64);
      mbar_init(&sm.sc_empty[i], MX ? 1 : CONSUMER_WARPS);
    }
    mbar_init(&sm.drain, 1);
    for (int i = 0; i < CONSUMER_WARPS; ++i) mbar_init(&sm.part_bar[i], 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(&sm.tmem_base, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&sm.tmem_base, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2) {
    cluster_sync_all();  // barriers of both CTAs initialised before any remote signal
  } else {
    __syncthreads();
  }
  tc_fence_after();
  grid_dependency_wait();  // inputs may come from the previous kernel in the stream
  grid_launch_dependents();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
    regs_dec<kWideProducerRegs>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        uint32_t issued = 0, issued_phase = 0;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        WorkIter it(unit, units, p.sk_iters);
        WorkItem w;
        while (ok && it.next(w, units, p.dp_tiles, p.KB)) {
          const TileCoord tc = tile_coord(w.tile, p.grid_m, p.grid_n, p.group_m);
          const int m0 = tc.pm * (BM * CG) + rank * BM;
          const int nb0 = tc.pn * BN + rank * BNL;  // this CTA's B rows (tile columns)
          for (int kb = w.kb0; kb < w.kb1; ++kb) {
            if (!wait_bounded(&sm.empty[stage], phase ^ 1u, abort, p.err,
                              kErrTimeout | kRoleProducer | kWaitStageEmpty)) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(&sm.full[stage], STAGE_TX);
            if constexpr (CG == 2) {
              const uint32_t bar = mapa_shared(smem_u32(&sm.full[stage]), 0);
              tma_load_3d_pair(sm.a[stage], &tmA, bar, kb * BK, m0, tc.g);
              tma_load_3d_pair(sm.b[stage], &tmB, bar, kb * BK, nb0, tc.g);
            } else {
              tma_load_3d(sm.a[stage], &tmA, &sm.full[stage], kb * BK, m0, tc.g);
              tma_load_3d(sm.b[stage], &tmB, &sm.full[stage], kb * BK, nb0, tc.g);
            }
            issued |= 1u << stage;
            issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (ok) {
          // tail: wait until the MMAs have released every filled stage, so no
          // commit arrives on this CTA's barriers after it has retired
          for (int i = 0; i < STAGES && ok; ++i) {
            ok = wait_bounded(&sm.empty[stage], phase ^ 1u, abort, p.err, kErrTimeout | kRoleProducer | kWaitDrain);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        } else if (CG == 1 || leader) {  // let copies already in flight land before the CTA retires
          volatile int never = 0;
          for (int s = 0; s < STAGES; ++s)
            if ((issued >> s) & 1u)
              wait_bounded(&sm.full[s], (issued_phase >> s) & 1u, &never, nullptr, 0);
        } else {
          pause_ns(1000000);  // the peer's copies signal the leader's barriers; give them time to land
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer (leader CTA)
      // The whole warp runs the loop, so its waits, fences and descriptor
      // arithmetic are warp-uniform; one elected lane (always the same) issues
      // the copies, MMAs and the commits that track them.
      if (leader) {
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        uint32_t sfc = 0;  // kFp8Mx: scale-factor slots consumed (ring position)
        bool ok = true;
        WorkIter it(unit, units, p.sk_iters);
        WorkItem w;
        while (ok && it.next(w, units, p.dp_tiles, p.KB)) {
          for (int kb = w.kb0; kb < w.kb1; ++kb) {
            const bool first = kb == w.kb0, last = kb == w.kb1 - 1;
            // FP8: every K block starts a fresh partial in the next buffer;
            // INT8: the work item's accumulator is claimed once, at its first K block
            if (!FULL_K || first) {
              if (!warp_wait(&sm.acc_empty[buf], bphase ^ 1u, abort, p.err, kErrTimeout | kRoleMma | kWaitAccEmpty)) {
                ok = false;
                break;
              }
              // kFp8Mx: the previous tile, in the other buffer, has also read
              // the columns the two buffers share
              if (MX && !warp_wait(&sm.ovl_empty[buf ^ 1], buf == 1 ? bphase : (bphase ^ 1u), abort, p.err,
                                   kErrTimeout | kRoleMma | kWaitAccEmpty)) {
                ok = false;
                break;
              }
            }
            if (!warp_wait(&sm.full[stage], phase, abort, p.err, kErrTimeout | kRoleMma | kWaitStageFull)) {
              ok = false;
              break;
            }
            const int sslot = static_cast<int>(sfc % kSfRing);
            // kFp8Mx: this K block's byte in its slot (slots start at the item's first K block)
            const uint32_t sf_id = static_cast<uint32_t>((kb - w.kb0) & 3);
            if constexpr (MX) {  // both CTAs' scale factors of K blocks kb..kb+3 are in shared memory
              if (sf_id == 0 && !warp_wait<true>(&sm.sc_full[sslot], (sfc / kSfRing) & 1u, abort, p.err,
                                                 kErrTimeout | kRoleMma | kWaitScaleFull)) {
                ok = false;
                break;
              }
            }
            tc_fence_after();
            const uint32_t d = tmem + acc_col(buf);
            const uint64_t ad = sdesc_k_sw128(smem_u32(sm.a[stage]));
            const uint64_t bd = sdesc_k_sw128(smem_u32(sm.b[stage]));
            const bool slot_done = MX && (sf_id == 3 || last);  // kFp8Mx: the slot's last K block
            if (elect_one()) {
            if constexpr (MX) {
              if (sf_id == 0) {
                // scale factors of four K blocks to TMEM; issued by this
                // thread, the copies are ordered after the previous blocks'
                // MMAs and before this block's
                const uint32_t sf0 = smem_u32(sm.sf[sslot][0]);
                tmem_cp_32x128b_x4_pair(tmem + kSfaCol, sdesc_k_plain(sf0, 128));
                tmem_cp_32x128b_x4_pair(tmem + kSfbCol, sdesc_k_plain(sf0 + 512, 128));
                tmem_cp_32x128b_x4_pair(tmem + kSfbCol + 4, sdesc_k_plain(sf0 + 1024, 128));
              }
            }
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) {
              const uint32_t acc = FULL_K ? ((!first || k > 0) ? 1u : 0u) : (k > 0 ? 1u : 0u);
              if constexpr (CG == 2) {
                if constexpr (IS_INT8) {
                  mma_i8_pair(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                } else if constexpr (MX) {
                  mma_mxf8f6f4_pair(d, ad + 2 * k, bd + 2 * k, IDESC | (sf_id << 29) | (sf_id << 4),
                                    tmem + kSfaCol, tmem + kSfbCol, acc);
                } else {
                  mma_f8f6f4_pair(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                }
              } else {
                if constexpr (IS_INT8) {
                  mma_i8(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                } else {
                  mma_f8f6f4(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                }
              }
            }
            // FP8: one commit per K block both frees the stage for the producers
            // and tells the consumers that the partial is complete.  INT8: the
            // tile's last K block also commits the accumulator barrier.
            if constexpr (CG == 2) {
              mma_commit_pair_mc(&sm.empty[stage], 0x3);
              if (slot_done) mma_commit_pair_mc(&sm.sc_empty[sslot], 0x3);  // free it in both CTAs
              if (FULL_K && last) mma_commit_pair_mc(&sm.acc_full[buf], 0x3);
            } else {
              mma_commit(&sm.empty[stage]);
              if (FULL_K && last) mma_commit(&sm.acc_full[buf]);
            }
            }
            __syncwarp();
            if (slot_done) ++sfc;
            if (!FULL_K || last) {
              if (++buf == NACC) {
                buf = 0;
                bphase ^= 1u;
              }
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) {  // wait until every MMA already issued has finished with TMEM and smem
          if (elect_one()) {
            if constexpr (CG == 2) {
              mma_commit_pair(&sm.drain);
            } else {
              mma_commit(&sm.drain);
            }
          }
          __syncwarp();
          volatile int never = 0;
          wait_bounded(&sm.drain, 0, &never, nullptr, 0);
        }
      }
      __syncwarp();
    } else if constexpr (MX) {
      // ---------------------------------------------------------- scale-factor producer (warps 2, 3)
      // For every four K blocks of a tile, this CTA's 128 row scales
      // (x_scale) and the tile's two 128-column scales (w_scale) as e8m0
      // bytes in the chunk layout tcgen05.cp reads, byte j of each word for
      // the slot's K block j.  Both CTAs signal the leader's barrier; the
      // MMA's commit frees the slot in both.  Rows, column blocks and K blocks
      // outside the problem get 2^0 (their operands are zero-filled or their
      // byte is never selected).
      const int t = threadIdx.x - 64;  // 0..63: rows t and t + 64
      const uint32_t sc_full0 = CG == 2 ? mapa_shared(smem_u32(&sm.sc_full[0]), 0) : smem_u32(&sm.sc_full[0]);
      uint32_t cnt = 0;  // slots staged so far (ring position)
      bool ok = true;
      WorkIter it(unit, units, p.sk_iters);
      WorkItem w;
      while (ok && it.next(w, units, p.dp_tiles, p.KB)) {
        const TileCoord tc = tile_coord(w.tile, p.grid_m, p.grid_n, p.group_m);
        const int m0 = tc.pm * (BM * CG) + rank * BM, nb0 = tc.pn * 2;
        const int ma = m0 + t, mc = m0 + t + 64;
        for (int kb0 = w.kb0; ok && kb0 < w.kb1; kb0 += 4) {
          // the 16 loads of a slot are in flight together
          uint32_t wa = 0, wc = 0, w0 = 0, w1 = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const long long kb = kb0 + j;
            const bool in_k = kb < w.kb1;
            const uint32_t a = in_k && ma < p.M ? __ldg(p.xs + (static_cast<long long>(ma) * p.G + tc.g) * p.KB + kb)
                                                : 127u;
            const uint32_t c = in_k && mc < p.M ? __ldg(p.xs + (static_cast<long long>(mc) * p.G + tc.g) * p.KB + kb)
                                                : 127u;
            const uint32_t b0 =
                in_k && nb0 < p.NB ? __ldg(p.ws + (static_cast<long long>(tc.g) * p.NB + nb0) * p.KB + kb) : 127u;
            const uint32_t b1 = in_k && nb0 + 1 < p.NB
                                    ? __ldg(p.ws + (static_cast<long long>(tc.g) * p.NB + nb0 + 1) * p.KB + kb)
                                    : 127u;
            wa |= a << (8 * j);
            wc |= c << (8 * j);
            w0 |= b0 << (8 * j);
            w1 |= b1 << (8 * j);
          }
          const int slot = static_cast<int>(cnt % kSfRing);
          if (!warp_wait(&sm.sc_empty[slot], ((cnt / kSfRing) & 1u) ^ 1u, abort, p.err,
                         kErrTimeout | kRoleScale | kWaitScaleEmpty)) {
            ok = false;
            break;
          }
          uint32_t* sfa = reinterpret_cast<uint32_t*>(sm.sf[slot][0]);
          uint32_t* sfb = reinterpret_cast<uint32_t*>(sm.sf[slot][1]);  // chunks 1 and 2: 256 words
          sfa[4 * (t & 31) + (t >> 5)] = wa;      // row t
          sfa[4 * (t & 31) + (t >> 5) + 2] = wc;  // row t + 64
#pragma unroll
          for (int q = 0; q < 4; ++q) sfb[t + 64 * q] = q < 2 ? w0 : w1;
          fence_proxy_async_smem();  // visible to tcgen05.cp
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(sc_full0 + static_cast<uint32_t>(slot * sizeof(uint64_t)));
          ++cnt;
        }
      }
    } else if (!FULL_K) {
      // ---------------------------------------------------------- scale producer (warps 2, 3)
      // Stages scale_a of this CTA's 128 rows and scale_b of the tile's two
      // 128-column blocks for each K block into a ring kScaleRing blocks deep.
      // The loads of kScaleBatch consecutive K blocks are issued together, so
      // one global-load latency is paid per batch rather than per K block.
      const int t = threadIdx.x - 64;  // 0..63
      uint32_t cnt = 0;                // K blocks staged so far (ring position)
      bool ok = true;
      WorkIter it(unit, units, p.sk_iters);
      WorkItem w;
      while (ok && it.next(w, units, p.dp_tiles, p.KB)) {
        const TileCoord tc = tile_coord(w.tile, p.grid_m, p.grid_n, p.group_m);
        const int m0 = tc.pm * (BM * CG) + rank * BM, n0 = tc.pn * BN;
        for (int kb0 = w.kb0; ok && kb0 < w.kb1; kb0 += kScaleBatch) {
          const int nb = w.kb1 - kb0 < kScaleBatch ? w.kb1 - kb0 : kScaleBatch;
          float va[kScaleBatch], vc[kScaleBatch], vb[kScaleBatch];
#pragma unroll
          for (int i = 0; i < kScaleBatch; ++i) {
            if (i < nb) {
              va[i] = scale_row<MODE>(p, tc.g, m0 + t, kb0 + i);
              vc[i] = scale_row<MODE>(p, tc.g, m0 + t + 64, kb0 + i);
              vb[i] = t < 2 ? scale_col<MODE>(p, tc.g, kb0 + i, (n0 >> 7) + t) : 0.f;
            }
          }
#pragma unroll
          for (int i = 0; i < kScaleBatch; ++i) {
            if (i < nb) {
              const uint32_t c = cnt + static_cast<uint32_t>(i);
              const int slot = static_cast<int>(c % kScaleRing);
              const uint32_t ph = (c / kScaleRing) & 1u;
              if (!warp_wait(&sm.sc_empty[slot], ph ^ 1u, abort, p.err, kErrTimeout | kRoleScale | kWaitScaleEmpty)) {
                ok = false;
                break;
              }
              sm.sa[slot][t] = va[i];
              sm.sa[slot][t + 64] = vc[i];
              if (t < 2) sm.sb[slot][t] = vb[i];
              mbar_arrive(&sm.sc_full[slot]);
            }
          }
          cnt += static_cast<uint32_t>(nb);
        }
      }
    }
  } else {
    regs_inc<kWideConsumerRegs>();
    // ------------------------------------------------------------ consumers
    const int cw = warp - 4;
    const int lg = warp & 3;
    const int half = cw >> 2;
    const uint32_t t_lane = static_cast<uint32_t>(lg * 32) << 16;
    const int row = lg * 32 + lane;
    uint8_t* const stg0 = sm.stage_out[0][cw];  // this warp's (first) output staging buffer
    // With two staging buffers (INT8 on CTA pairs) a warp's output chunks
    // alternate between them, and every chunk commits exactly one bulk group
    // (empty when its box lies outside the output), so "at most one group
    // still reading" before a chunk means the buffer it is about to fill --
    // used two chunks earlier -- is free.
    int sbuf = 0;
    // release target of the accumulator buffers: the leader's barrier
    // release target of this warpgroup's accumulator half: the leader's barrier
    const uint32_t acc_empty0 =
        CG == 2 ? mapa_shared(smem_u32(&sm.acc_empty[0]), 0) : smem_u32(&sm.acc_empty[0]);
    const uint32_t ovl_empty0 =
        CG == 2 ? mapa_shared(smem_u32(&sm.ovl_empty[0]), 0) : smem_u32(&sm.ovl_empty[0]);
    int buf = 0, sslot = 0;
    uint32_t bphase = 0, ssph = 0;
    uint32_t kbc = 0;  // K blocks of this CTA's work items seen so far (stage = kbc % STAGES)
    // stream-K hand-over: this warp's part of unit u's partial-sum slot (a
    // [column / 4][lane] array of 16-byte pieces) and its flag word
    auto slot_piece = [&](int u) -> uint4* {
      return reinterpret_cast<uint4*>(p.sk_ws) + (static_cast<long long>(u * CG + rank) * 8 + cw) * (128 * 32 / 4);
    };
    auto slot_flag = [&](int u) -> uint32_t* {
      return p.sk_flags + static_cast<long long>(u * CG + rank) * kWsFlagsPerSlot + cw;
    };
    auto has_range = [&](int u) {
      return sk_range_begin(p.sk_iters, u, units) != sk_range_begin(p.sk_iters, u + 1, units);
    };
    // The head's copy of giver u's partial (this warp's 16 KB piece of the
    // slot) into this warp's share of the operand ring -- idle once the head
    // item, the unit's last, has finished its MMAs -- with one bulk copy; the
    // use-th copy of this warp waits for mbarrier phase use & 1.
    uint4* const part_smem =
        reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(&sm.a[0][0]) + cw * (STAGES * (A_BYTES + B_BYTES) / 8));
    auto fetch_partial = [&](int u, uint32_t use) -> bool {
      if (lane == 0) {
        fence_proxy_async_smem();    // this warp's reads of the previous piece before the copy overwrites it
        fence_proxy_async_global();  // the giver's stores, seen through its flag, before the async-proxy copy
        mbar_arrive_expect_tx(&sm.part_bar[cw], 128 * 32 * 4);
        bulk_load_g2s(part_smem, slot_piece(u), 128 * 32 * 4, &sm.part_bar[cw]);
      }
      return warp_wait(&sm.part_bar[cw], use & 1u, abort, p.err, kErrTimeout | kRoleConsumer | kWaitPartial);
    };
    // The item's stream-K role: a whole tile; a later part of a split tile (a
    // giver: its partial goes to this unit's slot); or the head of a split
    // tile, which adds the partials of units c_lo..c_hi, in that order, to its
    // own and stores the result.  (Worked out after the promotion loop, so
    // none of it is live across that loop.)
    auto givers_of = [&](const WorkItem& wi, int& lo, int& hi) {
      lo = unit + 1;
      hi = sk_unit_of(static_cast<long long>(wi.tile - p.dp_tiles) * p.KB + p.KB - 1, p.sk_iters, units);
    };
    // one work item; false when a wait gave up (the CTA is winding down)
    auto process = [&](const WorkItem& w) -> bool {
      bool ok = true;
      if constexpr (!FULL_K) {
        // fp32 accumulators; the promotion uses the packed two-wide FMA, which
        // halves the consumers' instruction count (the tensor pipe's issue
        // rate suffers when the consumer warps sharing its SM sub-partition
        // issue one FMA per column)
        float acc[128];
#pragma unroll
        for (int j = 0; j < 128; ++j) acc[j] = 0.f;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!warp_wait(&sm.sc_full[sslot], ssph, abort, p.err, kErrTimeout | kRoleConsumer | kWaitScaleFull)) {
            ok = false;
            break;
          }
          const float s_cur = sm.sa[sslot][row] * sm.sb[sslot][half];
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.sc_empty[sslot]);
          if (++sslot == kScaleRing) {
            sslot = 0;
            ssph ^= 1u;
          }
          // the MMA's commit on this K block's stage marks the partial complete;
          // the MMA runs at most two K blocks ahead, so the stage's phase
          // cannot advance again before this wait observes it
          if (!warp_wait(&sm.empty[kbc % STAGES], (kbc / STAGES) & 1u, abort, p.err,
                         kErrTimeout | kRoleConsumer | kWaitAccFull)) {
            ok = false;
            break;
          }
          ++kbc;
          tc_fence_after();
          const uint32_t tb = tmem + t_lane + static_cast<uint32_t>(buf * BN + half * 128);
          {
            uint32_t r0[32], r1[32];
            tmem_ld32x2(tb, tb + 32, r0, r1);
            promote32(acc, s_cur, r0);
            promote32(acc + 32, s_cur, r1);
          }
          {
            uint32_t r0[32], r1[32];
            tmem_ld32x2(tb + 64, tb + 96, r0, r1);
            // the partial is in registers: hand the TMEM buffer back before the math
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0 + static_cast<uint32_t>(buf * sizeof(uint64_t)));
            promote32(acc + 64, s_cur, r0);
            promote32(acc + 96, s_cur, r1);
          }
          buf ^= 1;
          if (buf == 0) bphase ^= 1u;
        }
        if (!ok) return false;
        const bool whole = w.kb0 == 0 && w.kb1 == p.KB;
        if (w.kb0 > 0) {  // giver
          uint4* dst = slot_piece(unit);
#pragma unroll
          for (int q = 0; q < 32; ++q)
            dst[q * 32 + lane] = make_uint4(__float_as_uint(acc[4 * q]), __float_as_uint(acc[4 * q + 1]),
                                            __float_as_uint(acc[4 * q + 2]), __float_as_uint(acc[4 * q + 3]));
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release_gpu(slot_flag(unit), 1u);
          return true;
        }
        int c_lo = 0, c_hi = -1;
        if (!whole) givers_of(w, c_lo, c_hi);
        uint32_t uses = 0;
        for (int u = c_lo; u <= c_hi; ++u) {
          if (!has_range(u)) continue;
          if (!wait_flag_bounded(slot_flag(u), abort, p.err, kErrTimeout | kRoleConsumer | kWaitPartial) ||
              !fetch_partial(u, uses++)) {
            ok = false;
            break;
          }
          const uint4* src = part_smem;
          // four 16-byte pieces at a time: the 128 accumulators leave no
          // registers for more
#pragma unroll
          for (int q0 = 0; q0 < 32; q0 += 4) {
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = src[(q0 + q) * 32 + lane];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[4 * (q0 + q)] += __uint_as_float(v[q].x);
              acc[4 * (q0 + q) + 1] += __uint_as_float(v[q].y);
              acc[4 * (q0 + q) + 2] += __uint_as_float(v[q].z);
              acc[4 * (q0 + q) + 3] += __uint_as_float(v[q].w);
            }
            asm volatile("" ::: "memory");  // keep the next group's loads after these adds
          }
          __syncwarp();  // every lane has read the piece before the next copy overwrites it
          if (lane == 0) *slot_flag(u) = 0u;  // zero again for the next launch
        }
        if (!ok) return false;
        const TileCoord tc = tile_coord(w.tile, p.grid_m, p.grid_n, p.group_m);
        const int m0 = tc.pm * (BM * CG) + rank * BM;
        const int ncol0 = tc.pn * BN + half * 128;
#pragma unroll
        for (int ch = 0; ch < 128 / CPC; ++ch) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          float v[CPC];
#pragma unroll
          for (int j = 0; j < CPC; ++j) v[j] = acc[ch * CPC + j];
          stage_row64<OutT, CPC>(stg0, lane, v);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && m0 + lg * 32 < p.M && ncol0 + ch * CPC < p.N) {  // skip boxes wholly outside
            tma_store_3d(&tmD, stg0, ncol0 + ch * CPC, m0 + lg * 32, tc.g);
            bulk_commit();
          }
        }
      } else {
        const TileCoord tc = tile_coord(w.tile, p.grid_m, p.grid_n, p.group_m);
        const int m0 = tc.pm * (BM * CG) + rank * BM;
        const int m = m0 + row;
        const int ncol0 = tc.pn * BN + half * 128;
        const bool whole = w.kb0 == 0 && w.kb1 == p.KB;
        const bool giver = w.kb0 > 0;
        int c_lo = 0, c_hi = -1;
        if (!whole && !giver) givers_of(w, c_lo, c_hi);
        if (!warp_wait(&sm.acc_full[buf], bphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitAccFull))
          return false;
        tc_fence_after();
        // the head adds every giver's partial to its accumulator in TMEM, in
        // unit order, before the normal epilogue reads it
        {
          const uint32_t tb_add = tmem + t_lane + acc_col(buf) + static_cast<uint32_t>(half * 128);
          uint32_t uses = 0;
          for (int u = c_lo; u <= c_hi; ++u) {
            if (!has_range(u)) continue;
            if (!wait_flag_bounded(slot_flag(u), abort, p.err, kErrTimeout | kRoleConsumer | kWaitPartial) ||
                !fetch_partial(u, uses++)) {
              ok = false;
              break;
            }
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t r[32];
              tmem_ld32(tb_add + 32 * ch, r);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const uint4 g4 = part_smem[(8 * ch + q) * 32 + lane];
                const uint32_t gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  if constexpr (IS_INT8) {
                    r[4 * q + e] += gv[e];  // exact int32 sum (two's complement)
                  } else {
                    r[4 * q + e] = __float_as_uint(__uint_as_float(r[4 * q + e]) + __uint_as_float(gv[e]));
                  }
                }
              }
              tmem_st32(tb_add + 32 * ch, r);
            }
            __syncwarp();  // every lane has read the piece before the next copy overwrites it
          }
        }
        if (!ok) return false;
        const bool has_row = p.s_row != nullptr, has_col = p.s_col != nullptr;
        const float sr = (has_row && m < p.M) ? __ldg(p.s_row + (IS_INT8 || p.s_row_stride != 0 ? m : 0)) : 1.f;
        // FP8 rowwise: this thread's column scales start at s_col_n and advance by col_step
        const int col_step = !IS_INT8 && p.s_col_stride != 0 ? 1 : 0;
        const float* s_col_n = IS_INT8 ? nullptr : p.s_col + ncol0 * col_step;
        const float s_res = sizeof(OutT) == 1 && p.s_result != nullptr ? __ldg(p.s_result) : 1.f;
        // The column scales (and FP8 rowwise biases) of this warp's 128 columns,
        // staged once per tile in shared memory -- the block-scale ring is idle
        // in these modes -- with coalesced loads, instead of a dependent global
        // load per output element (which made the INT8 epilogue three times
        // slower than its stores).  [0, 128): scales, 0 past N; [128, 256): biases.
        constexpr bool kColStage = !MX && !(sizeof(OutT) == 4 && !std::is_same<OutT, float>::value);
        static_assert(kScaleRing * 128 >= CONSUMER_WARPS * 256, "the column staging fits the idle scale ring");
        float* const colst = &sm.sa[0][0] + cw * 256;
        if constexpr (kColStage) {
          if (!giver) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int cl = lane + 32 * q;
              const int n = ncol0 + cl;
              float sc = 1.f, bn = 0.f;
              if constexpr (IS_INT8) {
                if (has_col) sc = n < p.N ? __ldg(p.s_col + n) : 0.f;
              } else {
                sc = n < p.N ? __ldg(s_col_n + cl * col_step) : 0.f;
                bn = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + n) : 0.f;
              }
              colst[cl] = sc;
              colst[128 + cl] = bn;
            }
            __syncwarp();
          }
        }
        const uint32_t tb = tmem + t_lane + acc_col(buf) + static_cast<uint32_t>(half * 128);
        // kFp8Mx: the 32 columns this buffer shares with the other one are
        // the last of half 1 (buffer 0) or the first of half 0 (buffer 1);
        // the warps holding them read those chunks first and release them,
        // so the next tile's MMAs can start while the rest drains
        constexpr int NCH = 128 / CPC, OVC = 32 / CPC;
        const bool ovl_here = MX && (buf == 0 ? half == 1 : half == 0);
        const int rot = MX && buf == 0 && half == 1 ? NCH - OVC : 0;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          if (!giver) {
            if (lane == 0) {
              if constexpr (Smem::kStageBufs == 2) {
                bulk_wait_read1();
              } else {
                bulk_wait_read_all();
              }
            }
            __syncwarp();
          }
          const int c0 = (MX ? (ch + rot) % NCH : ch) * CPC;
          uint32_t r[CPC];
          if constexpr (CPC == 64) {
            tmem_ld64(tb + c0, r);
          } else if constexpr (CPC == 32) {
            tmem_ld32(tb + c0, r);
          } else {
            tmem_ld16(tb + c0, r);
          }
          if constexpr (MX) {
            if (ovl_here && ch == OVC - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(ovl_empty0 + static_cast<uint32_t>(buf * sizeof(uint64_t)));
            }
          }
          if (giver) {  // the raw accumulator (fp32, or int32 for INT8) to this unit's slot
            uint4* dst = slot_piece(unit) + (c0 / 4) * 32 + lane;
#pragma unroll
            for (int q = 0; q < CPC / 4; ++q) dst[q * 32] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
            continue;
          }
          float v[CPC];
          if constexpr (sizeof(OutT) == 4 && !std::is_same<OutT, float>::value) {
#pragma unroll
            for (int j = 0; j < CPC; ++j) v[j] = __uint_as_float(r[j]);  // raw int32 accumulator
          } else if constexpr (MX) {
#pragma unroll
            for (int j = 0; j < CPC; ++j) v[j] = __uint_as_float(r[j]);  // scales already applied
          } else if constexpr (!IS_INT8) {
            // FP8 rowwise / tensorwise: acc * (s_a * s_b) + bias[n]
#pragma unroll
            for (int j = 0; j < CPC; ++j)
              v[j] = fmaf(__uint_as_float(r[j]), sr * colst[c0 + j], colst[128 + c0 + j]);
            if constexpr (sizeof(OutT) == 1) {
#pragma unroll
              for (int j = 0; j < CPC; ++j) v[j] *= s_res;  // output scale of the e4m3 result
            }
          } else {
#pragma unroll
            for (int j = 0; j < CPC; ++j) {
              float f = __int2float_rn(static_cast<int>(r[j]));
              if (has_row) f = __fmul_rn(f, sr);
              if (has_col) f = __fmul_rn(f, colst[c0 + j]);
              v[j] = f;
            }
          }
          uint8_t* stg = stg0 + sbuf * static_cast<int>(sizeof(sm.stage_out[0]));
          stage_row64<OutT, CPC>(stg, lane, v);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (m0 + lg * 32 < p.M && ncol0 + c0 < p.N) tma_store_3d(&tmD, stg, ncol0 + c0, m0 + lg * 32, tc.g);
            bulk_commit();
          }
          if constexpr (Smem::kStageBufs == 2) sbuf ^= 1;
        }
        if (giver) {
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release_gpu(slot_flag(unit), 1u);
        } else if (!whole) {
          __syncwarp();
          if (lane == 0)
            for (int u = c_lo; u <= c_hi; ++u) *slot_flag(u) = 0u;  // zero again for the next launch
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0 + static_cast<uint32_t>(buf * sizeof(uint64_t)));
        if (++buf == NACC) {
          buf = 0;
          bphase ^= 1u;
        }
      }
          return true;
    };
    // whole tiles (the data-parallel rounds), then this unit's stream-K range
    bool live = true;
    for (int tile = unit; live && tile < p.dp_tiles; tile += units) live = process(WorkItem{tile, 0, p.KB});
    if (SPLIT && live && p.sk_iters > 0) {
      // the range's position lives in shared memory, so no iterator state is
      // held in registers across an item's promotion loop
      if (lane == 0) sm.sk_pos[cw] = sk_range_begin(p.sk_iters, unit, units);
      __syncwarp();
      while (live) {
        WorkIter it(unit, units, p.sk_iters);
        it.next_dp = p.dp_tiles;  // the whole tiles are done
        it.sk = sm.sk_pos[cw];
        WorkItem w;
        if (!it.next(w, units, p.dp_tiles, p.KB)) break;
        __syncwarp();
        if (lane == 0) sm.sk_pos[cw] = it.sk;
        __syncwarp();
        live = process(w);
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  if constexpr (CG == 2) {
    cluster_sync_all();  // no CTA retires while its peer may still signal it
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) {
      tmem_dealloc_pair(tmem, TMEM_COLS);
    } else {
      tmem_dealloc(tmem, TMEM_COLS);
    }
  }
}

}  // namespace bsg

// Skinny-M FP8 block-scaled GEMM for sm_100a: swap-AB + cluster split-K.
//
// For small M the weight stream B dominates (HBM-bound).  Each CTA computes the
// transposed tile  D^T[128 n-rows x BMT m-cols] = B_tile . A_tile^T  so the
// 128-row side of tcgen05.mma is filled by weight rows and the few activation
// rows become the MMA N dimension (16..128).  K is split across the S CTAs of
// a thread-block cluster; their fp32 partials are summed through distributed
// shared memory in rank order 0..S-1 (deterministic, no global workspace, no
// second launch) -- the same fp32 partial-sum-then-cast structure as the
// split-K decomposition decomposeK in pytorch/torch/_inductor/kernel/mm.py.
//
// Roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer of the even K
// blocks, warp 3 MMA issuer of the odd K blocks, warp 2 scale producer,
// warps 4.. consumers.  Consumer warp w reads TMEM lanes
// 32*(w%4).. (32 weight rows) and, when there are eight consumer warps, one
// half of the BMT accumulator columns.  The scale producer writes, per K block,
// s[j] = scale_a[m0+j, kb] * scale_b[kb, nb] (one value per activation row,
// shared by the CTA because its 128 weight rows form one 128-wide scale block)
// into a small shared ring.
//
// The grid never exceeds one wave (the host picks S accordingly), so every
// CTA streams its weights from the first microsecond: the producer issues the
// first ring of loads before the CTA-wide barrier, and with programmatic
// dependent launch the next kernel's prologue overlaps this one's tail.
#pragma once

#include "sm100.cuh"
#include "wide_kernel.cuh"

namespace bsg {

constexpr int kSkinnyScaleRing = 16;  // K blocks of scales staged ahead
constexpr int kSkinnyScaleBatch = 8;  // K blocks whose scale loads are in flight together
constexpr int kSkinnyAccBufs = 4;     // TMEM accumulator buffers (MMA runs up to 4 K blocks ahead)

// Shape of the kernel for an activation tile of BMT rows (the MMA N).
template <int BMT>
struct SkinnyCfg {
  static constexpr int CW = BMT >= 64 ? 8 : 4;  // consumer warps (two per TMEM lane group when 8)
  static constexpr int CPW = BMT * 4 / CW;      // accumulator columns per consumer thread
  static constexpr int THREADS = 128 + 32 * CW;
  // Shared memory (operand ring) and registers (CPW accumulators per consumer
  // thread) decide how many CTAs share an SM; the ring depth fills what is left.
  static constexpr int CTAS_PER_SM = BMT <= 16 ? 3 : (BMT <= 32 ? 2 : 1);
  static constexpr int STAGES = BMT <= 16 ? 4 : (BMT <= 32 ? 5 : (BMT <= 64 ? 8 : 6));
  static constexpr uint32_t ACC_COLS = BMT < 32 ? 32u : static_cast<uint32_t>(BMT);
  static constexpr uint32_t TMEM_COLS = kSkinnyAccBufs * ACC_COLS;  // a power of two: 128, 256 or 512
  static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "co-resident CTAs must fit in the SM's 512 TMEM columns");
};

template <int BMT, int STAGES, int SSTAGES>
struct SkinnySmem {
  uint8_t b[STAGES][128 * 128];  // weight rows  (MMA operand "A", 128 rows)
  uint8_t a[STAGES][BMT * 128];  // activation rows (MMA operand "B", BMT rows)
  float scale[SSTAGES][BMT];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[kSkinnyAccBufs];
  uint64_t acc_empty[kSkinnyAccBufs];
  uint64_t sc_full[SSTAGES];
  uint64_t sc_empty[SSTAGES];
  uint64_t drain[2];  // one per MMA-issuing thread (abort path)
  uint32_t tmem_base;
  int abort;
};

template <int BMT>
using SkinnySmemFor = SkinnySmem<BMT, SkinnyCfg<BMT>::STAGES, kSkinnyScaleRing>;

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* ptr, float v) {
  if constexpr (sizeof(OutT) == 2) {
    *reinterpret_cast<__nv_bfloat16*>(ptr) = __float2bfloat16_rn(v);
  } else {
    *reinterpret_cast<float*>(ptr) = v;
  }
}

// Four consecutive outputs; `ptr` is 8-byte (bf16) or 16-byte (f32) aligned.
template <typename OutT>
__device__ __forceinline__ void store_out4(OutT* ptr, float4 v) {
  if constexpr (sizeof(OutT) == 2) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(ptr) = u;
  } else {
    *reinterpret_cast<float4*>(ptr) = v;
  }
}

// Output element (m, g, n) lives at out + m*o_sm + g*o_sg + n.
struct SkinnyOut {
  void* out;
  long long o_sm, o_sg;
};

// CPW consecutive TMEM columns of this warp's 32 lanes with a single wait.
template <int CPW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[CPW]) {
  if constexpr (CPW == 16) {
    tmem_ld16(taddr, r);
  } else if constexpr (CPW == 32) {
    tmem_ld32(taddr, r);
  } else {
    static_assert(CPW == 64, "16, 32 or 64 columns per consumer thread");
    tmem_ld64(taddr, r);
  }
}

// Split-K reduction across the S CTAs of a cluster.  Every CTA has published
// its fp32 partial as red[j * 128 + row] (j = activation row of the tile, row =
// weight row).  CTA `rank` owns weight rows [rank*R, rank*R + R), R = 128/S;
// for each (j, 4 rows) it reads the S partials -- all loads of a thread are in
// flight together -- sums them in rank order 0..S-1 and stores 4 outputs.
template <int S, int BMT, int CT, typename OutT>
__device__ __forceinline__ void skinny_cluster_reduce(const float* red, int rank, int ct, int m0, int n0, int g,
                                                      const GemmArgs& p, const SkinnyOut& o) {
  constexpr int R = 128 / S;
  constexpr int R4 = R / 4;
  constexpr int T = BMT * R4;           // float4 items owned by this CTA
  constexpr int U = (T + CT - 1) / CT;  // items per consumer thread
  const uint32_t red_s = smem_u32(red);
  float4 v[U][S];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int it = ct + u * CT;
    if (it < T) {
      const int j = it / R4, r = rank * R + 4 * (it % R4);
      const uint32_t off = red_s + static_cast<uint32_t>((j * 128 + r) * 4);
#pragma unroll
      for (int q = 0; q < S; ++q) v[u][q] = ld_shared_cluster_f4(mapa_shared(off, static_cast<uint32_t>(q)));
    }
  }
  OutT* out = static_cast<OutT*>(o.out);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int it = ct + u * CT;
    if (it < T) {
      const int j = it / R4, r = rank * R + 4 * (it % R4);
      float4 s = v[u][0];
#pragma unroll
      for (int q = 1; q < S; ++q) {
        s.x += v[u][q].x;
        s.y += v[u][q].y;
        s.z += v[u][q].z;
        s.w += v[u][q].w;
      }
      const int m = m0 + j, n = n0 + r;
      if (m < p.M && n < p.N) {
        OutT* dst = out + static_cast<long long>(m) * o.o_sm + static_cast<long long>(g) * o.o_sg + n;
        if (n + 3 < p.N) {
          store_out4<OutT>(dst, s);
        } else {
          const float e[4] = {s.x, s.y, s.z, s.w};
          for (int c = 0; c < 4 && n + c < p.N; ++c) store_out<OutT>(dst + c, e[c]);
        }
      }
    }
  }
}

template <Mode MODE, int BMT, typename OutT>
__global__ void __launch_bounds__(SkinnyCfg<BMT>::THREADS, SkinnyCfg<BMT>::CTAS_PER_SM)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const GemmArgs p, const SkinnyOut o) {
  using Cfg = SkinnyCfg<BMT>;
  constexpr int BK = 128;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int SSTAGES = kSkinnyScaleRing;
  constexpr int SBATCH = kSkinnyScaleBatch;
  constexpr int NBUF = kSkinnyAccBufs;
  constexpr int CW = Cfg::CW;
  constexpr int CPW = Cfg::CPW;
  constexpr int CT = 32 * CW;  // consumer threads
  constexpr uint32_t A_BYTES = BMT * BK, B_BYTES = 128 * BK;
  constexpr uint32_t ACC_COLS = Cfg::ACC_COLS;
  constexpr uint32_t IDESC = idesc_e4m3_f32<128, BMT>();
  static_assert(MODE != Mode::kInt8, "skinny path is FP8 only");
  static_assert(BMT % 16 == 0 && BMT >= 16 && BMT <= 128, "MMA N must be 16..128 in steps of 16");
  using Smem = SkinnySmem<BMT, STAGES, SSTAGES>;
  static_assert(sizeof(float) * 128 * BMT <= sizeof(uint8_t) * STAGES * (128 + BMT) * 128,
                "split-K reduction buffer reuses the operand ring");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + sizeof(Smem) > dynamic_smem_bytes()) {  // never touch memory the launch did not provide
    if (threadIdx.x == 0) record_error(p.err, kErrSmemTooSmall);
    return;
  }
  if (p.splits != 1 && p.splits != 2 && p.splits != 4 && p.splits != 8) {  // the reduction handles these
    if (threadIdx.x == 0) record_error(p.err, kErrBadSplit);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + pad);
  volatile int* abort = &sm.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int S = p.splits;
  const int rank = S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int n_tile = blockIdx.x / S;
  const int m0 = blockIdx.y * BMT;
  const int g = blockIdx.z;
  const int n0 = n_tile * 128;
  const int nb = n0 >> 7;
  // balanced split of the K blocks over the cluster
  const int kb_lo = static_cast<int>((static_cast<long long>(p.KB) * rank) / S);
  const int kb_hi = static_cast<int>((static_cast<long long>(p.KB) * (rank + 1)) / S);
  const int nkb = kb_hi - kb_lo;

  // Producer state lives in thread 0, which initialises the barriers and
  // issues the first ring of loads before the CTA-wide barrier.
  int p_i = 0, p_stage = 0;
  uint32_t p_phase = 0, issued = 0, issued_phase = 0;
  bool p_ok = true;
  auto produce = [&](int upto) {
    for (; p_i < upto; ++p_i) {
      const int kb = kb_lo + p_i;
      if (!wait_bounded(&sm.empty[p_stage], p_phase ^ 1u, abort, p.err, kErrTimeout | kRoleProducer | kWaitStageEmpty)) {
        p_ok = false;
        return;
      }
      mbar_arrive_expect_tx(&sm.full[p_stage], A_BYTES + B_BYTES);
      tma_load_3d(sm.b[p_stage], &tmB, &sm.full[p_stage], kb * BK, n0, g);
      tma_load_3d(sm.a[p_stage], &tmA, &sm.full[p_stage], kb * BK, m0, g);
      issued |= 1u << p_stage;
      issued_phase = (issued_phase & ~(1u << p_stage)) | (p_phase << p_stage);
      if (++p_stage == STAGES) {
        p_stage = 0;
        p_phase ^= 1u;
      }
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], CW);
    }
    for (int s = 0; s < SSTAGES; ++s) {
      mbar_init(&sm.sc_full[s], 32);
      mbar_init(&sm.sc_empty[s], CW);
    }
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    sm.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    // Warm L2 with the first ring of tiles while the previous grid drains;
    // the copies into shared memory wait for it.
    for (int i = 0; i < nkb && i < STAGES; ++i) {
      tma_prefetch_l2_3d(&tmB, (kb_lo + i) * BK, n0, g);
      tma_prefetch_l2_3d(&tmA, (kb_lo + i) * BK, m0, g);
    }
    grid_dependency_wait();  // inputs may come from the previous kernel in the stream
    produce(nkb < STAGES ? nkb : STAGES);  // a fresh ring: these waits return at once
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  // Scale producer state: the loads of SBATCH K blocks are issued together
  // (one global-load latency per batch); the first batch is in flight before
  // the CTA-wide barrier.
  constexpr int PER_LANE = (BMT + 31) / 32;
  float sv[SBATCH][PER_LANE];  // scale_a of the batch, lane j of row j
  float sc[SBATCH];            // scale_b of the batch
  auto load_scales = [&](int i0) {
    const int cnt = nkb - i0 < SBATCH ? nkb - i0 : SBATCH;
#pragma unroll
    for (int i = 0; i < SBATCH; ++i) {
      if (i < cnt) {
        const int kb = kb_lo + i0 + i;
        sc[i] = scale_col<MODE>(p, g, kb, nb);
#pragma unroll
        for (int q = 0; q < PER_LANE; ++q) {
          const int j = lane + 32 * q;
          sv[i][q] = j < BMT ? scale_row<MODE>(p, g, m0 + j, kb) : 0.f;
        }
      }
    }
  };
  if (warp == 2) {
    grid_dependency_wait();
    load_scales(0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x != 0 && warp != 2) grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem = sm.tmem_base;

  float acc[CPW];
#pragma unroll
  for (int j = 0; j < CPW; ++j) acc[j] = 0.f;
  bool consumer_ok = true;

  if (warp == 0) {
    if (lane == 0) {
      if (p_ok) produce(nkb);
      if (!p_ok) {
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) wait_bounded(&sm.full[s], (issued_phase >> s) & 1u, &never, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // Two MMA-issuing threads: warp 1 takes the even K blocks and warp 3 the
    // odd ones.  Consecutive K blocks use different stages and accumulator
    // buffers, so the two streams are independent; each thread's commits
    // track its own MMAs.  (One thread issuing everything spends most of a
    // K block's time in the issue of its four MMAs.)
    // Each issuing warp runs its loop as a whole (warp-uniform waits and
    // descriptor arithmetic); one elected lane issues the MMAs and commits.
    {
      const int issuer = warp == 3 ? 1 : 0;
      bool ok = true;
      for (int i = issuer; i < nkb; i += 2) {
        const int stage = i % STAGES, buf = i % NBUF;
        const uint32_t phase = static_cast<uint32_t>(i / STAGES) & 1u;
        const uint32_t bphase = static_cast<uint32_t>(i / NBUF) & 1u;
        if (!warp_wait(&sm.acc_empty[buf], bphase ^ 1u, abort, p.err, kErrTimeout | kRoleMma | kWaitAccEmpty) ||
            !warp_wait(&sm.full[stage], phase, abort, p.err, kErrTimeout | kRoleMma | kWaitStageFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf) * ACC_COLS;
        const uint64_t ad = sdesc_k_sw128(smem_u32(sm.b[stage]));
        const uint64_t bd = sdesc_k_sw128(smem_u32(sm.a[stage]));
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) mma_f8f6f4(d, ad + 2 * k, bd + 2 * k, IDESC, k > 0 ? 1u : 0u);
          mma_commit(&sm.empty[stage]);
          mma_commit(&sm.acc_full[buf]);
        }
        __syncwarp();
      }
      if (!ok) {  // wait until this warp's MMAs have finished with TMEM and shared memory
        if (elect_one()) mma_commit(&sm.drain[issuer]);
        __syncwarp();
        volatile int never = 0;
        wait_bounded(&sm.drain[issuer], 0, &never, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // scale producer: s[j] = scale_a[m0+j, kb] * scale_b[kb, nb] for the BMT
    // activation rows of this CTA, SBATCH K blocks per batch
    bool ok = true;
    for (int i0 = 0; ok && i0 < nkb; i0 += SBATCH) {
      if (i0 > 0) load_scales(i0);
      const int cnt_batch = nkb - i0 < SBATCH ? nkb - i0 : SBATCH;
#pragma unroll
      for (int i = 0; i < SBATCH; ++i) {
        if (i < cnt_batch) {
          const uint32_t cnt = static_cast<uint32_t>(i0 + i);
          const int si = static_cast<int>(cnt % SSTAGES);
          const uint32_t ph = (cnt / SSTAGES) & 1u;
          if (!warp_wait(&sm.sc_empty[si], ph ^ 1u, abort, p.err, kErrTimeout | kRoleScale | kWaitScaleEmpty)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int q = 0; q < PER_LANE; ++q) {
            const int j = lane + 32 * q;
            if (j < BMT) sm.scale[si][j] = sv[i][q] * sc[i];
          }
          mbar_arrive(&sm.sc_full[si]);
        }
      }
    }
  } else if (warp >= 4) {
    // consumers: per K block, one TMEM load of CPW columns, release the
    // accumulator buffer, then acc[j] += s[j] * partial[j] in registers
    const int c0 = ((warp - 4) >> 2) * CPW;  // first accumulator column of this warp
    const uint32_t t_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int buf = 0, si = 0;
    uint32_t bphase = 0, sphase = 0;
    for (int i = 0; i < nkb; ++i) {
      if (!warp_wait(&sm.acc_full[buf], bphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitAccFull) ||
          !warp_wait(&sm.sc_full[si], sphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitScaleFull)) {
        consumer_ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[CPW];
      tmem_ld_cols<CPW>(tmem + t_lane + static_cast<uint32_t>(buf) * ACC_COLS + static_cast<uint32_t>(c0), r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
      const float4* s4 = reinterpret_cast<const float4*>(&sm.scale[si][c0]);
#pragma unroll
      for (int q = 0; q < CPW / 4; ++q) {  // packed two-wide FMAs
        const float4 s = s4[q];
        const float2 lo = __ffma2_rn(make_float2(s.x, s.y),
                                     make_float2(__uint_as_float(r[4 * q + 0]), __uint_as_float(r[4 * q + 1])),
                                     make_float2(acc[4 * q + 0], acc[4 * q + 1]));
        const float2 hi = __ffma2_rn(make_float2(s.z, s.w),
                                     make_float2(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])),
                                     make_float2(acc[4 * q + 2], acc[4 * q + 3]));
        acc[4 * q + 0] = lo.x;
        acc[4 * q + 1] = lo.y;
        acc[4 * q + 2] = hi.x;
        acc[4 * q + 3] = hi.y;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sc_empty[si]);
      if (++buf == NBUF) {
        buf = 0;
        bphase ^= 1u;
      }
      if (++si == SSTAGES) {
        si = 0;
        sphase ^= 1u;
      }
    }
  }

  // --------------------------------------------------------------- epilogue
  const bool is_consumer = warp >= 4;
  const int ct = static_cast<int>(threadIdx.x) - 128;  // 0..CT-1 for consumers
  const int wrow = (warp & 3) * 32 + lane;             // consumer's weight row = its TMEM lane
  const int c0 = ((warp - 4) >> 2) * CPW;
  if (S == 1) {
    // Stage the tile as output rows [m][n] in the idle operand ring (every MMA
    // has completed once the last partial was read), then write 16-byte
    // chunks, consecutive threads covering consecutive bytes of a row.
    if (is_consumer) {
      OutT* stg = reinterpret_cast<OutT*>(&sm.b[0][0]);
      if (consumer_ok) {
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          if constexpr (sizeof(OutT) == 2) {
            stg[(c0 + j) * 128 + wrow] = __float2bfloat16_rn(acc[j]);
          } else {
            stg[(c0 + j) * 128 + wrow] = acc[j];
          }
        }
      }
      named_bar_sync(1, CT);
      constexpr int EPC = 16 / static_cast<int>(sizeof(OutT));  // elements per 16-byte chunk
      constexpr int CPR = 128 / EPC;                            // chunks per staged row
      OutT* out = static_cast<OutT*>(o.out) + static_cast<long long>(g) * o.o_sg;
      if (consumer_ok) {
        for (int c = ct; c < BMT * CPR; c += CT) {
          const int row = c / CPR, col = (c % CPR) * EPC;
          const int m = m0 + row, n = n0 + col;
          if (m < p.M && n < p.N) {
            OutT* dst = out + static_cast<long long>(m) * o.o_sm + n;
            const OutT* src = stg + row * 128 + col;
            if (n + EPC <= p.N) {
              *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
            } else {
              for (int e = 0; e < EPC && n + e < p.N; ++e) dst[e] = src[e];
            }
          }
        }
      }
    }
  } else {
    // every consumer publishes its partial column-major: red[j][row]
    float* red = reinterpret_cast<float*>(&sm.b[0][0]);
    if (is_consumer) {
#pragma unroll
      for (int j = 0; j < CPW; ++j) red[(c0 + j) * 128 + wrow] = consumer_ok ? acc[j] : 0.f;
    }
    cluster_sync_all();
    if (is_consumer) {
      if (S == 2) skinny_cluster_reduce<2, BMT, CT, OutT>(red, rank, ct, m0, n0, g, p, o);
      else if (S == 4) skinny_cluster_reduce<4, BMT, CT, OutT>(red, rank, ct, m0, n0, g, p, o);
      else skinny_cluster_reduce<8, BMT, CT, OutT>(red, rank, ct, m0, n0, g, p, o);
    }
    cluster_sync_all();  // peers may still be reading this CTA's partial
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace bsg

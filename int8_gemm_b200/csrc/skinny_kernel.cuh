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
// Roles: warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 consumers (warp w
// owns TMEM lanes 32*(w%4).., i.e. 32 weight rows, and all BMT columns),
// warp 6 scale producer: per K block it writes s[j] = scale_a[m0+j, kb] *
// scale_b[kb, nb] (one value per activation row, shared by the CTA because the
// 128 weight rows form one 128-wide scale block) into a small shared ring.
#pragma once

#include "sm100.cuh"
#include "wide_kernel.cuh"

namespace bsg {

constexpr int kSkinnyScaleRing = 16;  // K blocks of scales staged ahead
constexpr int kSkinnyScaleBatch = 8;  // K blocks whose scale loads are in flight together

template <int BMT, int STAGES, int SSTAGES>
struct SkinnySmem {
  uint8_t b[STAGES][128 * 128];  // weight rows  (MMA operand "A", 128 rows)
  uint8_t a[STAGES][BMT * 128];  // activation rows (MMA operand "B", BMT rows)
  float scale[SSTAGES][BMT];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t sc_full[SSTAGES];
  uint64_t sc_empty[SSTAGES];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ constexpr uint32_t tmem_cols_for(int cols) {
  return cols <= 32 ? 32u : cols <= 64 ? 64u : cols <= 128 ? 128u : cols <= 256 ? 256u : 512u;
}

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* ptr, float v) {
  if constexpr (sizeof(OutT) == 2) {
    *reinterpret_cast<__nv_bfloat16*>(ptr) = __float2bfloat16_rn(v);
  } else {
    *reinterpret_cast<float*>(ptr) = v;
  }
}

// Output element (m, g, n) lives at out + m*o_sm + g*o_sg + n.
struct SkinnyOut {
  void* out;
  long long o_sm, o_sg;
};

template <Mode MODE, int BMT, int STAGES, typename OutT>
__global__ void __launch_bounds__(224, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const GemmArgs p, const SkinnyOut o) {
  constexpr int BK = 128;
  constexpr int SSTAGES = kSkinnyScaleRing;
  constexpr int SBATCH = kSkinnyScaleBatch;
  constexpr uint32_t A_BYTES = BMT * BK, B_BYTES = 128 * BK;
  constexpr int CONSUMER_WARPS = 4;
  constexpr uint32_t ACC_COLS = BMT < 32 ? 32u : static_cast<uint32_t>(BMT);  // one accumulator buffer
  constexpr uint32_t TMEM_COLS = tmem_cols_for(2 * ACC_COLS);
  constexpr uint32_t IDESC = idesc_e4m3_f32<128, BMT>();
  static_assert(MODE != Mode::kInt8, "skinny path is FP8 only");
  static_assert(BMT % 16 == 0 && BMT >= 16 && BMT <= 128, "MMA N must be 16..128 in steps of 16");
  static_assert(2 * ACC_COLS <= TMEM_COLS, "two accumulator buffers");
  using Smem = SkinnySmem<BMT, STAGES, SSTAGES>;
  static_assert(sizeof(float) * 128 * BMT <= sizeof(uint8_t) * STAGES * (128 + BMT) * 128,
                "split-K reduction buffer reuses the operand ring");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + sizeof(Smem) > dynamic_smem_bytes()) {  // never touch memory the launch did not provide
    if (threadIdx.x == 0) record_error(p.err, kErrSmemTooSmall);
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], CONSUMER_WARPS);
    }
    for (int s = 0; s < SSTAGES; ++s) {
      mbar_init(&sm.sc_full[s], 32);
      mbar_init(&sm.sc_empty[s], CONSUMER_WARPS);
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

  float acc[BMT];
#pragma unroll
  for (int j = 0; j < BMT; ++j) acc[j] = 0.f;
  bool consumer_ok = true;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      uint32_t issued = 0, issued_phase = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int kb = kb_lo + i;
        if (!wait_bounded(&sm.empty[stage], phase ^ 1u, abort, p.err, kErrTimeout | kRoleProducer | kWaitStageEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[stage], A_BYTES + B_BYTES);
        tma_load_3d(sm.b[stage], &tmB, &sm.full[stage], kb * BK, n0, g);
        tma_load_3d(sm.a[stage], &tmA, &sm.full[stage], kb * BK, m0, g);
        issued |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) wait_bounded(&sm.full[s], (issued_phase >> s) & 1u, &never, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!wait_bounded(&sm.acc_empty[buf], bphase ^ 1u, abort, p.err, kErrTimeout | kRoleMma | kWaitAccEmpty) ||
            !wait_bounded(&sm.full[stage], phase, abort, p.err, kErrTimeout | kRoleMma | kWaitStageFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf) * ACC_COLS;
        const uint64_t ad = sdesc_k_sw128(smem_u32(sm.b[stage]));
        const uint64_t bd = sdesc_k_sw128(smem_u32(sm.a[stage]));
#pragma unroll
        for (int k = 0; k < BK / 32; ++k) mma_f8f6f4(d, ad + 2 * k, bd + 2 * k, IDESC, k > 0 ? 1u : 0u);
        mma_commit(&sm.empty[stage]);
        mma_commit(&sm.acc_full[buf]);
        buf ^= 1;
        if (buf == 0) bphase ^= 1u;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        mma_commit(&sm.drain);
        volatile int never = 0;
        wait_bounded(&sm.drain, 0, &never, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // scale producer: s[j] = scale_a[m0+j, kb] * scale_b[kb, nb] for the BMT
    // activation rows of this CTA.  The loads of SBATCH K blocks are issued
    // together, so one global-load latency is paid per batch.
    constexpr int PER_LANE = (BMT + 31) / 32;
    bool ok = true;
    for (int i0 = 0; ok && i0 < nkb; i0 += SBATCH) {
      const int nb_batch = nkb - i0 < SBATCH ? nkb - i0 : SBATCH;
      float v[SBATCH][PER_LANE];
      float c[SBATCH];
#pragma unroll
      for (int i = 0; i < SBATCH; ++i) {
        if (i < nb_batch) {
          const int kb = kb_lo + i0 + i;
          c[i] = scale_col<MODE>(p, g, kb, nb);
#pragma unroll
          for (int q = 0; q < PER_LANE; ++q) {
            const int j = lane + 32 * q;
            v[i][q] = j < BMT ? scale_row<MODE>(p, g, m0 + j, kb) : 0.f;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < SBATCH; ++i) {
        if (i < nb_batch) {
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
            if (j < BMT) sm.scale[si][j] = v[i][q] * c[i];
          }
          mbar_arrive(&sm.sc_full[si]);
        }
      }
    }
  } else {
    // consumers (warps 2..5)
    const int lg = warp & 3;
    const uint32_t t_lane = static_cast<uint32_t>(lg * 32) << 16;
    int buf = 0, si = 0;
    uint32_t bphase = 0, sphase = 0;
    for (int i = 0; i < nkb; ++i) {
      if (!warp_wait(&sm.sc_full[si], sphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitScaleFull) ||
          !warp_wait(&sm.acc_full[buf], bphase, abort, p.err, kErrTimeout | kRoleConsumer | kWaitAccFull)) {
        consumer_ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem + t_lane + static_cast<uint32_t>(buf) * ACC_COLS;
      const float4* s4 = reinterpret_cast<const float4*>(sm.scale[si]);
      constexpr int CH = BMT < 32 ? BMT : 32;  // columns per TMEM load
#pragma unroll
      for (int c = 0; c < BMT / CH; ++c) {
        uint32_t r[CH];
        if constexpr (CH == 16) {
          tmem_ld16(tb + c * CH, r);
        } else {
          tmem_ld32(tb + c * CH, r);
        }
#pragma unroll
        for (int q = 0; q < CH / 4; ++q) {
          const float4 s = s4[c * (CH / 4) + q];
          const int j = c * CH + 4 * q;
          acc[j + 0] = fmaf(s.x, __uint_as_float(r[4 * q + 0]), acc[j + 0]);
          acc[j + 1] = fmaf(s.y, __uint_as_float(r[4 * q + 1]), acc[j + 1]);
          acc[j + 2] = fmaf(s.z, __uint_as_float(r[4 * q + 2]), acc[j + 2]);
          acc[j + 3] = fmaf(s.w, __uint_as_float(r[4 * q + 3]), acc[j + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.acc_empty[buf]);
        mbar_arrive(&sm.sc_empty[si]);
      }
      buf ^= 1;
      if (buf == 0) bphase ^= 1u;
      if (++si == SSTAGES) {
        si = 0;
        sphase ^= 1u;
      }
    }
  }

  // --------------------------------------------------------------- epilogue
  const bool is_consumer = warp >= 2 && warp <= 5;
  const int ctid = threadIdx.x - 64;            // 0..127 for consumers (work index)
  const int wrow = (warp & 3) * 32 + lane;      // consumer's weight row = its TMEM lane
  char* outb = static_cast<char*>(o.out);
  if (S == 1) {
    if (is_consumer && consumer_ok) {
      const int n = n0 + wrow;
      if (n < p.N) {
#pragma unroll
        for (int j = 0; j < BMT; ++j) {
          const int m = m0 + j;
          if (m < p.M)
            store_out<OutT>(reinterpret_cast<OutT*>(outb) + static_cast<long long>(m) * o.o_sm +
                                static_cast<long long>(g) * o.o_sg + n,
                            acc[j]);
        }
      }
    }
  } else {
    // every consumer publishes its partial column-major: red[j][row]
    float* red = reinterpret_cast<float*>(&sm.b[0][0]);
    if (is_consumer) {
#pragma unroll
      for (int j = 0; j < BMT; ++j) red[j * 128 + wrow] = consumer_ok ? acc[j] : 0.f;
    }
    cluster_sync_all();
    if (is_consumer) {
      const int R = 128 / S;  // weight rows reduced by this CTA
      const int per = (R * BMT) / 128;
      const uint32_t red_s = smem_u32(red);
      for (int it = 0; it < per; ++it) {
        const int idx = ctid + 128 * it;
        const int r = rank * R + idx % R;
        const int j = idx / R;
        const uint32_t off = red_s + static_cast<uint32_t>((j * 128 + r) * 4);
        float v = ld_shared_cluster_f32(mapa_shared(off, 0));
        for (int q = 1; q < S; ++q) v += ld_shared_cluster_f32(mapa_shared(off, static_cast<uint32_t>(q)));
        const int n = n0 + r, m = m0 + j;
        if (n < p.N && m < p.M)
          store_out<OutT>(reinterpret_cast<OutT*>(outb) + static_cast<long long>(m) * o.o_sm +
                              static_cast<long long>(g) * o.o_sg + n,
                          v);
      }
    }
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace bsg

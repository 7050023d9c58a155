// Small-M FP8 block-scaled GEMM (M <= 8): a weight stream at HBM speed.
//
// With one to eight activation rows the operation is a matrix-vector
// product: every weight byte is read once and used M times, so the time is
// the weight stream plus the fixed latency of a launch.  The tcgen05 skinny
// kernel pays for its 128-row MMA tiles in TMEM round trips and a cluster
// reduction; this kernel instead keeps everything in registers and uses the
// warp-level e4m3 MMA (mma.sync m16n8k32, fp32 accumulate) as the fp8
// multiplier, so no e4m3 value is ever decoded on the CUDA cores.
//
// A CTA of 8 warps owns 16 weight rows (output columns n0 .. n0+15) of one
// batch; its warps split the K blocks into 8 contiguous ranges, and each warp
// has the loads of KBS K blocks in flight before its MMAs: one for grids of
// more than two CTAs per SM, two for grids of up to two, four for grids of at
// most one CTA per SM (small grids need more bytes in flight per CTA).  Per 64-deep
// K group a thread loads 16 contiguous bytes of weight rows g and g+8
// (g = lane / 4) and 16 bytes of activation row lane / 4 at the same K
// offset (lane % 4) * 16, and issues two MMAs: the dot product does not care
// in which order K is summed, so A and B only need the same K permutation,
// and every load stays a 16-byte vector.  After each 128-deep block the
// fp32 partial is promoted with its block scale (scale_a[m, kb] *
// scale_b[kb, nb], or the two e8m0 powers of two); the 8 warps' sums meet in
// shared memory and are added in warp order (deterministic).
//   Sources: pytorch issue "torch._scaled_mm with blockwise scaling doesn't
//   work with torch.compile" (1x128 / 128x128 scale shapes); ROCm/aiter PR
//   "Add opus fp8 mxscale BMM kernels for gfx950" (batched m-major layout,
//   e8m0 scales, m = 1 .. 16 among its test sizes).  From 9 to 16 rows the
//   tcgen05 skinny kernel measured faster (16 activation rows, eight batches
//   of a 1024 x 4096 weight: 11.4 against 20.3 us), so this kernel stops at 8.
#include <cuda_bf16.h>

#include "launch.h"

namespace bsg {

namespace {

constexpr int kGemvRows = 16;  // weight rows (output columns) per CTA
constexpr int kGemvWarps = 8;  // warps per CTA, splitting K

__device__ __forceinline__ void mma_e4m3_16x8x32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Output element (m, g, n) at out[m * o_sm + g * o_sg + n].  KBS = 1 keeps a
// thread at 64 registers, so four CTAs share an SM and the grid of a 7168-row
// weight (448 CTAs) or of eight 1024-row batches (512) runs in one wave;
// KBS = 2 (two CTAs per SM) and KBS = 4 (one) serve the smaller grids.
template <Mode MODE, int KBS, typename OutT>
__global__ void __launch_bounds__(kGemvWarps * 32, KBS == 1 ? 4 : (KBS == 2 ? 2 : 1))
    gemv_kernel(const uint8_t* __restrict__ A, long long a_sm, long long a_sg, const uint8_t* __restrict__ B,
                long long b_sn, long long b_sg, const GemmArgs p, void* out, long long o_sm, long long o_sg) {
  constexpr int NT = 1;  // one 8-wide activation tile: M <= 8
  __shared__ float red[kGemvWarps][NT][kGemvRows][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int n0 = blockIdx.x * kGemvRows;
  const int nb = n0 >> 7;  // the 16 rows lie in one 128-row scale block
  const int gr = lane >> 2, t = lane & 3;
  // this warp's K blocks
  const int kb_lo = (p.KB * warp) / kGemvWarps, kb_hi = (p.KB * (warp + 1)) / kGemvWarps;

  grid_dependency_wait();  // inputs may come from the previous kernel in the stream
  grid_launch_dependents();

  // weight rows g and g + 8 of the tile (rows past N read as zero), activation
  // rows gr + 8 j (rows past M read as zero)
  const int r0 = n0 + gr, r1 = n0 + gr + 8;
  const uint8_t* w0 = B + static_cast<long long>(g) * b_sg + static_cast<long long>(r0) * b_sn + 16 * t;
  const uint8_t* w1 = B + static_cast<long long>(g) * b_sg + static_cast<long long>(r1) * b_sn + 16 * t;
  const bool ok0 = r0 < p.N, ok1 = r1 < p.N;
  const uint8_t* xa[NT];
  bool oka[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int m = gr + 8 * j;
    oka[j] = m < p.M;
    xa[j] = A + static_cast<long long>(m) * a_sm + static_cast<long long>(g) * a_sg + 16 * t;
  }

  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;

  // KBS K blocks per step: their operand and block-scale loads all in flight
  // before the MMAs (a scale loaded after the MMAs would add its latency to
  // every step)
  for (int kb0 = kb_lo; kb0 < kb_hi; kb0 += KBS) {
    uint4 wa[KBS][2], wb[KBS][2], xv[KBS][2][NT];
    float sbk[KBS], sam[KBS][2];  // the block's weight scale; activation rows 2t, 2t + 1
#pragma unroll
    for (int u = 0; u < KBS; ++u) {
      const int kb = kb0 + u;
      const bool in = kb < kb_hi;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const long long k = static_cast<long long>(kb) * 128 + 64 * h;
        wa[u][h] = in && ok0 ? __ldg(reinterpret_cast<const uint4*>(w0 + k)) : make_uint4(0, 0, 0, 0);
        wb[u][h] = in && ok1 ? __ldg(reinterpret_cast<const uint4*>(w1 + k)) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < NT; ++j)
          xv[u][h][j] = in && oka[j] ? __ldg(reinterpret_cast<const uint4*>(xa[j] + k)) : make_uint4(0, 0, 0, 0);
      }
      if constexpr (MODE == Mode::kFp8F32Scale) {
        sbk[u] = in && nb < p.NB ? __ldg(p.sb + static_cast<long long>(kb) * p.sb_sk + static_cast<long long>(nb) * p.sb_sn)
                                 : 0.f;
      } else {
        sbk[u] = in && nb < p.NB ? e8m0_to_f32(__ldg(p.ws + (static_cast<long long>(g) * p.NB + nb) * p.KB + kb)) : 0.f;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int m = 2 * t + c;
        float v = 0.f;
        if (in && m < p.M) {
          if constexpr (MODE == Mode::kFp8F32Scale) {
            v = __ldg(p.sa + static_cast<long long>(m) * p.sa_sm + static_cast<long long>(kb) * p.sa_sk);
          } else {
            v = e8m0_to_f32(__ldg(p.xs + (static_cast<long long>(m) * p.G + g) * p.KB + kb));
          }
        }
        sam[u][c] = v;
      }
    }
#pragma unroll
    for (int u = 0; u < KBS; ++u) {
      const int kb = kb0 + u;
      if (kb >= kb_hi) break;
      float part[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) part[j][i] = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // bytes 0-7 of each 16-byte piece feed the first MMA, bytes 8-15 the
        // second; in each, the fragment's K columns 4t.. and 4t+16.. are the
        // piece's first and second 4 bytes
        const uint32_t lo[4] = {wa[u][h].x, wb[u][h].x, wa[u][h].y, wb[u][h].y};
        const uint32_t hi[4] = {wa[u][h].z, wb[u][h].z, wa[u][h].w, wb[u][h].w};
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          mma_e4m3_16x8x32(part[j], lo, xv[u][h][j].x, xv[u][h][j].y);
          mma_e4m3_16x8x32(part[j], hi, xv[u][h][j].z, xv[u][h][j].w);
        }
      }
      // promotion: part[0][i] is row (gr or gr + 8) x activation row
      // m = 2 t + (i & 1) of this block's partial
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float s = sam[u][c] * sbk[u];
        acc[0][c] = fmaf(s, part[0][c], acc[0][c]);
        acc[0][2 + c] = fmaf(s, part[0][2 + c], acc[0][2 + c]);
      }
    }
  }

  // the 8 warps' partial sums, added in warp order
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    red[warp][j][gr][2 * t] = acc[j][0];
    red[warp][j][gr][2 * t + 1] = acc[j][1];
    red[warp][j][gr + 8][2 * t] = acc[j][2];
    red[warp][j][gr + 8][2 * t + 1] = acc[j][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NT * kGemvRows * 8; i += kGemvWarps * 32) {
    const int j = i / (kGemvRows * 8), row = (i / 8) % kGemvRows, c = i % 8;
    const int m = 8 * j + c, n = n0 + row;
    if (m < p.M && n < p.N) {
      float s = red[0][j][row][c];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) s += red[w][j][row][c];
      OutT* dst = static_cast<OutT*>(out) + static_cast<long long>(m) * o_sm + static_cast<long long>(g) * o_sg + n;
      if constexpr (sizeof(OutT) == 2) {
        *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(s);
      } else {
        *reinterpret_cast<float*>(dst) = s;
      }
    }
  }
}

template <Mode MODE, int KBS, typename OutT>
cudaError_t launch_kbs(const GemvProblem& q, const GemmArgs& args, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  // programmatic dependent launch: the prologue may overlap the previous kernel
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((args.N + kGemvRows - 1) / kGemvRows), static_cast<unsigned>(args.G), 1);
  cfg.blockDim = dim3(kGemvWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<MODE, KBS, OutT>, static_cast<const uint8_t*>(q.a), q.a_sm, q.a_sg,
                            static_cast<const uint8_t*>(q.b), q.b_sn, q.b_sg, args, q.out, q.o_sm, q.o_sg);
}

template <Mode MODE, typename OutT>
cudaError_t launch_mode(const GemvProblem& q, const GemmArgs& args, cudaStream_t stream) {
  const long long ctas = static_cast<long long>((args.N + kGemvRows - 1) / kGemvRows) * args.G;
  if (ctas <= q.sms) return launch_kbs<MODE, 4, OutT>(q, args, stream);
  return ctas <= 2LL * q.sms ? launch_kbs<MODE, 2, OutT>(q, args, stream) : launch_kbs<MODE, 1, OutT>(q, args, stream);
}

}  // namespace

cudaError_t launch_gemv(Mode mode, OutKind out, const GemvProblem& q, const GemmArgs& args, cudaStream_t stream) {
  if (args.M > kGemvMaxM) return cudaErrorInvalidValue;
  if (mode == Mode::kFp8F32Scale) {
    if (out == OutKind::kBF16) return launch_mode<Mode::kFp8F32Scale, __nv_bfloat16>(q, args, stream);
    if (out == OutKind::kF32) return launch_mode<Mode::kFp8F32Scale, float>(q, args, stream);
  } else if (mode == Mode::kFp8E8M0) {
    if (out == OutKind::kBF16) return launch_mode<Mode::kFp8E8M0, __nv_bfloat16>(q, args, stream);
    if (out == OutKind::kF32) return launch_mode<Mode::kFp8E8M0, float>(q, args, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace bsg

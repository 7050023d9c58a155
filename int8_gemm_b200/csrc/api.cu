// C-ABI layer: argument validation, kernel planning, tensor-map encoding and
// launches.  All heavy work happens in the sm_100a kernels; nothing here
// computes a GEMM result, and there is no fallback path.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda_fp8.h>

#include "bsgemm.h"
#include "launch.h"
#include "quantize.h"

using namespace bsg;

// Per-device error word written by kernels whose bounded waits give up.
__device__ uint32_t g_bs_error_word = 0;

namespace {

// ---------------------------------------------------------------------------
// error reporting
// ---------------------------------------------------------------------------
thread_local char g_msg[512] = {0};

bs_status fail(bs_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

void clear_msg() { g_msg[0] = 0; }

// ---------------------------------------------------------------------------
// driver entry point for tensor-map encoding (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// ---------------------------------------------------------------------------
// per-device facts
// ---------------------------------------------------------------------------
// `ready` is published with release order after the other fields are written,
// and read with acquire order, so a thread that sees it set also sees them.
struct DeviceCtx {
  int sms = 0;
  uint32_t* err = nullptr;
  std::atomic<bool> ready{false};
  bs_status status = BS_OK;
  // stream-K workspace registered with bs_set_workspace (caller-owned)
  std::atomic<void*> ws{nullptr};
  std::atomic<size_t> ws_bytes{0};
  // built-in scratch of bs_int_scaled_mm_noalloc, looked up on its first call
  std::atomic<void*> scratch{nullptr};
};

constexpr int kMaxDevices = 64;
DeviceCtx g_dev[kMaxDevices];
std::mutex g_dev_mu;

bs_status device_ctx(DeviceCtx** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(BS_ERR_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(BS_ERR_DEVICE, "device index %d out of range", dev);
  DeviceCtx& d = g_dev[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!d.ready.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (major != 10 || minor != 0) {
        d.status = BS_ERR_DEVICE;
      } else {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_bs_error_word);
        if (e != cudaSuccess) {
          d.status = BS_ERR_CUDA;
        } else {
          d.err = static_cast<uint32_t*>(p);
          d.sms = sms;
          d.status = BS_OK;
        }
      }
      d.ready.store(true, std::memory_order_release);
    }
  }
  if (d.status == BS_ERR_DEVICE) return fail(BS_ERR_DEVICE, "device %d is not an sm_100 GPU", dev);
  if (d.status != BS_OK) return fail(d.status, "device %d setup failed", dev);
  *out = &d;
  return BS_OK;
}

// ---------------------------------------------------------------------------
// planning (pure host logic)
// ---------------------------------------------------------------------------
std::atomic<int32_t> g_path_override{0};
std::atomic<int32_t> g_stream_k{0};  // stream-K split: off unless enabled
std::atomic<int32_t> g_split_override{0};  // skinny kernel: forced split factor (0 = planner's choice)

// Bytes of the stream-K workspace for a GPU with `sms` SMs: one partial-sum
// slot per CTA (the 128 x 256 fp32 accumulator, 128 KB) and one flag word per
// slot and consumer warp, the flags after the slots.
size_t workspace_slots_bytes(int sms) { return static_cast<size_t>(sms) * kWsSlotWords * sizeof(uint32_t); }
size_t workspace_bytes_for(int sms) {
  const size_t flags = static_cast<size_t>(sms) * kWsFlagsPerSlot * sizeof(uint32_t);
  return workspace_slots_bytes(sms) + ((flags + 255) / 256) * 256;
}

constexpr int kSkinnyMaxM = 256;

// CTAs of the skinny kernel that fit on one SM (shared memory of the operand
// ring, and registers of the BMT accumulators per consumer thread).
int skinny_ctas_per_sm(int bmt) {
  return bmt <= 16 ? SkinnyCfg<16>::CTAS_PER_SM
                   : (bmt <= 32 ? SkinnyCfg<32>::CTAS_PER_SM
                                : (bmt <= 64 ? SkinnyCfg<64>::CTAS_PER_SM : SkinnyCfg<128>::CTAS_PER_SM));
}
constexpr int kGroupM = 16;

struct Plan {
  bs_plan pub;
  int cg = 2;  // wide kernel: CTAs per tile (2 = CTA pair, 256-row tiles)
  int bmt = 0;
  int m_tiles = 0, n_tiles = 0;
  int grid_m = 0, grid_n = 0, num_tiles = 0;
  int dp_tiles = 0;        // wide kernel: tiles computed whole
  long long sk_iters = 0;  // K blocks of the remaining tiles, split evenly over the units
};

// Stream-K split of the wide kernel's persistent loop (tile_order.h): when
// the tiles leave the last round of units badly filled, that round's K
// blocks (and, if that leaves fewer than kSkMinPerUnit per unit, one more
// round's) are spread evenly over every unit.  Each unit then hands over at
// most one partial sum and finishes at most one split tile.
constexpr double kSkMinFill = 0.9;  // below this fraction of busy unit-rounds, split
constexpr int kSkMinPerUnit = 4;    // K blocks per unit, at least
void plan_stream_k(Plan& x, long long tiles, long long units, int KB) {
  x.dp_tiles = static_cast<int>(tiles);
  x.sk_iters = 0;
  if (units <= 1 || KB < 2) return;
  const long long full = tiles / units, rem = tiles % units;
  if (rem == 0) return;
  const double fill = static_cast<double>(tiles) / static_cast<double>((full + 1) * units);
  if (fill >= kSkMinFill) return;
  long long dp = full * units;
  if ((tiles - dp) * KB < kSkMinPerUnit * units && full >= 1) dp -= units;
  const long long iters = (tiles - dp) * KB;
  if (iters < kSkMinPerUnit * units) return;
  x.dp_tiles = static_cast<int>(dp);
  x.sk_iters = iters;
  x.pub.sk_tiles = static_cast<int32_t>(tiles - dp);
}

// stream_k_ok: a workspace for the split is at hand; force_split: apply the
// split rule even while bs_set_stream_k is off.
Plan make_plan(int op, int64_t M, int64_t G, int64_t N, int64_t K, int sms, bool stream_k_ok,
               bool force_split = false) {
  Plan x;
  std::memset(&x.pub, 0, sizeof(x.pub));
  if (M == 0 || N == 0 || G == 0) return x;  // kernel 0: nothing to do
  if (K == 0) {
    x.pub.kernel = 3;
    x.pub.launches = 1;
    x.pub.splits = 1;
    x.pub.cluster = 1;
    x.pub.ctas = sms > 0 ? 2 * sms : 1;
    return x;
  }
  const int KB = static_cast<int>((K + 127) / 128);
  const int ov = g_path_override.load();
  const bool skinny_ok = op == 1 || op == 3;  // block-scaled FP8 only
  // M <= kGemvMaxM: the warp-MMA weight stream (kernels_gemv.cu)
  if (skinny_ok && M <= kGemvMaxM && (ov == 5 || ov == 0)) {
    x.pub.kernel = 4;
    x.pub.tile_m = 8;
    x.pub.tile_n = 16;
    x.pub.splits = 1;
    x.pub.cluster = 1;
    x.pub.ctas = static_cast<int32_t>(((N + 15) / 16) * G);
    x.pub.launches = 1;
    return x;
  }
  const bool skinny = skinny_ok && (ov == 2 || (ov == 0 && M <= kSkinnyMaxM));
  if (skinny) {
    const long long n_tiles = (N + 127) / 128;
    const long long sm_count = sms > 0 ? sms : 148;
    int bmt = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    // Each CTA issues its K blocks' MMAs as one serial chain, so for long K
    // (32 or more blocks) two co-resident CTAs per SM -- possible only for
    // activation tiles of at most 32 rows -- beat one wider tile per SM, as
    // long as the grid of 32-row tiles is still resident in one wave.
    if (bmt > 32 && KB >= 32 &&
        ((M + 31) / 32) * n_tiles * G <= static_cast<long long>(skinny_ctas_per_sm(32)) * sm_count)
      bmt = 32;
    x.bmt = bmt;
    x.m_tiles = static_cast<int>((M + bmt - 1) / bmt);
    x.n_tiles = static_cast<int>(n_tiles);
    const long long units = static_cast<long long>(x.m_tiles) * x.n_tiles * G;
    // Split K over a cluster of S CTAs only as far as every CTA stays resident
    // at once (a second partial wave would double the time of an HBM-bound
    // stream), S a power of two <= 8 and <= the number of K blocks.
    const long long slots = static_cast<long long>(skinny_ctas_per_sm(bmt)) * sm_count;
    // Clusters of 8 CTAs that each fill an SM do not all fit in the GPCs at
    // once, so those kernels split at most 4 ways.
    const int max_s = skinny_ctas_per_sm(bmt) > 1 ? 8 : 4;
    int S = 1;
    while (S < max_s && 2 * S <= KB && units * 2 * S <= slots) S *= 2;
    // With 32-row or wider activation tiles, a CTA holding fewer than 8 K
    // blocks spends more on its fixed costs than the extra CTAs gain, while
    // the halved grid still has half as many CTAs as SMs (measured: M=32,
    // N=7168, K=2048 takes 6.7 us split 2 ways against 7.2 us 4 ways).
    while (bmt >= 32 && S > 1 && KB / S < 8 && units * (S / 2) >= sm_count / 2) S /= 2;
    const int forced = g_split_override.load();
    if (forced == 1 || forced == 2 || forced == 4 || forced == 8) S = forced <= KB ? forced : S;
    x.pub.kernel = 2;
    x.pub.tile_m = bmt;
    x.pub.tile_n = 128;
    x.pub.splits = S;
    x.pub.cluster = S;
    x.pub.ctas = static_cast<int32_t>(units * S);
    x.pub.launches = 1;
  } else {
    x.cg = ov == 3 ? 1 : 2;
    const int tile_m = 128 * x.cg;
    x.grid_m = static_cast<int>((M + tile_m - 1) / tile_m);
    x.grid_n = static_cast<int>((N + kWideBN - 1) / kWideBN);
    const long long tiles = static_cast<long long>(x.grid_m) * x.grid_n * G;
    const long long units = (sms > 0 ? sms : 148) / x.cg;  // persistent CTAs (or CTA pairs)
    x.num_tiles = static_cast<int>(tiles);
    x.dp_tiles = x.num_tiles;
    if (stream_k_ok && (force_split || g_stream_k.load() != 0)) plan_stream_k(x, tiles, units, KB);
    x.pub.kernel = 1;
    x.pub.tile_m = tile_m;
    x.pub.tile_n = kWideBN;
    x.pub.splits = 1;
    x.pub.cluster = x.cg;
    // a split plan keeps every unit busy; otherwise no more units than tiles
    x.pub.ctas = static_cast<int32_t>(x.cg * (x.sk_iters > 0 || tiles > units ? units : tiles));
    x.pub.launches = 1;
  }
  return x;
}

// A registered workspace large enough for this device's stream-K slots.
bool workspace_ok(const DeviceCtx* dc) {
  return dc->ws.load() != nullptr && dc->ws_bytes.load() >= workspace_bytes_for(dc->sms);
}

// The persistent loop's split (whole tiles, stream-K blocks) and, for a split
// plan, the workspace slots and flags of this device.
void set_work_split(GemmArgs& a, const Plan& pl, const DeviceCtx* dc) {
  a.dp_tiles = pl.dp_tiles;
  a.sk_iters = pl.sk_iters;
  if (pl.sk_iters > 0) {
    uint8_t* base = static_cast<uint8_t*>(dc->ws.load());
    a.sk_ws = reinterpret_cast<uint32_t*>(base);
    a.sk_flags = reinterpret_cast<uint32_t*>(base + workspace_slots_bytes(dc->sms));
  }
}

// ---------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------
bs_status encode_3d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, uint64_t d0, uint64_t d1,
                    uint64_t d2, uint64_t s1, uint64_t s2, uint32_t box0, uint32_t box1, const char* what,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(BS_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1 * static_cast<uint64_t>(esize), s2 * static_cast<uint64_t>(esize)};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(BS_ERR_CUDA, "tensor map encoding failed for %s (CUresult %d)", what, static_cast<int>(r));
  return BS_OK;
}

// Tensor maps of a quantiser's input x and codes q, both [R, C] in their own
// orientation (128 x 128 boxes; x without swizzle, q with the 128-byte
// swizzle of the kernels' code tiles), for the TMA-fed kernels; `tma`
// is false (and nothing is encoded) unless x and q have 16-byte bases and row
// strides and C is a multiple of 16, so that no row ends inside a 16-byte
// piece.
bs_status encode_quant_maps(const void* x, bs_in_dtype x_dtype, int64_t R, int64_t C, int64_t ldx, const void* q,
                            int64_t ldq, CUtensorMap* tmx, CUtensorMap* tmq, bool* tma) {
  const int es = x_dtype == BS_IN_BF16 ? 2 : 4;
  *tma = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (ldx * es) % 16 == 0 && C % 16 == 0 &&
         (reinterpret_cast<uintptr_t>(q) & 15u) == 0 && ldq % 16 == 0;
  if (!*tma) return BS_OK;
  const CUtensorMapDataType xt =
      x_dtype == BS_IN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  bs_status st = encode_3d(tmx, xt, es, x, static_cast<uint64_t>(C), static_cast<uint64_t>(R), 1,
                           static_cast<uint64_t>(ldx), static_cast<uint64_t>(ldx) * static_cast<uint64_t>(R), 128, 128,
                           "x", CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != BS_OK) return st;
  return encode_3d(tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q, static_cast<uint64_t>(C), static_cast<uint64_t>(R), 1,
                   static_cast<uint64_t>(ldq), static_cast<uint64_t>(ldq) * static_cast<uint64_t>(R), 128, 128, "q",
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

// Rows of one B box of the wide kernel: single CTAs load all 256 tile columns,
// each CTA of a pair its 128.
uint32_t wide_b_box_rows(int cg) { return static_cast<uint32_t>(kWideBN / cg); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int out_size(bs_out_dtype t) { return t == BS_OUT_E4M3 ? 1 : (t == BS_OUT_BF16 ? 2 : 4); }

CUtensorMapDataType out_tmap_type(bs_out_dtype t) {
  if (t == BS_OUT_E4M3) return CU_TENSOR_MAP_DATA_TYPE_UINT8;
  return t == BS_OUT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                          : (t == BS_OUT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_INT32);
}

OutKind out_kind(bs_out_dtype t) {
  if (t == BS_OUT_E4M3) return OutKind::kE4M3;
  return t == BS_OUT_BF16 ? OutKind::kBF16 : (t == BS_OUT_F32 ? OutKind::kF32 : OutKind::kI32);
}

constexpr int64_t kMaxDim = 0x7FFFFFFF;

bs_status check_launch(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(BS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  e = cudaPeekAtLastError();
  if (e != cudaSuccess) return fail(BS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return BS_OK;
}

// Shared launch of the FP8 paths (operations 1 and 3).  Coordinates of the
// three-dimensional tensor maps are (k, row, batch) for operands and
// (n, m, batch) for the output.
struct Fp8Problem {
  const void* a;
  int64_t a_rs, a_bs;  // row and batch strides of A (bytes)
  const void* b;
  int64_t b_rs, b_bs;  // row (= output column) and batch strides of B (bytes)
  void* out;
  int64_t o_rs, o_bs;  // row and batch strides of out (elements)
  bs_out_dtype out_dtype;
  int64_t M, G, N, K;
  Mode mode;
};

bs_status run_fp8(const Fp8Problem& q, GemmArgs args, cudaStream_t stream, DeviceCtx* dc) {
  const Plan pl = make_plan(q.mode == Mode::kFp8E8M0 ? 3 : 1, q.M, q.G, q.N, q.K, dc->sms, workspace_ok(dc));
  if (pl.pub.kernel == 0) return BS_OK;
  if (pl.pub.kernel == 3)
    return check_launch(launch_fill_zero(q.out, out_size(q.out_dtype), q.M, q.N, q.o_rs, q.G, q.o_bs, stream),
                        "zero-fill launch");
  if (pl.pub.kernel == 4) {
    args.err = dc->err;
    GemvProblem gq;
    gq.a = q.a;
    gq.a_sm = q.a_rs;
    gq.a_sg = q.G > 1 ? q.a_bs : 0;
    gq.b = q.b;
    gq.b_sn = q.b_rs;
    gq.b_sg = q.G > 1 ? q.b_bs : 0;
    gq.out = q.out;
    gq.o_sm = q.o_rs;
    gq.o_sg = q.G > 1 ? q.o_bs : 0;
    gq.sms = dc->sms;
    return check_launch(launch_gemv(q.mode, out_kind(q.out_dtype), gq, args, stream), "small-M kernel launch");
  }
  args.err = dc->err;
  CUtensorMap ta, tb, td;
  const uint64_t a_bs = q.G > 1 ? static_cast<uint64_t>(q.a_bs) : static_cast<uint64_t>(q.a_rs) * q.M;
  const uint64_t b_bs = q.G > 1 ? static_cast<uint64_t>(q.b_bs) : static_cast<uint64_t>(q.b_rs) * q.N;
  const uint64_t o_bs = q.G > 1 ? static_cast<uint64_t>(q.o_bs) : static_cast<uint64_t>(q.o_rs) * q.M;
  bs_status st;
  if (pl.pub.kernel == 1) {
    args.grid_m = pl.grid_m;
    args.grid_n = pl.grid_n;
    args.num_tiles = pl.num_tiles;
    args.group_m = kGroupM;
    args.splits = 1;
    set_work_split(args, pl, dc);
    if ((st = encode_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.a, q.K, q.M, q.G, q.a_rs, a_bs, 128, 128, "A")))
      return st;
    if ((st = encode_3d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.b, q.K, q.N, q.G, q.b_rs, b_bs, 128,
                        wide_b_box_rows(pl.cg), "B")))
      return st;
    const int es = out_size(q.out_dtype);
    if ((st = encode_3d(&td, out_tmap_type(q.out_dtype), es, q.out, q.N, q.M, q.G, q.o_rs, o_bs,
                        static_cast<uint32_t>(64 / es), 32, "out", CU_TENSOR_MAP_SWIZZLE_64B)))
      return st;
    // e8m0 block scales on CTA pairs: applied by the tensor core (block-scaled
    // MMA) unless path 4 asks for the per-block promotion on the CUDA cores
    const Mode mode = q.mode == Mode::kFp8E8M0 && pl.cg == 2 && g_path_override.load() != 4 ? Mode::kFp8Mx : q.mode;
    return check_launch(launch_wide(mode, out_kind(q.out_dtype), pl.cg, ta, tb, td, args, pl.pub.ctas, stream),
                        "wide kernel launch");
  }
  args.splits = pl.pub.splits;
  if ((st = encode_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.a, q.K, q.M, q.G, q.a_rs, a_bs, 128,
                      static_cast<uint32_t>(pl.bmt), "A")))
    return st;
  if ((st = encode_3d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q.b, q.K, q.N, q.G, q.b_rs, b_bs, 128, 128, "B")))
    return st;
  SkinnyOut o;
  o.out = q.out;
  o.o_sm = q.o_rs;
  o.o_sg = q.o_bs;
  return check_launch(
      launch_skinny(q.mode, out_kind(q.out_dtype), pl.bmt, ta, tb, args, o, pl.n_tiles, pl.m_tiles, stream),
      "skinny kernel launch");
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* bs_status_string(bs_status s) {
  switch (s) {
    case BS_OK: return "BS_OK";
    case BS_ERR_NULL: return "BS_ERR_NULL";
    case BS_ERR_SHAPE: return "BS_ERR_SHAPE";
    case BS_ERR_LAYOUT: return "BS_ERR_LAYOUT";
    case BS_ERR_ALIGNMENT: return "BS_ERR_ALIGNMENT";
    case BS_ERR_DTYPE: return "BS_ERR_DTYPE";
    case BS_ERR_DEVICE: return "BS_ERR_DEVICE";
    case BS_ERR_CUDA: return "BS_ERR_CUDA";
    case BS_ERR_TIMEOUT: return "BS_ERR_TIMEOUT";
    case BS_ERR_WORKSPACE: return "BS_ERR_WORKSPACE";
  }
  return "BS_ERR_UNKNOWN";
}

const char* bs_last_error_message(void) { return g_msg; }

int32_t bs_version(void) { return 200; }  // 0.2.0: rowwise e4m3 output (scale_result), transposed quantiser

bs_status bs_check_blockwise_scale_shapes(int64_t M, int64_t N, int64_t K, int64_t sa_rows, int64_t sa_cols,
                                          int64_t sb_rows, int64_t sb_cols) {
  clear_msg();
  const int64_t KB = (K + 127) / 128, NB = (N + 127) / 128;
  if (sa_rows != M || sa_cols != KB || sb_rows != KB || sb_cols != NB)
    return fail(BS_ERR_SHAPE,
                "blockwise scaling needs scale_a of shape (%lld, %lld) [1x128 groups] and scale_b of shape "
                "(%lld, %lld) [128x128 blocks]; got scale_a (%lld, %lld) and scale_b (%lld, %lld)",
                (long long)M, (long long)KB, (long long)KB, (long long)NB, (long long)sa_rows, (long long)sa_cols,
                (long long)sb_rows, (long long)sb_cols);
  return BS_OK;
}

int32_t bs_set_path_override(int32_t path) { return g_path_override.exchange(path); }

int32_t bs_set_stream_k(int32_t enable) { return g_stream_k.exchange(enable != 0 ? 1 : 0); }

int32_t bs_set_split_override(int32_t splits) { return g_split_override.exchange(splits); }

size_t bs_workspace_size(int32_t num_sms) { return num_sms > 0 ? workspace_bytes_for(num_sms) : 0; }

bs_status bs_set_workspace(void* workspace, size_t bytes) {
  clear_msg();
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  if (workspace == nullptr) {
    dc->ws.store(nullptr);
    dc->ws_bytes.store(0);
    return BS_OK;
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(BS_ERR_ALIGNMENT, "the workspace must be 256-byte aligned");
  const size_t need = workspace_bytes_for(dc->sms);
  if (bytes < need)
    return fail(BS_ERR_WORKSPACE, "workspace of %zu bytes; this device needs %zu (bs_workspace_size)", bytes, need);
  dc->ws_bytes.store(0);
  dc->ws.store(workspace);
  dc->ws_bytes.store(bytes);
  return BS_OK;
}

int32_t bs_work_items(int32_t num_tiles, int32_t dp_tiles, int64_t sk_iters, int32_t kb, int32_t units, int32_t unit,
                      int32_t* out, int32_t capacity) {
  if (num_tiles < 0 || dp_tiles < 0 || dp_tiles > num_tiles || sk_iters < 0 || kb <= 0 || units <= 0 || unit < 0 ||
      unit >= units || (sk_iters > 0 && sk_iters != static_cast<int64_t>(num_tiles - dp_tiles) * kb))
    return -1;
  WorkIter it(unit, units, sk_iters);
  WorkItem w;
  int32_t n = 0;
  while (it.next(w, units, dp_tiles, kb)) {
    if (out && n < capacity) {
      out[3 * n + 0] = w.tile;
      out[3 * n + 1] = w.kb0;
      out[3 * n + 2] = w.kb1;
    }
    ++n;
  }
  return n;
}

bs_status bs_plan_for(int32_t op, int64_t M, int64_t G, int64_t N, int64_t K, int32_t num_sms, bs_plan* plan) {
  clear_msg();
  if (!plan) return fail(BS_ERR_NULL, "plan is NULL");
  if (op < 1 || op > 4) return fail(BS_ERR_SHAPE, "op must be 1, 2, 3 or 4");
  if (M < 0 || N < 0 || K < 0 || G < 0 || num_sms <= 0) return fail(BS_ERR_SHAPE, "negative size");
  *plan = make_plan(op, M, G, N, K, num_sms, true).pub;
  return BS_OK;
}

bs_status bs_tile_order(int32_t grid_m, int32_t grid_n, int32_t batches, int32_t group_m, int32_t* out,
                        int64_t count) {
  clear_msg();
  if (!out) return fail(BS_ERR_NULL, "out is NULL");
  if (grid_m <= 0 || grid_n <= 0 || batches <= 0 || group_m <= 0) return fail(BS_ERR_SHAPE, "bad grid");
  if (count > static_cast<int64_t>(grid_m) * grid_n * batches) return fail(BS_ERR_SHAPE, "count exceeds tiles");
  for (int64_t t = 0; t < count; ++t) {
    const TileCoord c = tile_coord(static_cast<int>(t), grid_m, grid_n, group_m);
    out[3 * t + 0] = c.g;
    out[3 * t + 1] = c.pm;
    out[3 * t + 2] = c.pn;
  }
  return BS_OK;
}

bs_status bs_get_device_error(void* stream, uint32_t* code) {
  clear_msg();
  if (code) *code = 0;
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(BS_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpy(&v, dc->err, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(BS_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
  if (v == 0) return BS_OK;
  const uint32_t zero = 0;
  e = cudaMemcpy(dc->err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail(BS_ERR_CUDA, "clear error word: %s", cudaGetErrorString(e));
  if (code) *code = v;
  return fail(BS_ERR_TIMEOUT, "a kernel wait timed out (code 0x%x)", v);
}

bs_status bs_gemm_fp8_blockwise(const void* A, int64_t lda, const void* B, int64_t ldb, const float* scale_a,
                                int64_t sa_sm, int64_t sa_sk, const float* scale_b, int64_t sb_sk, int64_t sb_sn,
                                void* out, int64_t ldo, bs_out_dtype out_dtype, int64_t M, int64_t N, int64_t K,
                                void* stream) {
  clear_msg();
  if (M < 0 || N < 0 || K < 0) return fail(BS_ERR_SHAPE, "negative size M=%lld N=%lld K=%lld", (long long)M,
                                           (long long)N, (long long)K);
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return fail(BS_ERR_SHAPE, "size exceeds 2^31-1");
  if (K % 128 != 0) return fail(BS_ERR_SHAPE, "K=%lld is not a multiple of 128 (one scale per 128-deep group)",
                                (long long)K);
  if (out_dtype != BS_OUT_BF16 && out_dtype != BS_OUT_F32)
    return fail(BS_ERR_DTYPE, "bs_gemm_fp8_blockwise writes bf16 or f32 only");
  if (M == 0 || N == 0) return BS_OK;
  if (!out) return fail(BS_ERR_NULL, "out is NULL");
  if (ldo < N) return fail(BS_ERR_LAYOUT, "ldo=%lld < N=%lld", (long long)ldo, (long long)N);
  if (!aligned16(out) || (ldo * out_size(out_dtype)) % 16 != 0)
    return fail(BS_ERR_ALIGNMENT, "out must be 16-byte aligned with a row stride that is a multiple of 16 bytes");
  if (K > 0) {
    if (!A || !B || !scale_a || !scale_b) return fail(BS_ERR_NULL, "A, B, scale_a and scale_b must be non-NULL");
    if (lda < K || ldb < K) return fail(BS_ERR_LAYOUT, "lda/ldb must be >= K (A row-major, B column-major)");
    if (!aligned16(A) || !aligned16(B) || lda % 16 != 0 || ldb % 16 != 0)
      return fail(BS_ERR_ALIGNMENT, "A and B must be 16-byte aligned with lda, ldb multiples of 16");
    if (!aligned4(scale_a) || !aligned4(scale_b)) return fail(BS_ERR_ALIGNMENT, "scales must be 4-byte aligned");
    if (sa_sm < 0 || sa_sk < 0 || sb_sk < 0 || sb_sn < 0) return fail(BS_ERR_LAYOUT, "negative scale stride");
  }
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;

  GemmArgs args;
  std::memset(&args, 0, sizeof(args));
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.G = 1;
  args.KB = static_cast<int>(K / 128);
  args.NB = static_cast<int>((N + 127) / 128);
  args.sa = scale_a;
  args.sa_sm = sa_sm;
  args.sa_sk = sa_sk;
  args.sb = scale_b;
  args.sb_sk = sb_sk;
  args.sb_sn = sb_sn;
  Fp8Problem q{A, lda, 0, B, ldb, 0, out, ldo, 0, out_dtype, M, 1, N, K, Mode::kFp8F32Scale};
  return run_fp8(q, args, static_cast<cudaStream_t>(stream), dc);
}

bs_status bmm_a8w8_blockscale(const void* x, int64_t x_sm, int64_t x_sg, const void* w, int64_t w_sg, int64_t w_sn,
                              const uint8_t* x_scale, const uint8_t* w_scale, void* out, int64_t o_sm, int64_t o_sg,
                              bs_out_dtype out_dtype, int64_t M, int64_t G, int64_t N, int64_t K, void* stream) {
  clear_msg();
  if (M < 0 || N < 0 || K < 0 || G < 0) return fail(BS_ERR_SHAPE, "negative size");
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim || G > 65535) return fail(BS_ERR_SHAPE, "size out of range");
  if (K % 128 != 0) return fail(BS_ERR_SHAPE, "K=%lld is not a multiple of 128", (long long)K);
  if (out_dtype != BS_OUT_BF16 && out_dtype != BS_OUT_F32)
    return fail(BS_ERR_DTYPE, "bmm_a8w8_blockscale writes bf16 or f32 only");
  if (M == 0 || N == 0 || G == 0) return BS_OK;
  if (!out) return fail(BS_ERR_NULL, "out is NULL");
  const int es = out_size(out_dtype);
  if (o_sm < 0 || o_sg < 0) return fail(BS_ERR_LAYOUT, "negative output stride");
  if (!aligned16(out) || (o_sm * es) % 16 != 0 || (o_sg * es) % 16 != 0)
    return fail(BS_ERR_ALIGNMENT, "out must be 16-byte aligned with strides that are multiples of 16 bytes");
  if (K > 0) {
    if (!x || !w || !x_scale || !w_scale) return fail(BS_ERR_NULL, "x, w, x_scale and w_scale must be non-NULL");
    if (x_sm < 0 || x_sg < 0 || w_sg < 0 || w_sn < K) return fail(BS_ERR_LAYOUT, "bad x / w strides");
    if (!aligned16(x) || !aligned16(w) || x_sm % 16 || x_sg % 16 || w_sg % 16 || w_sn % 16)
      return fail(BS_ERR_ALIGNMENT, "x and w must be 16-byte aligned with strides that are multiples of 16");
  }
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;

  GemmArgs args;
  std::memset(&args, 0, sizeof(args));
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.G = static_cast<int>(G);
  args.KB = static_cast<int>(K / 128);
  args.NB = static_cast<int>((N + 127) / 128);
  args.xs = x_scale;
  args.ws = w_scale;
  Fp8Problem q{x, x_sm, x_sg, w, w_sn, w_sg, out, o_sm, o_sg, out_dtype, M, G, N, K, Mode::kFp8E8M0};
  return run_fp8(q, args, static_cast<cudaStream_t>(stream), dc);
}

bs_status bs_gemm_fp8_rowwise(const void* A, int64_t lda, const void* B, int64_t ldb, const float* scale_a,
                              int64_t sa_stride, const float* scale_b, int64_t sb_stride, const float* bias,
                              const float* scale_result, void* out, int64_t ldo, bs_out_dtype out_dtype, int64_t M,
                              int64_t N, int64_t K, void* stream) {
  clear_msg();
  if (M < 0 || N < 0 || K < 0) return fail(BS_ERR_SHAPE, "negative size");
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return fail(BS_ERR_SHAPE, "size exceeds 2^31-1");
  if (sa_stride != sb_stride || (sa_stride != 0 && sa_stride != 1))
    return fail(BS_ERR_SHAPE,
                "scales must be both tensorwise (strides 0: scalars) or both rowwise (strides 1: scale_a (M, 1), "
                "scale_b (1, N)); got strides %lld and %lld",
                (long long)sa_stride, (long long)sb_stride);
  if (out_dtype != BS_OUT_BF16 && out_dtype != BS_OUT_F32 && out_dtype != BS_OUT_E4M3)
    return fail(BS_ERR_DTYPE, "bs_gemm_fp8_rowwise writes bf16, f32 or e4m3 only");
  if (scale_result && out_dtype != BS_OUT_E4M3)
    return fail(BS_ERR_DTYPE, "scale_result applies to an e4m3 output only");
  if (M == 0 || N == 0) return BS_OK;
  if (!out) return fail(BS_ERR_NULL, "out is NULL");
  if (ldo < N) return fail(BS_ERR_LAYOUT, "ldo < N");
  if (!aligned16(out) || (ldo * out_size(out_dtype)) % 16 != 0)
    return fail(BS_ERR_ALIGNMENT, "out must be 16-byte aligned with a row stride that is a multiple of 16 bytes");
  if (bias && !aligned4(bias)) return fail(BS_ERR_ALIGNMENT, "bias must be 4-byte aligned");
  if (scale_result && !aligned4(scale_result)) return fail(BS_ERR_ALIGNMENT, "scale_result must be 4-byte aligned");
  if (K > 0) {
    if (!A || !B || !scale_a || !scale_b) return fail(BS_ERR_NULL, "A, B, scale_a and scale_b must be non-NULL");
    if (lda < K || ldb < K) return fail(BS_ERR_LAYOUT, "lda/ldb must be >= K (A row-major, B column-major)");
    if (!aligned16(A) || !aligned16(B) || lda % 16 != 0 || ldb % 16 != 0)
      return fail(BS_ERR_ALIGNMENT, "A and B must be 16-byte aligned with lda, ldb multiples of 16");
    if (!aligned4(scale_a) || !aligned4(scale_b)) return fail(BS_ERR_ALIGNMENT, "scales must be 4-byte aligned");
  }
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const Plan pl = make_plan(4, M, 1, N, K, dc->sms, workspace_ok(dc));
  if (pl.pub.kernel == 3)
    return check_launch(launch_fill_zero(out, out_size(out_dtype), M, N, ldo, 1, 0, cs, bias, scale_result),
                        "bias-fill launch");

  GemmArgs args;
  std::memset(&args, 0, sizeof(args));
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.G = 1;
  args.KB = static_cast<int>((K + 127) / 128);
  args.NB = static_cast<int>((N + 127) / 128);
  args.s_row = scale_a;
  args.s_col = scale_b;
  args.s_row_stride = sa_stride;
  args.s_col_stride = sb_stride;
  args.bias = bias;
  args.s_result = scale_result;
  args.grid_m = pl.grid_m;
  args.grid_n = pl.grid_n;
  args.num_tiles = pl.num_tiles;
  args.group_m = kGroupM;
  args.splits = 1;
  args.err = dc->err;
  set_work_split(args, pl, dc);
  CUtensorMap ta, tb, td;
  if ((st = encode_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, 1, lda, lda * M, 128, 128, "A"))) return st;
  if ((st = encode_3d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, 1, ldb, ldb * N, 128, wide_b_box_rows(pl.cg),
                      "B")))
    return st;
  const int es = out_size(out_dtype);
  if ((st = encode_3d(&td, out_tmap_type(out_dtype), es, out, N, M, 1, ldo, ldo * M, static_cast<uint32_t>(64 / es),
                      32, "out", CU_TENSOR_MAP_SWIZZLE_64B)))
    return st;
  return check_launch(launch_wide(Mode::kFp8Rowwise, out_kind(out_dtype), pl.cg, ta, tb, td, args, pl.pub.ctas, cs),
                      "fp8 rowwise kernel launch");
}

bs_status bs_quantize_fp8_1x128(const void* x, bs_in_dtype x_dtype, int64_t M, int64_t K, int64_t ldx, void* q,
                                int64_t ldq, void* scale, bs_scale_fmt scale_fmt, int64_t ld_scale, void* stream) {
  clear_msg();
  if (M < 0 || K < 0) return fail(BS_ERR_SHAPE, "negative size");
  if (M > kMaxDim || K > kMaxDim) return fail(BS_ERR_SHAPE, "size exceeds 2^31-1");
  if (x_dtype != BS_IN_BF16 && x_dtype != BS_IN_F32) return fail(BS_ERR_DTYPE, "x must be bf16 or f32");
  if (scale_fmt != BS_SCALE_F32 && scale_fmt != BS_SCALE_E8M0) return fail(BS_ERR_DTYPE, "unknown scale format");
  if (M == 0 || K == 0) return BS_OK;
  if (!x || !q || !scale) return fail(BS_ERR_NULL, "x, q and scale must be non-NULL");
  const int64_t KB = (K + 127) / 128;
  if (ldx < K || ldq < K || ld_scale < KB)
    return fail(BS_ERR_LAYOUT, "ldx and ldq must be >= K and ld_scale >= ceil(K/128) = %lld", (long long)KB);
  if (M * ((KB + 3) / 4) > kMaxDim) return fail(BS_ERR_SHAPE, "M * ceil(K/512) exceeds 2^31-1");
  const uintptr_t es = x_dtype == BS_IN_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(x) % es != 0) return fail(BS_ERR_ALIGNMENT, "x must be aligned to its element size");
  if (scale_fmt == BS_SCALE_F32 && !aligned4(scale))
    return fail(BS_ERR_ALIGNMENT, "fp32 scales must be 4-byte aligned");
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  CUtensorMap tmx, tmq;
  bool tma = false;
  if ((st = encode_quant_maps(x, x_dtype, M, K, ldx, q, ldq, &tmx, &tmq, &tma))) return st;
  return check_launch(launch_quantize_1x128(x, x_dtype == BS_IN_BF16, M, K, ldx, static_cast<uint8_t*>(q), ldq, scale,
                                            scale_fmt == BS_SCALE_E8M0, ld_scale, dc->sms, tma ? &tmx : nullptr,
                                            tma ? &tmq : nullptr, dc->err, static_cast<cudaStream_t>(stream)),
                      "quantise launch");
}

bs_status bs_quantize_fp8_t(const void* x, bs_in_dtype x_dtype, int64_t R, int64_t C, int64_t ldx, void* q_t,
                           int64_t ldq, void* scale, bs_scale_fmt scale_fmt, bs_group group, int64_t ld_scale,
                           void* stream) {
  clear_msg();
  if (R < 0 || C < 0) return fail(BS_ERR_SHAPE, "negative size");
  if (R > kMaxDim || C > kMaxDim) return fail(BS_ERR_SHAPE, "size exceeds 2^31-1");
  if (x_dtype != BS_IN_BF16 && x_dtype != BS_IN_F32) return fail(BS_ERR_DTYPE, "x must be bf16 or f32");
  if (scale_fmt != BS_SCALE_F32 && scale_fmt != BS_SCALE_E8M0) return fail(BS_ERR_DTYPE, "unknown scale format");
  if (group != BS_GROUP_128x1 && group != BS_GROUP_128x128) return fail(BS_ERR_SHAPE, "unknown group shape");
  if (R == 0 || C == 0) return BS_OK;
  if (!x || !q_t || !scale) return fail(BS_ERR_NULL, "x, q_t and scale must be non-NULL");
  const int64_t RB = (R + 127) / 128, CB = (C + 127) / 128;
  const int64_t min_lds = group == BS_GROUP_128x1 ? RB : CB;
  if (ldx < C || ldq < R || ld_scale < min_lds)
    return fail(BS_ERR_LAYOUT, "ldx must be >= C, ldq >= R and ld_scale >= %lld", (long long)min_lds);
  if (RB * CB > kMaxDim) return fail(BS_ERR_SHAPE, "more than 2^31-1 tiles of 128 x 128");
  const uintptr_t es = x_dtype == BS_IN_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(x) % es != 0) return fail(BS_ERR_ALIGNMENT, "x must be aligned to its element size");
  if (scale_fmt == BS_SCALE_F32 && !aligned4(scale))
    return fail(BS_ERR_ALIGNMENT, "fp32 scales must be 4-byte aligned");
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  // The TMA-fed kernel where x and q_t allow tensor copies: 16-byte bases and row strides, and rows whose
  // used bytes (C elements of x, R codes of q_t) end on a 16-byte boundary.  (A tensor store of a last row
  // tile that ended inside a 16-byte piece, R = 260, wrote bytes past R.)
  CUtensorMap tmx, tmq;
  const int64_t esz = static_cast<int64_t>(es);
  const bool tma = aligned16(x) && (ldx * esz) % 16 == 0 && (C * esz) % 16 == 0 && aligned16(q_t) && ldq % 16 == 0 &&
                   R % 16 == 0;
  if (tma) {
    st = encode_3d(&tmx, x_dtype == BS_IN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   static_cast<int>(es), x, static_cast<uint64_t>(C), static_cast<uint64_t>(R), 1,
                   static_cast<uint64_t>(ldx), static_cast<uint64_t>(ldx) * static_cast<uint64_t>(R), 128, 128, "x",
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != BS_OK) return st;
    st = encode_3d(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q_t, static_cast<uint64_t>(R), static_cast<uint64_t>(C), 1,
                   static_cast<uint64_t>(ldq), static_cast<uint64_t>(ldq) * static_cast<uint64_t>(C), 128, 128, "q_t",
                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != BS_OK) return st;
  }
  return check_launch(launch_quantize_t(x, x_dtype == BS_IN_BF16, R, C, ldx, static_cast<uint8_t*>(q_t), ldq, scale,
                                        scale_fmt == BS_SCALE_E8M0, group == BS_GROUP_128x128, ld_scale, dc->sms,
                                        tma ? &tmx : nullptr, tma ? &tmq : nullptr, dc->err,
                                        static_cast<cudaStream_t>(stream)),
                      "transposed quantise launch");
}

bs_status bs_quantize_fp8_128x128(const void* x, bs_in_dtype x_dtype, int64_t R, int64_t C, int64_t ldx, void* q,
                                  int64_t ldq, void* scale, bs_scale_fmt scale_fmt, int64_t s_rb, int64_t s_cb,
                                  void* stream) {
  clear_msg();
  if (R < 0 || C < 0) return fail(BS_ERR_SHAPE, "negative size");
  if (R > kMaxDim || C > kMaxDim) return fail(BS_ERR_SHAPE, "size exceeds 2^31-1");
  if (x_dtype != BS_IN_BF16 && x_dtype != BS_IN_F32) return fail(BS_ERR_DTYPE, "x must be bf16 or f32");
  if (scale_fmt != BS_SCALE_F32 && scale_fmt != BS_SCALE_E8M0) return fail(BS_ERR_DTYPE, "unknown scale format");
  if (R == 0 || C == 0) return BS_OK;
  if (!x || !q || !scale) return fail(BS_ERR_NULL, "x, q and scale must be non-NULL");
  const int64_t RB = (R + 127) / 128, CB = (C + 127) / 128;
  if (ldx < C || ldq < C) return fail(BS_ERR_LAYOUT, "ldx and ldq must be >= C");
  if (s_rb < 0 || s_cb < 0 || (RB > 1 && s_rb == 0) || (CB > 1 && s_cb == 0))
    return fail(BS_ERR_LAYOUT, "scale strides must be non-negative and non-zero along a dimension with several blocks");
  if (RB * CB > kMaxDim) return fail(BS_ERR_SHAPE, "more than 2^31-1 blocks of 128 x 128");
  const uintptr_t es = x_dtype == BS_IN_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(x) % es != 0) return fail(BS_ERR_ALIGNMENT, "x must be aligned to its element size");
  if (scale_fmt == BS_SCALE_F32 && !aligned4(scale))
    return fail(BS_ERR_ALIGNMENT, "fp32 scales must be 4-byte aligned");
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  CUtensorMap tmx, tmq;
  bool tma = false;
  if ((st = encode_quant_maps(x, x_dtype, R, C, ldx, q, ldq, &tmx, &tmq, &tma))) return st;
  return check_launch(launch_quantize_blocks(x, x_dtype == BS_IN_BF16, R, C, ldx, static_cast<uint8_t*>(q), ldq, scale,
                                             scale_fmt == BS_SCALE_E8M0, s_rb, s_cb, dc->sms, tma ? &tmx : nullptr,
                                             tma ? &tmq : nullptr, dc->err, static_cast<cudaStream_t>(stream)),
                      "block quantise launch");
}

}  // extern "C"

namespace {

// The address of the built-in scratch of bs_int_scaled_mm_noalloc on the
// current device, looked up once per device (this loads the scratch's module).
bs_status split_scratch(DeviceCtx* dc, void** out) {
  if (workspace_bytes_for(dc->sms) > kStaticScratchBytes)
    return fail(BS_ERR_WORKSPACE,
                "this device has %d SMs; the built-in scratch of bs_int_scaled_mm_noalloc holds the stream-K "
                "split of at most %d (%zu bytes)",
                dc->sms, kStaticScratchMaxSms, kStaticScratchBytes);
  void* p = dc->scratch.load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    p = dc->scratch.load(std::memory_order_relaxed);
    if (!p) {
      const cudaError_t e = static_scratch_address(&p);
      if (e != cudaSuccess || !p)
        return fail(BS_ERR_CUDA, "address of the built-in scratch: %s", cudaGetErrorString(e));
      dc->scratch.store(p, std::memory_order_release);
    }
  }
  *out = p;
  return BS_OK;
}

// int_scaled_mm on the wide kernel.  noalloc = false: the plan and workspace
// of int_scaled_mm (a split only while bs_set_stream_k is on and a workspace
// is registered); true: the split rule always applies, with the partials and
// flags in the built-in scratch, whose flag words are cleared on `stream`
// before the kernel.
bs_status int8_gemm(const int8_t* A, int64_t lda, const int8_t* B, int64_t ldb, const float* s_a, const float* s_b,
                    void* out, int64_t ldo, bs_out_dtype out_dtype, int64_t M, int64_t N, int64_t K, void* stream,
                    bool noalloc) {
  clear_msg();
  if (M < 0 || N < 0 || K < 0) return fail(BS_ERR_SHAPE, "negative size");
  if (M > kMaxDim || N > kMaxDim) return fail(BS_ERR_SHAPE, "size exceeds 2^31-1");
  if (K > 131071) return fail(BS_ERR_SHAPE, "K=%lld > 131071 could overflow the int32 accumulator", (long long)K);
  if (out_dtype != BS_OUT_BF16 && out_dtype != BS_OUT_F32 && out_dtype != BS_OUT_I32)
    return fail(BS_ERR_DTYPE, "unknown output dtype");
  if (M == 0 || N == 0) return BS_OK;
  if (!out) return fail(BS_ERR_NULL, "out is NULL");
  if (ldo < N) return fail(BS_ERR_LAYOUT, "ldo < N");
  if (!aligned16(out) || (ldo * out_size(out_dtype)) % 16 != 0)
    return fail(BS_ERR_ALIGNMENT, "out must be 16-byte aligned with a row stride that is a multiple of 16 bytes");
  if (K > 0) {
    if (!A || !B) return fail(BS_ERR_NULL, "A and B must be non-NULL");
    if (lda < K || ldb < K) return fail(BS_ERR_LAYOUT, "lda/ldb must be >= K (A row-major, B column-major)");
    if (!aligned16(A) || !aligned16(B) || lda % 16 != 0 || ldb % 16 != 0)
      return fail(BS_ERR_ALIGNMENT, "A and B must be 16-byte aligned with lda, ldb multiples of 16");
    if ((s_a && !aligned4(s_a)) || (s_b && !aligned4(s_b)))
      return fail(BS_ERR_ALIGNMENT, "scales must be 4-byte aligned");
  }
  DeviceCtx* dc = nullptr;
  bs_status st = device_ctx(&dc);
  if (st != BS_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  if (noalloc && (st = split_scratch(dc, &scratch)) != BS_OK) return st;
  const Plan pl = noalloc ? make_plan(2, M, 1, N, K, dc->sms, true, true)
                          : make_plan(2, M, 1, N, K, dc->sms, workspace_ok(dc));
  if (pl.pub.kernel == 3)
    return check_launch(launch_fill_zero(out, out_size(out_dtype), M, N, ldo, 1, 0, cs), "zero-fill launch");

  GemmArgs args;
  std::memset(&args, 0, sizeof(args));
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.G = 1;
  args.KB = static_cast<int>((K + 127) / 128);
  args.NB = static_cast<int>((N + 127) / 128);
  args.s_row = s_a;
  args.s_col = s_b;
  args.s_row_stride = 1;
  args.s_col_stride = 1;
  args.grid_m = pl.grid_m;
  args.grid_n = pl.grid_n;
  args.num_tiles = pl.num_tiles;
  args.group_m = kGroupM;
  args.splits = 1;
  args.err = dc->err;
  if (!noalloc) {
    set_work_split(args, pl, dc);
  } else {
    args.dp_tiles = pl.dp_tiles;
    args.sk_iters = pl.sk_iters;
    if (pl.sk_iters > 0) {
      uint8_t* base = static_cast<uint8_t*>(scratch);
      args.sk_ws = reinterpret_cast<uint32_t*>(base);
      args.sk_flags = reinterpret_cast<uint32_t*>(base + workspace_slots_bytes(dc->sms));
      const size_t flag_bytes = static_cast<size_t>(dc->sms) * kWsFlagsPerSlot * sizeof(uint32_t);
      const cudaError_t e = cudaMemsetAsync(args.sk_flags, 0, flag_bytes, cs);
      if (e != cudaSuccess) return fail(BS_ERR_CUDA, "clear the scratch flags: %s", cudaGetErrorString(e));
    }
  }
  CUtensorMap ta, tb, td;
  if ((st = encode_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, 1, lda, lda * M, 128, 128, "A"))) return st;
  if ((st = encode_3d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, 1, ldb, ldb * N, 128, wide_b_box_rows(pl.cg),
                      "B")))
    return st;
  const int es = out_size(out_dtype);
  if ((st = encode_3d(&td, out_tmap_type(out_dtype), es, out, N, M, 1, ldo, ldo * M, static_cast<uint32_t>(64 / es),
                      32, "out", CU_TENSOR_MAP_SWIZZLE_64B)))
    return st;
  return check_launch(launch_wide(Mode::kInt8, out_kind(out_dtype), pl.cg, ta, tb, td, args, pl.pub.ctas, cs),
                      "int8 kernel launch");
}

}  // namespace

extern "C" {

bs_status int_scaled_mm(const int8_t* A, int64_t lda, const int8_t* B, int64_t ldb, const float* s_a,
                        const float* s_b, void* out, int64_t ldo, bs_out_dtype out_dtype, int64_t M, int64_t N,
                        int64_t K, void* stream) {
  return int8_gemm(A, lda, B, ldb, s_a, s_b, out, ldo, out_dtype, M, N, K, stream, false);
}

bs_status bs_int_scaled_mm_noalloc(const int8_t* A, int64_t lda, const int8_t* B, int64_t ldb, const float* s_a,
                                   const float* s_b, void* out, int64_t ldo, bs_out_dtype out_dtype, int64_t M,
                                   int64_t N, int64_t K, void* stream) {
  return int8_gemm(A, lda, B, ldb, s_a, s_b, out, ldo, out_dtype, M, N, K, stream, true);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// zero (or bias) fill, K == 0
// ---------------------------------------------------------------------------
namespace bsg {

// out[b][r][c] = bias[c] (bias may be null: zero).  es = 2 stores bf16, es = 4
// stores fp32 (or a zero int32), es = 1 stores the saturating e4m3 code of
// s_result[0] * bias[c] (s_result null: 1).
__global__ void fill_zero_kernel(char* out, int es, long long rows, long long cols, long long ld, long long batches,
                                 long long bstride, const float* bias, const float* s_result) {
  const float sr = s_result ? *s_result : 1.f;
  const long long total = rows * cols * batches;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long b = i / (rows * cols);
    const long long rc = i - b * rows * cols;
    const long long r = rc / cols, c = rc - r * cols;
    char* p = out + (b * bstride + r * ld + c) * es;
    const float v = bias ? bias[c] : 0.f;
    if (es == 1)
      *reinterpret_cast<__nv_fp8_storage_t*>(p) = __nv_cvt_float_to_fp8(v * sr, __NV_SATFINITE, __NV_E4M3);
    else if (es == 2)
      *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
    else
      *reinterpret_cast<float*>(p) = v;
  }
}

cudaError_t launch_fill_zero(void* out, int elem_size, long long rows, long long cols, long long ld,
                             long long batches, long long bstride, cudaStream_t stream, const float* bias,
                             const float* s_result) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  fill_zero_kernel<<<2 * sms, 256, 0, stream>>>(static_cast<char*>(out), elem_size, rows, cols, ld, batches, bstride,
                                                bias, s_result);
  return cudaGetLastError();
}

}  // namespace bsg

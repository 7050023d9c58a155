// Instantiations and launcher of the skinny split-K kernel.
#include <atomic>

#include "launch.h"

namespace bsg {

namespace {

constexpr int kMaxDevices = 64;

template <Mode MODE, int BMT, typename OutT>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, const SkinnyOut& o,
                       int n_tiles, int m_tiles, cudaStream_t stream) {
  auto kernel = skinny_gemm_kernel<MODE, BMT, OutT>;
  constexpr size_t smem = sizeof(SkinnySmemFor<BMT>) + 1024;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev % kMaxDevices);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_release);
  }
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(args.splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the prologue may overlap the previous kernel
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_tiles * args.splits), static_cast<unsigned>(m_tiles),
                     static_cast<unsigned>(args.G));
  cfg.blockDim = dim3(SkinnyCfg<BMT>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, a, b, args, o);
}

template <Mode MODE, typename OutT>
cudaError_t by_bmt(int bmt, const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, const SkinnyOut& o,
                   int n_tiles, int m_tiles, cudaStream_t stream) {
  switch (bmt) {
    case 16: return launch_one<MODE, 16, OutT>(a, b, args, o, n_tiles, m_tiles, stream);
    case 32: return launch_one<MODE, 32, OutT>(a, b, args, o, n_tiles, m_tiles, stream);
    case 64: return launch_one<MODE, 64, OutT>(a, b, args, o, n_tiles, m_tiles, stream);
    case 128: return launch_one<MODE, 128, OutT>(a, b, args, o, n_tiles, m_tiles, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_skinny(Mode mode, OutKind out, int bmt, const CUtensorMap& a, const CUtensorMap& b,
                          const GemmArgs& args, const SkinnyOut& o, int n_tiles, int m_tiles, cudaStream_t stream) {
  if (mode == Mode::kFp8F32Scale) {
    if (out == OutKind::kBF16) return by_bmt<Mode::kFp8F32Scale, __nv_bfloat16>(bmt, a, b, args, o, n_tiles, m_tiles, stream);
    if (out == OutKind::kF32) return by_bmt<Mode::kFp8F32Scale, float>(bmt, a, b, args, o, n_tiles, m_tiles, stream);
  } else if (mode == Mode::kFp8E8M0) {
    if (out == OutKind::kBF16) return by_bmt<Mode::kFp8E8M0, __nv_bfloat16>(bmt, a, b, args, o, n_tiles, m_tiles, stream);
    if (out == OutKind::kF32) return by_bmt<Mode::kFp8E8M0, float>(bmt, a, b, args, o, n_tiles, m_tiles, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace bsg

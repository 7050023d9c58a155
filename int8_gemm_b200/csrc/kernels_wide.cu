// Instantiations and launcher of the persistent wide kernel.
#include <atomic>
#include <type_traits>

#include "launch.h"

namespace bsg {

namespace {

constexpr int kMaxDevices = 64;

template <Mode MODE, int CG, typename OutT, bool SPLIT>
cudaError_t launch_split(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d, const GemmArgs& args,
                         int grid, cudaStream_t stream) {
  constexpr int STAGES = wide_stages<MODE, CG>();
  auto kernel = wide_gemm_kernel<MODE, CG, STAGES, OutT, SPLIT>;
  constexpr size_t smem = sizeof(WideSmem<kWideBN / CG, STAGES, wide_stage_bufs<MODE, CG>()>) + 1024;
  static std::atomic<uint64_t> configured{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev % kMaxDevices);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_release);
  }
  // programmatic dependent launch (the prologue may overlap the previous
  // kernel) and, for CTA pairs, clusters of two
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CG;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kWideThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = CG == 2 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, b, d, args);
}

// The stream-K instantiation only for plans that split the last round.
template <Mode MODE, int CG, typename OutT>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d, const GemmArgs& args,
                       int grid, cudaStream_t stream) {
  return args.sk_iters > 0 ? launch_split<MODE, CG, OutT, true>(a, b, d, args, grid, stream)
                           : launch_split<MODE, CG, OutT, false>(a, b, d, args, grid, stream);
}

template <int CG>
cudaError_t launch_cg(Mode mode, OutKind out, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d,
                      const GemmArgs& args, int grid, cudaStream_t stream) {
  switch (mode) {
    case Mode::kFp8F32Scale:
      if (out == OutKind::kBF16) return launch_one<Mode::kFp8F32Scale, CG, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kFp8F32Scale, CG, float>(a, b, d, args, grid, stream);
      break;
    case Mode::kFp8E8M0:
      if (out == OutKind::kBF16) return launch_one<Mode::kFp8E8M0, CG, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kFp8E8M0, CG, float>(a, b, d, args, grid, stream);
      break;
    case Mode::kFp8Rowwise:
      if (out == OutKind::kBF16) return launch_one<Mode::kFp8Rowwise, CG, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kFp8Rowwise, CG, float>(a, b, d, args, grid, stream);
      if (out == OutKind::kE4M3) return launch_one<Mode::kFp8Rowwise, CG, uint8_t>(a, b, d, args, grid, stream);
      break;
    case Mode::kFp8Mx:
      if constexpr (CG == 2) {
        if (out == OutKind::kBF16) return launch_one<Mode::kFp8Mx, CG, __nv_bfloat16>(a, b, d, args, grid, stream);
        if (out == OutKind::kF32) return launch_one<Mode::kFp8Mx, CG, float>(a, b, d, args, grid, stream);
      }
      break;
    case Mode::kInt8:
      if (out == OutKind::kBF16) return launch_one<Mode::kInt8, CG, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kInt8, CG, float>(a, b, d, args, grid, stream);
      if (out == OutKind::kI32) return launch_one<Mode::kInt8, CG, int32_t>(a, b, d, args, grid, stream);
      break;
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_wide(Mode mode, OutKind out, int cta_group, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& d, const GemmArgs& args, int grid, cudaStream_t stream) {
  if (cta_group == 2) return launch_cg<2>(mode, out, a, b, d, args, grid, stream);
  if (cta_group == 1) return launch_cg<1>(mode, out, a, b, d, args, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace bsg

// Instantiations and launcher of the persistent wide kernel.
#include <atomic>
#include <type_traits>

#include "launch.h"

namespace bsg {

namespace {

constexpr int kMaxDevices = 64;

template <Mode MODE, typename OutT>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d, const GemmArgs& args,
                       int grid, cudaStream_t stream) {
  auto kernel = wide_gemm_kernel<MODE, kWideBN, kWideStages, OutT>;
  constexpr size_t smem = sizeof(WideSmem<kWideBN, kWideStages>) + 1024;
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kWideThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, kernel, a, b, d, args);
}

}  // namespace

cudaError_t launch_wide(Mode mode, OutKind out, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d,
                        const GemmArgs& args, int grid, cudaStream_t stream) {
  switch (mode) {
    case Mode::kFp8F32Scale:
      if (out == OutKind::kBF16) return launch_one<Mode::kFp8F32Scale, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kFp8F32Scale, float>(a, b, d, args, grid, stream);
      break;
    case Mode::kFp8E8M0:
      if (out == OutKind::kBF16) return launch_one<Mode::kFp8E8M0, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kFp8E8M0, float>(a, b, d, args, grid, stream);
      break;
    case Mode::kInt8:
      if (out == OutKind::kBF16) return launch_one<Mode::kInt8, __nv_bfloat16>(a, b, d, args, grid, stream);
      if (out == OutKind::kF32) return launch_one<Mode::kInt8, float>(a, b, d, args, grid, stream);
      if (out == OutKind::kI32) return launch_one<Mode::kInt8, int32_t>(a, b, d, args, grid, stream);
      break;
  }
  return cudaErrorInvalidValue;
}

}  // namespace bsg

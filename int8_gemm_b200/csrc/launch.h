// Internal interface between the C-ABI layer (api.cu) and the kernel
// translation units.  Not part of the public header.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "skinny_kernel.cuh"
#include "wide_kernel.cuh"

namespace bsg {

enum class OutKind : int { kBF16 = 0, kF32 = 1, kI32 = 2, kE4M3 = 3 };

constexpr int kWideBN = 256;
constexpr int kWideThreads = 384;

// Persistent wide kernel over `grid` CTAs; cta_group 2 launches clusters of two
// CTAs computing 256 x 256 tiles, cta_group 1 single CTAs computing 128 x 256.
cudaError_t launch_wide(Mode mode, OutKind out, int cta_group, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& d, const GemmArgs& args, int grid, cudaStream_t stream);

// Skinny split-K kernel: grid (n_tiles * splits, m_tiles, G), cluster (splits, 1, 1).
cudaError_t launch_skinny(Mode mode, OutKind out, int bmt, const CUtensorMap& a, const CUtensorMap& b,
                          const GemmArgs& args, const SkinnyOut& o, int n_tiles, int m_tiles, cudaStream_t stream);

// Small-M kernel (kernels_gemv.cu): M <= kGemvMaxM activation rows, FP8
// modes kFp8F32Scale and kFp8E8M0.  Activation (m, g, k) at
// a[m * a_sm + g * a_sg + k], weight (g, n, k) at b[g * b_sg + n * b_sn + k],
// output (m, g, n) at out[m * o_sm + g * o_sg + n] (byte strides for a and b,
// element strides for out).  Grid: ceil(N / 16) x G CTAs of 8 warps.
constexpr int kGemvMaxM = 8;
struct GemvProblem {
  const void* a;
  long long a_sm, a_sg;
  const void* b;
  long long b_sn, b_sg;
  void* out;
  long long o_sm, o_sg;
  int sms;  // SMs of the device (grid size choice)
};
cudaError_t launch_gemv(Mode mode, OutKind out, const GemvProblem& q, const GemmArgs& args, cudaStream_t stream);

// Built-in scratch of bs_int_scaled_mm_noalloc (static_scratch.cu): the
// stream-K slots and flag words of a device with at most kStaticScratchMaxSms
// SMs, in the layout of a registered workspace (20 MB in all).
constexpr int kStaticScratchMaxSms = 160;
constexpr size_t kStaticScratchBytes =
    static_cast<size_t>(kStaticScratchMaxSms) * kWsSlotWords * sizeof(uint32_t) +
    ((static_cast<size_t>(kStaticScratchMaxSms) * kWsFlagsPerSlot * sizeof(uint32_t) + 255) / 256) * 256;
// Device address of that array (cudaGetSymbolAddress; the current device).
cudaError_t static_scratch_address(void** ptr);

// Fill of `batches` matrices [rows, cols] (row stride ld, batch stride
// bstride, elements of `elem_size` bytes: bf16, fp32, or 1 = e4m3) with zero,
// or with bias[col] (fp32 [cols]) when bias is given; e4m3 elements take the
// saturating e4m3 of s_result[0] * value (s_result NULL: 1).
cudaError_t launch_fill_zero(void* out, int elem_size, long long rows, long long cols, long long ld,
                             long long batches, long long bstride, cudaStream_t stream,
                             const float* bias = nullptr, const float* s_result = nullptr);

}  // namespace bsg

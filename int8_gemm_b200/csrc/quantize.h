// Internal interface of the quantiser kernels (kernels_quantize.cu,
// kernels_quantize_t.cu, kernels_quantize_blocks.cu) for the C-ABI layer.
// Not part of the public header.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace bsg {

// Launch facts of a kernel that hold for the whole process, worked out on a
// device's first launch only (as the GEMM launchers do): the dynamic
// shared-memory limit is raised to `smem` bytes and the number of CTAs of
// `threads` threads that fit on one SM is queried.  Devices are told apart by
// their index modulo 64.
template <auto KERNEL>
cudaError_t ctas_per_sm_once(int threads, size_t smem, int* per_sm) {
  static std::atomic<int> known[64];  // 0: not yet worked out on that device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::atomic<int>& slot = known[dev % 64];
  int v = slot.load(std::memory_order_acquire);
  if (v == 0) {
    if (smem > 0) {
      e = cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, KERNEL, threads, smem);
    if (e != cudaSuccess) return e;
    if (v < 1) v = 1;
    slot.store(v, std::memory_order_release);
  }
  *per_sm = v;
  return cudaSuccess;
}

// 1x128 group quantisation of x [M, K] (bf16 or fp32, row stride ldx
// elements) to e4m3 codes q (row stride ldq bytes) and one scale per group:
// fp32 amax / 448, or an e8m0 byte (e8m0 = true); scale row stride lds.
// tmx / tmq: tensor maps of x and q (box 128 x 128; q with the 128-byte
// swizzle), or null where x or q is not 16-byte aligned with 16-byte row
// strides or K is not a multiple of 16; with both given the TMA-fed kernel of
// quant_ring.cuh runs, whose bounded waits record a timeout in the device
// error word `err`.
cudaError_t launch_quantize_1x128(const void* x, bool x_bf16, long long M, long long K, long long ldx, uint8_t* q,
                                  long long ldq, void* scale, bool e8m0, long long lds, int sms,
                                  const CUtensorMap* tmx, const CUtensorMap* tmq, uint32_t* err,
                                  cudaStream_t stream);

// Transposed-output quantisation of x [R, C] (bf16 or fp32, row stride ldx
// elements) to e4m3 codes q_t [C, R] (row stride ldq bytes), q_t[c][r] the
// code of x[r][c].  block128 = false: 128x1 groups (rows 128rb.. of one
// column), scale [C, ceil(R/128)]; true: 128x128 blocks, scale
// [ceil(R/128), ceil(C/128)]; scale row stride lds, fp32 or e8m0 bytes.
// tmx / tmq: tensor maps of x (box 128 x 128, no swizzle) and q_t (box 128 x
// 128 bytes, 128-byte swizzle), or null unless x and q_t have 16-byte bases and
// row strides and their rows' used bytes (C elements, R codes) end on 16-byte
// boundaries; with both given the TMA-fed kernel runs, whose bounded waits
// record a timeout in the device error word `err`.
cudaError_t launch_quantize_t(const void* x, bool x_bf16, long long R, long long C, long long ldx, uint8_t* q_t,
                              long long ldq, void* scale, bool e8m0, bool block128, long long lds, int sms,
                              const CUtensorMap* tmx, const CUtensorMap* tmq, uint32_t* err, cudaStream_t stream);

// 128x128 block quantisation of x [R, C] (bf16 or fp32, row stride ldx
// elements) in its own orientation: codes q [R, C] (row stride ldq bytes),
// q[r][c] the code of x[r][c], one scale per block (rb, cb) at
// scale[rb * s_rb + cb * s_cb] (element strides), fp32 or e8m0 bytes.
// tmx / tmq: tensor maps of x and q (box 128 x 128; q with the 128-byte
// swizzle), or null where x or q is not 16-byte aligned with 16-byte row
// strides or C is not a multiple of 16; with both given the TMA-fed kernel of
// quant_ring.cuh runs, whose bounded waits record a timeout in the device
// error word `err`.
cudaError_t launch_quantize_blocks(const void* x, bool x_bf16, long long R, long long C, long long ldx, uint8_t* q,
                                   long long ldq, void* scale, bool e8m0, long long s_rb, long long s_cb, int sms,
                                   const CUtensorMap* tmx, const CUtensorMap* tmq, uint32_t* err,
                                   cudaStream_t stream);

}  // namespace bsg

// Internal interface of the 1x128 group quantiser (kernels_quantize.cu) for the
// C-ABI layer.  Not part of the public header.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bsg {

// 1x128 group quantisation of x [M, K] (bf16 or fp32, row stride ldx
// elements) to e4m3 codes q (row stride ldq bytes) and one scale per group:
// fp32 amax / 448, or an e8m0 byte (e8m0 = true); scale row stride lds.
cudaError_t launch_quantize_1x128(const void* x, bool x_bf16, long long M, long long K, long long ldx, uint8_t* q,
                                  long long ldq, void* scale, bool e8m0, long long lds, int sms,
                                  cudaStream_t stream);

}  // namespace bsg

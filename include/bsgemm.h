/*
 * bsgemm -- scaled low-precision GEMMs with the dequantisation fused in,
 * hand-written for NVIDIA B200 (sm_100a: TMA, tcgen05 tensor cores, TMEM).
 *
 * C ABI.  Every pointer argument is a DEVICE pointer unless stated otherwise,
 * owned by the caller; the library keeps no reference after the call returns
 * and allocates no device memory.  Every call that launches work (the GEMMs
 * and the quantisers) is asynchronous on the given stream (a cudaStream_t
 * passed as void*; NULL = legacy default stream).
 * Argument checks run synchronously on the host before anything is launched;
 * a call that returns an error status has launched nothing.  There is no CPU
 * fallback: on a device other than compute capability 10.0 the calls return
 * BS_ERR_DEVICE.
 *
 * Conventions shared by the GEMM operations
 *   - Sizes are in elements, strides ("ld", "s_*") in elements of the tensor
 *     they describe.
 *   - FP8 operands are OCP e4m3 ("float8_e4m3fn") bytes; INT8 operands are
 *     signed bytes.
 *   - A is row-major [M, K]; B is the logical [K, N] matrix stored
 *     column-major, i.e. as N rows of K contiguous bytes (the layout contract
 *     of check_supported_striding in pytorch/torch/_inductor/kernel/mm.py:
 *     mat_a row-major, mat_b column-major).
 *   - Base pointers of A, B and the output must be 16-byte aligned and their
 *     row strides multiples of 16 bytes (the tensor-memory-accelerator rule).
 *   - M == 0 or N == 0 is a no-op returning BS_OK (the early exit of
 *     mm_template in the same file); K == 0 writes zeros.
 *   - The scale tensors multiply: the dequantised value is code * scale (the
 *     scaling of the accumulator in apply_scaling, same file).
 */
#ifndef BSGEMM_H
#define BSGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BS_OK = 0,
  BS_ERR_NULL = 1,      /* a required pointer is NULL */
  BS_ERR_SHAPE = 2,     /* negative / unsupported size, or scale shape mismatch */
  BS_ERR_LAYOUT = 3,    /* stride smaller than the row it describes, bad unit stride */
  BS_ERR_ALIGNMENT = 4, /* pointer or stride breaks the 16-byte rule */
  BS_ERR_DTYPE = 5,     /* output dtype not supported by this operation */
  BS_ERR_DEVICE = 6,    /* current device is not an sm_100 (B200-class) GPU */
  BS_ERR_CUDA = 7,      /* a CUDA runtime call failed (launch, encode, ...) */
  BS_ERR_TIMEOUT = 8,   /* a kernel gave up on a bounded wait (bs_get_device_error) */
  BS_ERR_WORKSPACE = 9  /* workspace smaller than bs_workspace_size(), or a device with more
                           SMs than bs_int_scaled_mm_noalloc's built-in scratch holds */
} bs_status;

typedef enum {
  BS_OUT_BF16 = 0, /* bfloat16, round-to-nearest-even from the fp32 result */
  BS_OUT_F32 = 1,  /* float32 */
  BS_OUT_I32 = 2,  /* raw int32 accumulator (int_scaled_mm only) */
  BS_OUT_E4M3 = 3  /* e4m3 bytes: round-to-nearest-even, saturated at +-448, of
                      scale_result * result (bs_gemm_fp8_rowwise only) */
} bs_out_dtype;

/*
 * Operation 1 -- FP8 block-scaled GEMM.
 *
 *   out[m, n] = sum_kb  scale_a[m, kb] * scale_b[kb, n / 128]
 *                       * sum_{k in block kb} A[m, k] * B[k, n]
 *
 * i.e. (A . expand(scale_a)) @ (B . expand(scale_b)) with 1x128 activation
 * groups and 128x128 weight blocks.  Source: pytorch issue "torch._scaled_mm
 * with blockwise scaling doesn't work with torch.compile" -- the error text
 * gives scale_a (16640, 64) and scale_b (64, 40) for M = 16640, K = 8192,
 * N = 5120, that is scale_a [M, K/128] and scale_b [K/128, N/128].
 * Accumulation is fp32 inside each 128-deep block and across blocks.
 *
 *   A        e4m3 [M, K], row m at A + m*lda                (lda >= K)
 *   B        e4m3 [K, N] column-major, column n at B + n*ldb (ldb >= K)
 *   scale_a  fp32 [M, K/128], element (m, kb) at scale_a[m*sa_sm + kb*sa_sk]
 *   scale_b  fp32 [K/128, ceil(N/128)], element (kb, nb) at
 *            scale_b[kb*sb_sk + nb*sb_sn]
 *   out      [M, N] row-major, row stride ldo (>= N), BS_OUT_BF16 or BS_OUT_F32
 *   K must be a multiple of 128 (one scale per 128-deep group).
 * Zero and subnormal scales are accepted.  Each block's scale product
 * scale_a * scale_b is formed in fp32: below 2^-140 in magnitude, where fp32
 * subnormals keep fewer than ten significant bits, that block contributes with
 * an absolute error of up to 2^-150 times its sum of |A*B|.  bf16 outputs are
 * coarser than that error; fp32 outputs whose blocks all have products of zero
 * or at least 2^-140 meet the relative bound of the other inputs.
 */
bs_status bs_gemm_fp8_blockwise(const void* A, int64_t lda, const void* B, int64_t ldb,
                                const float* scale_a, int64_t sa_sm, int64_t sa_sk,
                                const float* scale_b, int64_t sb_sk, int64_t sb_sn,
                                void* out, int64_t ldo, bs_out_dtype out_dtype,
                                int64_t M, int64_t N, int64_t K, void* stream);

/*
 * FP8 GEMM with tensorwise or rowwise scales and an optional bias (the other
 * scaling modes of torch._scaled_mm).
 *
 *   out[m, n] = (sum_k A[m, k] * B[k, n]) * (scale_a[m * sa_stride] * scale_b[n * sb_stride])
 *               + bias[n]
 *
 * Source: pytorch/torch/_inductor/kernel/mm.py -- apply_scaling (tensorwise:
 * accumulator * (a_scale * b_scale); rowwise: a per-row scale_a times a
 * per-column scale_b) and tuned_scaled_mm (optional bias [N] added to every
 * row); the pytorch issue "torch._scaled_mm with blockwise scaling doesn't
 * work with torch.compile" states the shapes: tensorwise scales are scalars,
 * rowwise scale_a is (M, 1) and scale_b is (1, N).  The scales are constant
 * along K, so the fp32 accumulator covers all of K before the scaling.
 *
 *   A        e4m3 [M, K], row m at A + m*lda                (lda >= K)
 *   B        e4m3 [K, N] column-major, column n at B + n*ldb (ldb >= K)
 *   scale_a  fp32; sa_stride = 0: one scale (tensorwise), 1: [M] (rowwise)
 *   scale_b  fp32; sb_stride = 0: one scale (tensorwise), 1: [N] (rowwise)
 *            (both strides equal: the two operands use the same mode)
 *   bias     fp32 [N] or NULL
 *   scale_result  fp32 scalar or NULL (1): with BS_OUT_E4M3 the result is
 *            multiplied by it before the saturating e4m3 cast, the output
 *            scale of an fp8 result (tuned_scaled_mm's scale_result, same
 *            file); it must be NULL for the other output types
 *   out      [M, N] row-major, row stride ldo (>= N), BS_OUT_BF16, BS_OUT_F32
 *            or BS_OUT_E4M3
 *   K is free (lda and ldb multiples of 16); K == 0 writes bias (or zeros).
 * The accumulator is fp32 in tensor memory over all of K; tuned_scaled_mm's
 * use_fast_accum chooses between accumulating inside the MMA and adding each
 * K tile's product in fp32, and on this hardware both are the fp32
 * accumulation done here, so it is not a parameter.
 * Not a block-scaled operation: it has no counterpart in the block-scaled
 * statement of the problem above and follows the mm.py scaling modes.
 */
bs_status bs_gemm_fp8_rowwise(const void* A, int64_t lda, const void* B, int64_t ldb,
                              const float* scale_a, int64_t sa_stride, const float* scale_b, int64_t sb_stride,
                              const float* bias, const float* scale_result, void* out, int64_t ldo,
                              bs_out_dtype out_dtype, int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Operation 2 -- INT8 GEMM with a fused, fixed-order fp32 dequantisation.
 *
 *   acc[m, n] = sum_k A[m, k] * B[k, n]              (exact, int32)
 *   out[m, n] = (float(acc) * s_a[m]) * s_b[n]       (two fp32 RNE multiplies)
 *
 * Sources: pytorch/ao PR "Remove int_scaled_mm's dependency on triton for
 * cpu" (the CPU definition: _int_mm, then cast to the scale dtype and
 * multiply); pytorch/ao issue "Unify scaled INT8 matmul" (both scales fused,
 * the int32 accumulator cast to fp32 before scaling).  s_b == NULL gives the
 * row-scale-only form of that CPU definition; s_a == NULL skips the row
 * multiply.  BS_OUT_BF16 rounds the fp32 result to nearest-even;
 * BS_OUT_I32 writes acc and ignores the scales (the int32 output layout of
 * tuned_int_mm, pytorch/torch/_inductor/kernel/mm.py).
 *
 *   A    int8 [M, K] row-major (lda >= K);  B int8 [K, N] column-major (ldb >= K)
 *   s_a  fp32 [M] or NULL;  s_b fp32 [N] or NULL
 *   out  [M, N] row-major, row stride ldo (>= N)
 *   K <= 131071, which keeps every int32 accumulator exact.
 */
bs_status int_scaled_mm(const int8_t* A, int64_t lda, const int8_t* B, int64_t ldb,
                        const float* s_a, const float* s_b,
                        void* out, int64_t ldo, bs_out_dtype out_dtype,
                        int64_t M, int64_t N, int64_t K, void* stream);

/*
 * int_scaled_mm that allocates nothing, for callers that cannot allocate
 * device memory: a serving loop that reserves all of HBM up front (a cache
 * or a pool holding the rest), code running inside a custom allocator's own
 * callbacks (which must not re-enter it), or a C host with no device
 * allocator of its own.  cudaMalloc and cudaFree also synchronise the
 * device, which such callers cannot afford between launches.
 *
 * Arguments, layouts, results (bit-exact) and error codes are those of
 * int_scaled_mm.  The difference: the stream-K split of the wide kernel's
 * last round of tiles always applies where the planner's rule calls for it
 * (whether or not bs_set_stream_k is on), and its partial sums and flag
 * words live in a fixed array built into the library -- 20 MB, enough for
 * devices of up to 160 SMs -- not in a registered workspace.  Neither this
 * call nor the library allocates device memory for it.
 *
 * The first call on a device does the set-up, with that device current: it
 * looks up the array's address (cudaGetSymbolAddress, which loads the
 * array's module).  Make that first call before any stream capture.  Every
 * call that splits clears the array's flag words on `stream` (an
 * asynchronous memset) before its kernel, so they start at zero.  Calls
 * whose work overlaps on the GPU -- on different streams or from different
 * threads -- share the array and race: order them on one stream or
 * synchronise between them.
 *
 * Returns BS_ERR_WORKSPACE on a device with more than 160 SMs, BS_ERR_CUDA if
 * the set-up fails.  The published method has no counterpart of this entry
 * point: it is a deployment variant of int_scaled_mm.
 */
bs_status bs_int_scaled_mm_noalloc(const int8_t* A, int64_t lda, const int8_t* B, int64_t ldb,
                                   const float* s_a, const float* s_b,
                                   void* out, int64_t ldo, bs_out_dtype out_dtype,
                                   int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Operation 3 -- batched FP8 GEMM with e8m0 (power-of-two) block scales.
 *
 *   out[m, g, n] = sum_kb 2^(x_scale[m, g, kb] - 127) * 2^(w_scale[g, n/128, kb] - 127)
 *                         * sum_{k in block kb} x[m, g, k] * w[g, n, k]
 *
 * Source: ROCm/aiter PR "Add opus fp8 mxscale BMM kernels for gfx950"
 * (Motivation: the m-major layout x [M, G, K], w [G, N, K] batch-major,
 * x_scale [M, G, K/128], w_scale [G, N/128, K/128], optional out [M, G, N],
 * bf16 output; Test Plan: m-major and batch-first layouts of x).
 *
 *   x        e4m3, element (m, g, k) at x[m*x_sm + g*x_sg + k].  m-major:
 *            (x_sm, x_sg) = (G*K, K); batch-first storage [G, M, K]: (K, M*K).
 *   w        e4m3, element (g, n, k) at w[g*w_sg + n*w_sn + k]  (w_sn >= K)
 *   x_scale  e8m0 bytes [M, G, K/128], contiguous
 *   w_scale  e8m0 bytes [G, ceil(N/128), K/128], contiguous
 *   out      element (m, g, n) at out[m*o_sm + g*o_sg + n]; BS_OUT_BF16 or BS_OUT_F32
 *   K must be a multiple of 128.  Scale byte 255 encodes NaN and is not checked.
 * Every byte 0..254 is decoded exactly (byte 0 is 2^-127, an fp32 subnormal),
 * whether the tensor core applies the scales (CTA pairs) or the CUDA cores
 * promote each block; block products that underflow fp32 contribute zero.
 */
bs_status bmm_a8w8_blockscale(const void* x, int64_t x_sm, int64_t x_sg,
                              const void* w, int64_t w_sg, int64_t w_sn,
                              const uint8_t* x_scale, const uint8_t* w_scale,
                              void* out, int64_t o_sm, int64_t o_sg, bs_out_dtype out_dtype,
                              int64_t M, int64_t G, int64_t N, int64_t K, void* stream);

/* ------------------------------------------------------------------------ */
/* host-side helpers (no device work unless stated)                          */
/* ------------------------------------------------------------------------ */

/* Static name of a status code ("BS_OK", ...).  Never NULL. */
const char* bs_status_string(bs_status status);

/* Human-readable detail of the last error returned on the calling host
 * thread (empty string after a successful call).  Never NULL. */
const char* bs_last_error_message(void);

/*
 * Shape rule of operation 1 (the blockwise case of the scale-shape check in
 * the pytorch issue above): BS_OK iff scale_a is [M, ceil(K/128)] and scale_b
 * is [ceil(K/128), ceil(N/128)].  The rowwise shapes (M, 1) / (1, N) are
 * rejected here.  Pure host logic.
 */
bs_status bs_check_blockwise_scale_shapes(int64_t M, int64_t N, int64_t K,
                                          int64_t sa_rows, int64_t sa_cols,
                                          int64_t sb_rows, int64_t sb_cols);

/* Which kernel a call would launch, for tests and benchmarks. */
typedef struct {
  int32_t kernel;  /* 0: none (empty problem), 1: persistent wide, 2: skinny split-K, 3: zero fill,
                      4: small-M weight stream (warp-level MMA, M <= 8) */
  int32_t tile_m;  /* rows of A (M direction) per tile */
  int32_t tile_n;  /* columns of B (N direction) per tile */
  int32_t splits;  /* K splits reduced through cluster shared memory (1 = none) */
  int32_t ctas;    /* CTAs launched */
  int32_t cluster; /* CTAs per thread-block cluster (2 for the CTA-pair wide kernel) */
  int32_t launches;/* kernel launches the call makes */
  int32_t sk_tiles;/* wide kernel: tiles whose K blocks are split over several CTA pairs (or CTAs)
                      to balance the last wave (stream-K); 0 = every tile is computed whole */
} bs_plan;

/*
 * Fused quantiser -- 1x128 activation groups to e4m3 (the input side of
 * operations 1 and 3).
 *
 * For every row m of x and every group g of 128 consecutive elements along K
 * (the last group of a row holds K - 128*(ceil(K/128) - 1) elements):
 *   amax = max |x[m, k]| over the group
 *   BS_SCALE_F32:  scale[m, g] = amax / 448 (fp32 division; 1 when that is 0:
 *                  amax == 0, or amax < 448 * 2^-150 and the quotient underflows)
 *                  q[m, k]     = e4m3(x[m, k] / scale[m, g])   (fp32 division)
 *   BS_SCALE_E8M0: scale[m, g] = clamp(ceil(log2(amax / 448)) + 127, 0, 254),
 *                  the e8m0 byte of the smallest power of two 2^e with
 *                  amax <= 448 * 2^e (127 when amax == 0)
 *                  q[m, k]     = e4m3(x[m, k] * 2^-(scale[m, g] - 127))
 * where e4m3() rounds to nearest, ties to even, saturates at +-448 and maps
 * NaN to NaN (0x7F / 0xFF).  448 is the largest finite e4m3 magnitude, so the
 * group's amax element becomes +-448.  The fp32 form gives exactly the A and
 * scale_a [M, K/128] of bs_gemm_fp8_blockwise (pytorch issue
 * "torch._scaled_mm with blockwise scaling doesn't work with torch.compile":
 * 1x128 groups, one fp32 scale each); the e8m0 form gives the power-of-two
 * group scales of bmm_a8w8_blockscale (ROCm/aiter PR "Add opus fp8 mxscale
 * BMM kernels for gfx950").  Results are bit-exact (integer codes and exact
 * scales); non-finite inputs other than NaN give unspecified codes.
 *
 *   x      bf16 or fp32 [M, K], row m at x + m*ldx (ldx >= K, in elements)
 *   q      e4m3 codes [M, K], row m at q + m*ldq bytes (ldq >= K)
 *   scale  [M, ceil(K/128)] fp32 or e8m0 bytes, row stride ld_scale elements
 *   x must be aligned to its element size and fp32 scales to 4 bytes; any
 *   row strides work (groups whose x row segment is 16-byte aligned and whose
 *   q segment is 4-byte aligned use vector loads and stores).
 *   M * ceil(K/512) must stay below 2^31.  M == 0 or K == 0 is a no-op.
 */
typedef enum {
  BS_IN_BF16 = 0, /* bfloat16 */
  BS_IN_F32 = 1   /* float32 */
} bs_in_dtype;

typedef enum {
  BS_SCALE_F32 = 0, /* fp32 scale = amax / 448 */
  BS_SCALE_E8M0 = 1 /* e8m0 byte: power-of-two scale 2^(byte - 127) */
} bs_scale_fmt;

bs_status bs_quantize_fp8_1x128(const void* x, bs_in_dtype x_dtype, int64_t M, int64_t K, int64_t ldx, void* q,
                                int64_t ldq, void* scale, bs_scale_fmt scale_fmt, int64_t ld_scale, void* stream);

/*
 * Transposed-output quantiser -- the operands of the backward GEMMs of a
 * blockwise fp8 linear layer y = x W^T (x [M, K] in 1x128 groups, W [N, K] in
 * 128x128 blocks; the forward and backward benchmark of the pytorch issue
 * "torch._scaled_mm with blockwise scaling doesn't work with torch.compile").
 * The backward GEMMs contract over the rows of their inputs (the M tokens for
 * the weight gradient dW = dy^T x, the N outputs for the input gradient
 * dx = dy W), so the codes are written transposed, with groups along those
 * rows:
 *   q_t[c, r] = code of x[r, c],  q_t [C, R], row c at q_t + c*ldq (ldq >= R)
 *   BS_GROUP_128x1:   one scale per column c and 128-row block rb (rows
 *                     128rb .. min(128rb + 128, R) - 1), scale[c, rb] at
 *                     scale + c*ld_scale + rb, [C, ceil(R/128)]: the 1x128
 *                     groups of x^T, i.e. scale_a of bs_gemm_fp8_blockwise
 *                     for A = q_t
 *   BS_GROUP_128x128: one scale per 128 x 128 block, scale[rb, cb] at
 *                     scale + rb*ld_scale + cb, [ceil(R/128), ceil(C/128)]:
 *                     scale_b of bs_gemm_fp8_blockwise for B_t = q_t (B the
 *                     column-major view of q_t)
 * with the scale and code rules of bs_quantize_fp8_1x128 (amax over the group;
 * fp32 amax / 448 or the e8m0 byte; saturating RNE e4m3 codes).  Bit-exact.
 *   dW = dy^T x:  A = q_t(dy, 128x1), B_t = q_t(x, 128x128)
 *   dx = dy W:    A = bs_quantize_fp8_1x128(dy), B_t = q_t(W, 128x128)
 *   x      bf16 or fp32 [R, C], row r at x + r*ldx (ldx >= C, in elements),
 *          aligned to its element size
 *   fp32 scales must be 4-byte aligned.  R == 0 or C == 0 is a no-op.
 *   16-byte loads and stores are used where x, ldx, q_t and ldq allow them.
 */
typedef enum {
  BS_GROUP_128x1 = 0,  /* 128 rows of one column */
  BS_GROUP_128x128 = 1 /* 128 x 128 blocks */
} bs_group;

bs_status bs_quantize_fp8_t(const void* x, bs_in_dtype x_dtype, int64_t R, int64_t C, int64_t ldx, void* q_t,
                           int64_t ldq, void* scale, bs_scale_fmt scale_fmt, bs_group group, int64_t ld_scale,
                           void* stream);

/*
 * Weight quantiser -- 128x128 blocks to e4m3 in the input's own orientation
 * (the weight operand of the forward GEMM).
 *
 * For every block of rows 128rb .. min(128rb + 128, R) - 1 and columns
 * 128cb .. min(128cb + 128, C) - 1 of x, one scale from the block's amax and
 * one code per element, with the scale and code rules of
 * bs_quantize_fp8_1x128:
 *   q[r, c] = code of x[r, c],  q [R, C], row r at q + r*ldq bytes (ldq >= C)
 *   scale of block (rb, cb) at scale[rb*s_rb + cb*s_cb] (element strides)
 * A weight W [N, K] (y = x W^T) becomes the B_t [N, K] codes that
 * bs_gemm_fp8_blockwise reads as its column-major B, and with
 * (s_rb, s_cb) = (1, ceil(N/128)) the scales land as its
 * scale_b [K/128, N/128] -- no transpose copy of either.  Source: pytorch
 * issue "torch._scaled_mm with blockwise scaling doesn't work with
 * torch.compile" (128x128 weight blocks, one fp32 scale each: scale_b
 * (64, 40) for K = 8192, N = 5120).  Bit-exact (integer codes, exact scales).
 *   x      bf16 or fp32 [R, C], row r at x + r*ldx (ldx >= C, in elements),
 *          aligned to its element size
 *   s_rb, s_cb >= 0, and non-zero along a dimension that has several blocks.
 *   fp32 scales must be 4-byte aligned.  R == 0 or C == 0 is a no-op.
 *   16-byte loads are used where x and ldx allow them.
 */
bs_status bs_quantize_fp8_128x128(const void* x, bs_in_dtype x_dtype, int64_t R, int64_t C, int64_t ldx, void* q,
                                  int64_t ldq, void* scale, bs_scale_fmt scale_fmt, int64_t s_rb, int64_t s_cb,
                                  void* stream);

/* Plan of operation `op` (1 = bs_gemm_fp8_blockwise, 2 = int_scaled_mm,
 * 3 = bmm_a8w8_blockscale, 4 = bs_gemm_fp8_rowwise; G = 1 for ops 1, 2 and 4)
 * on a GPU with `num_sms`
 * streaming multiprocessors.  Pure host logic; honours bs_set_path_override. */
bs_status bs_plan_for(int32_t op, int64_t M, int64_t G, int64_t N, int64_t K, int32_t num_sms, bs_plan* plan);

/* Force the kernel family for subsequent calls in this process (testing):
 * 0 = automatic (default), 1 = persistent wide kernel on CTA pairs (256 x 256
 * tiles), 2 = skinny split-K kernel where the operation has one, 3 = persistent
 * wide kernel on single CTAs (128 x 256 tiles), 4 = as 1, but
 * bmm_a8w8_blockscale promotes every 128-deep block on the CUDA cores instead
 * of letting the tensor core apply its e8m0 scales (block-scaled MMA), 5 = the
 * small-M weight-stream kernel (operations 1 and 3 with M <= 8).
 * Returns the previous setting. */
int32_t bs_set_path_override(int32_t path);

/* Force the skinny kernel's split-K factor (1, 2, 4 or 8 CTAs per cluster, at
 * most the number of K blocks) for subsequent calls in this process (testing
 * and tuning); 0 restores the planner's choice.  Returns the previous setting. */
int32_t bs_set_split_override(int32_t splits);

/*
 * Stream-K workspace.  When a problem's tiles would leave the last round of
 * the persistent wide kernel's CTA pairs (or CTAs) badly filled, the K blocks
 * of the remaining tiles are spread evenly over all of them and the pieces of
 * a split tile meet in this workspace: fp32 (int32 for int_scaled_mm) partial
 * sums, added in a fixed order by the CTA that holds the tile's first K block,
 * so results are deterministic.  The split is off by default (on the B200
 * shapes measured, INT8 4096^3, FP8 1000 x 7168 x 2048 and BMMs of 1024-row
 * batches, it was 14-35% slower than computing every tile whole: a split
 * tile's hand-over costs more than the idle part of the last round); it runs
 * only after bs_set_stream_k(1) and with a registered workspace.
 *
 * bs_workspace_size(num_sms): bytes needed on a GPU with num_sms SMs
 *   (num_sms * 131,104 rounded up; about 19.4 MB on a 148-SM B200).  Pure host logic.
 * bs_set_workspace(ptr, bytes): registers a caller-owned device buffer for the
 *   current device (NULL unregisters).  `ptr` must be 256-byte aligned and
 *   zero-filled before its first use; every call that completes leaves its
 *   flag words zero again.  The library keeps the pointer until it is replaced
 *   or unregistered and never frees it.  Calls that may split K share this
 *   buffer, so they must not run concurrently on different streams of the
 *   device (as with a library handle's workspace).  Returns BS_ERR_WORKSPACE
 *   if `bytes` < bs_workspace_size(device SMs), BS_ERR_ALIGNMENT if misaligned.
 * bs_set_stream_k(enable): 1 enables the split process-wide, 0 (the
 *   default) disables it; returns the previous setting.
 */
size_t bs_workspace_size(int32_t num_sms);
bs_status bs_set_workspace(void* workspace, size_t bytes);
int32_t bs_set_stream_k(int32_t enable);

/* The work items of one unit (CTA pair or CTA) `unit` of `units` in the
 * persistent wide kernel, in processing order: tiles [0, dp_tiles) whole
 * (tile t by unit t % units), then that unit's share of the sk_iters =
 * (num_tiles - dp_tiles) * kb split K blocks.  Writes (tile, first K block,
 * end K block) triples to out[3*i ..] for the first `capacity` items and
 * returns the number of items, or -1 for inconsistent arguments.  Pure host
 * logic (the host copy of the kernels' decomposition). */
int32_t bs_work_items(int32_t num_tiles, int32_t dp_tiles, int64_t sk_iters, int32_t kb, int32_t units, int32_t unit,
                      int32_t* out, int32_t capacity);

/* The persistent tile order: fills out[3*t .. 3*t+2] = (batch, tile_row,
 * tile_col) of linear tile t for t < count (host copy of the mapping the
 * kernels use).  Pure host logic. */
bs_status bs_tile_order(int32_t grid_m, int32_t grid_n, int32_t batches, int32_t group_m,
                        int32_t* out, int64_t count);

/*
 * Synchronises `stream`, then reads and clears this device's error word,
 * which a kernel sets when one of its bounded waits gives up (instead of
 * hanging).  Returns BS_ERR_TIMEOUT and stores the code (0x1000 | role<<8 |
 * wait kind) in *code when it was set, BS_OK and 0 otherwise.  `code` may be
 * NULL.  Device work: one stream synchronisation and two small copies.
 */
bs_status bs_get_device_error(void* stream, uint32_t* code);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t bs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSGEMM_H */

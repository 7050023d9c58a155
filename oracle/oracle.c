/*
 * CPU oracle for the scaled low-precision GEMMs -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct statement of what the three
 * GPU entry points compute.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * Arithmetic (no blocking, no reordering beyond the definitions below):
 *   - e4m3 codes are decoded through a 256-entry table built from the format
 *     definition (sign, 4 exponent bits with bias 7, 3 mantissa bits,
 *     subnormals at exponent field 0, code S.1111.111 = NaN, no infinities).
 *   - FP8 block-scaled GEMM: for every output element the 128-deep K-block
 *     partial P_kb = sum_{k in kb} a[m,k] * b[k,n] is formed in fp64 (exact:
 *     every e4m3 x e4m3 product has <= 8 significant bits and lies in
 *     [2^-18, 2^17.6], so 128 of them sum without rounding), then
 *     y = sum_kb (scale_a[m,kb] * scale_b[kb, n/128]) * P_kb in fp64, kb
 *     ascending.  This is the dequantise-then-multiply definition
 *     out = (A_q . expand(scale_a)) @ (B_q . expand(scale_b)) written per
 *     block.  Alongside, S = sum_kb |scale_a*scale_b| * sum_{k in kb} |a*b|
 *     is returned for the acceptance bound.
 *       Sources: pytorch issue "torch._scaled_mm with blockwise scaling doesn't
 *       work with torch.compile" (the RuntimeError quoting scale_a (16640, 64),
 *       scale_b (64, 40) for M=16640, K=8192, N=5120 -- 1x128 groups for A,
 *       128x128 blocks for B); pytorch/torch/_inductor/kernel/mm.py,
 *       apply_scaling (the scale tensors multiply the accumulator).
 *   - INT8: acc = sum_k a*b accumulated in int64 and checked to fit int32,
 *     then y = ((float)acc * s_a[m]) * s_b[n], each step an fp32 RNE
 *     operation, and bf16 = RNE(y).
 *       Sources: pytorch/ao PR "Remove int_scaled_mm's dependency on triton
 *       for cpu" (int_scaled_matmul_cpu: _int_mm then .to(scales.dtype) *
 *       scales); pytorch/ao issue "Unify scaled INT8 matmul" (key-differences
 *       table: acc_i32.to(f32) x scale.to(f32), both scales fused).
 *   - FP8 with tensorwise or rowwise scales (and an optional bias): the exact
 *     fp64 dot product over all of K times scale_a * scale_b, plus bias[n]
 *     (see orc_fp8_rowwise for the sources).
 *   - Batched block-scaled GEMM: a loop over g of the FP8 definition with
 *     scale = 2^(byte - 127) decoded exactly from the e8m0 bytes (byte 255 is
 *     NaN).
 *       Source: ROCm/aiter PR "Add opus fp8 mxscale BMM kernels for gfx950"
 *       (Motivation: m-major layout x [M, G, K], w [G, N, K],
 *       x_scale [M, G, K/128], w_scale [G, N/128, K/128]).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Parallelism is OpenMP over output rows only; every element is computed by
 * one thread in the fixed order above, so results do not depend on threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_SHAPE 1
#define ORC_ERR_OVERFLOW 2
#define ORC_ERR_NOMEM 3

static double e4m3_value[256];
static int e4m3_built = 0;

static void build_e4m3_table(void)
{
    if (e4m3_built) return;
    for (int code = 0; code < 256; ++code) {
        const int sign = (code >> 7) & 1;
        const int expo = (code >> 3) & 0xF;
        const int mant = code & 0x7;
        double mag;
        if (expo == 0xF && mant == 0x7)
            mag = NAN;                                  /* the only NaN encoding */
        else if (expo == 0)
            mag = ldexp((double)mant / 8.0, 1 - 7);     /* subnormal: m/8 * 2^-6 */
        else
            mag = ldexp(1.0 + (double)mant / 8.0, expo - 7);
        e4m3_value[code] = sign ? -mag : mag;
    }
    e4m3_built = 1;
}

/* Fills out[256] with the decoded value of every e4m3 code. */
void orc_e4m3_table(double *out)
{
    build_e4m3_table();
    memcpy(out, e4m3_value, sizeof(e4m3_value));
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* rounding of an fp64 value to the output formats                           */
/* ------------------------------------------------------------------------ */

/* Round an fp64 value to bfloat16 (8 significant bits, fp32 exponent range)
 * with round-to-nearest-even, directly from fp64 (no intermediate fp32).
 * Returns the 16-bit pattern. */
uint16_t orc_bf16_from_f64(double v)
{
    if (isnan(v)) return 0x7FC0;
    const int neg = signbit(v) ? 1 : 0;
    const double a = fabs(v);
    uint16_t bits;
    if (a == 0.0) {
        bits = 0;
    } else {
        int e2;
        frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5, 1) */
        int q = (e2 - 1) - 7;          /* exponent of one bf16 ulp at a */
        if (q < -133) q = -133;        /* subnormal spacing 2^-133 */
        const double r = nearbyint(ldexp(a, -q));   /* ties to even */
        const double rounded = ldexp(r, q);
        if (rounded >= 0x1p128) {
            bits = 0x7F80;             /* overflow to infinity */
        } else {
            const float f = (float)rounded; /* exact: rounded is a bf16 value */
            uint32_t u;
            memcpy(&u, &f, 4);
            bits = (uint16_t)(u >> 16);
        }
    }
    return (uint16_t)(bits | (neg ? 0x8000 : 0));
}

void orc_round_bf16(const double *v, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_f64(v[i]);
}

void orc_round_f32(const double *v, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (float)v[i];  /* C conversion: RNE */
}

/* bf16 pattern of an fp32 value, round-to-nearest-even, NaN kept quiet. */
static uint16_t bf16_from_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x0040);
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* FP8 block-scaled GEMM core, scales already decoded to fp64                */
/* ------------------------------------------------------------------------ */

/* A: e4m3 codes, row m at A + m*lda.  B: e4m3 codes of B[K,N] stored K-major,
 * column n at B + n*ldb.  sa[m*KB + kb], sb[kb*NB + nb] in fp64.
 * Computes the rows listed in `rows` (all rows when rows == NULL; nrows is
 * then M) into y[i*N + n] and S[i*N + n]. */
static int fp8_core(const uint8_t *A, int64_t lda, const uint8_t *B, int64_t ldb,
                    const double *sa, const double *sb, int64_t M, int64_t N, int64_t K,
                    const int64_t *rows, int64_t nrows, double *y, double *S)
{
    if (K % 128 != 0 || M < 0 || N < 0 || K < 0) return ORC_ERR_SHAPE;
    build_e4m3_table();
    const int64_t KB = K / 128, NB = (N + 127) / 128;
    (void)NB;
    if (rows) {
        for (int64_t i = 0; i < nrows; ++i)
            if (rows[i] < 0 || rows[i] >= M) return ORC_ERR_SHAPE;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows ? rows[i] : i;
        const uint8_t *arow = A + m * lda;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t *bcol = B + n * ldb;
            double acc = 0.0, mag = 0.0;
            for (int64_t kb = 0; kb < KB; ++kb) {
                double p = 0.0, pabs = 0.0;
                for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
                    const double t = e4m3_value[arow[k]] * e4m3_value[bcol[k]];
                    p += t;
                    pabs += fabs(t);
                }
                const double s = sa[m * KB + kb] * sb[kb * NB + n / 128];
                acc += s * p;
                mag += fabs(s) * pabs;
            }
            y[i * N + n] = acc;
            S[i * N + n] = mag;
        }
    }
    return ORC_OK;
}

/* Operation 1: FP8 e4m3 A[M,K] x B[K,N], scale_a fp32 [M, K/128] with element
 * strides (sa_sm, sa_sk), scale_b fp32 [K/128, ceil(N/128)] with element
 * strides (sb_sk, sb_sn). */
int orc_fp8_blockwise(const uint8_t *A, int64_t lda, const uint8_t *B, int64_t ldb,
                      const float *scale_a, int64_t sa_sm, int64_t sa_sk,
                      const float *scale_b, int64_t sb_sk, int64_t sb_sn,
                      int64_t M, int64_t N, int64_t K,
                      const int64_t *rows, int64_t nrows, double *y, double *S)
{
    if (K % 128 != 0) return ORC_ERR_SHAPE;
    const int64_t KB = K / 128, NB = (N + 127) / 128;
    double *sa = (double *)malloc(sizeof(double) * (size_t)(M * KB + 1));
    double *sb = (double *)malloc(sizeof(double) * (size_t)(KB * NB + 1));
    if (!sa || !sb) { free(sa); free(sb); return ORC_ERR_NOMEM; }
    for (int64_t m = 0; m < M; ++m)
        for (int64_t kb = 0; kb < KB; ++kb)
            sa[m * KB + kb] = (double)scale_a[m * sa_sm + kb * sa_sk];
    for (int64_t kb = 0; kb < KB; ++kb)
        for (int64_t nb = 0; nb < NB; ++nb)
            sb[kb * NB + nb] = (double)scale_b[kb * sb_sk + nb * sb_sn];
    const int rc = fp8_core(A, lda, B, ldb, sa, sb, M, N, K, rows, rows ? nrows : M, y, S);
    free(sa);
    free(sb);
    return rc;
}

/* FP8 e4m3 A[M,K] x B[K,N] with tensorwise or rowwise fp32 scales and an
 * optional fp32 bias[N]:
 *   y[m,n] = (sum_k a[m,k] * b[k,n]) * (scale_a[m * sa_stride] * scale_b[n * sb_stride]) + bias[n]
 * sa_stride / sb_stride are 0 (one scale for the operand) or 1 (one per row of A
 * / column of B).  The dot product is exact in fp64 for K < 2^20 (every
 * product has <= 8 significant bits in [2^-18, 2^17.6]); the scale product is
 * exact in fp64; the scaling and bias add round once each in fp64.
 * S[m,n] = |scale_a * scale_b| * sum_k |a * b| for the acceptance bound.
 *   Sources: pytorch/torch/_inductor/kernel/mm.py, apply_scaling (tensorwise:
 *   accumulator * (a_scale * b_scale); rowwise: the per-row scale_a times the
 *   per-column scale_b) and tuned_scaled_mm (bias [N] broadcast over rows);
 *   the pytorch issue "torch._scaled_mm with blockwise scaling doesn't work
 *   with torch.compile" (RuntimeError: tensorwise scales are scalars, rowwise
 *   scale_a is (M, 1) and scale_b is (1, N)). */
int orc_fp8_rowwise(const uint8_t *A, int64_t lda, const uint8_t *B, int64_t ldb,
                    const float *scale_a, int64_t sa_stride, const float *scale_b, int64_t sb_stride,
                    const float *bias, int64_t M, int64_t N, int64_t K,
                    const int64_t *rows, int64_t nrows, double *y, double *S)
{
    if (M < 0 || N < 0 || K < 0 || K >= (1 << 20)) return ORC_ERR_SHAPE;
    if ((sa_stride != 0 && sa_stride != 1) || (sb_stride != 0 && sb_stride != 1)) return ORC_ERR_SHAPE;
    build_e4m3_table();
    if (!rows) nrows = M;
    for (int64_t i = 0; rows && i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= M) return ORC_ERR_SHAPE;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const int64_t m = rows ? rows[i] : i;
        const uint8_t *arow = A + m * lda;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t *bcol = B + n * ldb;
            double p = 0.0, pabs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const double t = e4m3_value[arow[k]] * e4m3_value[bcol[k]];
                p += t;
                pabs += fabs(t);
            }
            const double s = (double)scale_a[m * sa_stride] * (double)scale_b[n * sb_stride];
            y[i * N + n] = p * s + (bias ? (double)bias[n] : 0.0);
            S[i * N + n] = fabs(s) * pabs;
        }
    }
    return ORC_OK;
}

static double e8m0_value(uint8_t byte)
{
    if (byte == 0xFF) return NAN;
    return ldexp(1.0, (int)byte - 127);
}

/* Operation 3: for g in [0, G): out[m, g, n] = FP8 block-scaled product of
 * x[:, g, :] (row m at x + m*x_sm + g*x_sg) and w[g] ([N, K] contiguous, at
 * w + g*w_sg), scales 2^(byte-127) from x_scale [M, G, K/128] and
 * w_scale [G, ceil(N/128), K/128] (both contiguous).  y and S are laid out
 * [nrows][G][N]. */
int orc_bmm_blockscale(const uint8_t *x, int64_t x_sm, int64_t x_sg,
                       const uint8_t *w, int64_t w_sg, int64_t w_sn,
                       const uint8_t *x_scale, const uint8_t *w_scale,
                       int64_t M, int64_t G, int64_t N, int64_t K,
                       const int64_t *rows, int64_t nrows, double *y, double *S)
{
    if (K % 128 != 0) return ORC_ERR_SHAPE;
    const int64_t KB = K / 128, NB = (N + 127) / 128;
    const int64_t R = rows ? nrows : M;
    double *sa = (double *)malloc(sizeof(double) * (size_t)(M * KB + 1));
    double *sb = (double *)malloc(sizeof(double) * (size_t)(KB * NB + 1));
    double *yg = (double *)malloc(sizeof(double) * (size_t)(R * N + 1));
    double *Sg = (double *)malloc(sizeof(double) * (size_t)(R * N + 1));
    if (!sa || !sb || !yg || !Sg) { free(sa); free(sb); free(yg); free(Sg); return ORC_ERR_NOMEM; }
    int rc = ORC_OK;
    for (int64_t g = 0; g < G && rc == ORC_OK; ++g) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t kb = 0; kb < KB; ++kb)
                sa[m * KB + kb] = e8m0_value(x_scale[(m * G + g) * KB + kb]);
        for (int64_t kb = 0; kb < KB; ++kb)
            for (int64_t nb = 0; nb < NB; ++nb)
                sb[kb * NB + nb] = e8m0_value(w_scale[(g * NB + nb) * KB + kb]);
        /* x[:, g, :] is a row-major [M, K] matrix with row stride x_sm. */
        rc = fp8_core(x + g * x_sg, x_sm, w + g * w_sg, w_sn, sa, sb, M, N, K,
                      rows, R, yg, Sg);
        for (int64_t i = 0; i < R && rc == ORC_OK; ++i)
            for (int64_t n = 0; n < N; ++n) {
                y[(i * G + g) * N + n] = yg[i * N + n];
                S[(i * G + g) * N + n] = Sg[i * N + n];
            }
    }
    free(sa); free(sb); free(yg); free(Sg);
    return rc;
}

/* Operation 2: INT8 A[M,K] (row m at A + m*lda) x B[K,N] stored K-major
 * (column n at B + n*ldb).  acc is exact; y = ((float)acc * s_a[m]) * s_b[n]
 * in fp32 with that fixed order (s_b == NULL: y = (float)acc * s_a[m];
 * s_a == NULL: y = (float)acc).  Outputs are laid out [nrows][N]; any output
 * pointer may be NULL. */
int orc_int_scaled_mm(const int8_t *A, int64_t lda, const int8_t *B, int64_t ldb,
                      const float *s_a, const float *s_b,
                      int64_t M, int64_t N, int64_t K,
                      const int64_t *rows, int64_t nrows,
                      int32_t *acc_out, float *y_out, uint16_t *bf16_out)
{
    const int64_t R = rows ? nrows : M;
    if (rows)
        for (int64_t i = 0; i < nrows; ++i)
            if (rows[i] < 0 || rows[i] >= M) return ORC_ERR_SHAPE;
    int overflow = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : overflow)
    for (int64_t i = 0; i < R; ++i) {
        const int64_t m = rows ? rows[i] : i;
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k)
                acc += (int64_t)A[m * lda + k] * (int64_t)B[n * ldb + k];
            if (acc > INT32_MAX || acc < INT32_MIN) overflow = 1;
            const int32_t a32 = (int32_t)acc;
            float f = (float)a32;
            if (s_a) f = f * s_a[m];
            if (s_b) f = f * s_b[n];
            if (acc_out) acc_out[i * N + n] = a32;
            if (y_out) y_out[i * N + n] = f;
            if (bf16_out) bf16_out[i * N + n] = bf16_from_f32(f);
        }
    }
    return overflow ? ORC_ERR_OVERFLOW : ORC_OK;
}

/*
 * e4m3 encoding with round-to-nearest-even and saturation, straight from the
 * decode table: the finite magnitudes are the table values of codes 0..126
 * (ascending); v is mapped to the nearest one, a tie to the code with an even
 * mantissa (last bit 0), anything beyond 448 to 448, NaN to 0x7F.  The sign
 * is carried separately (so -0.0 and values rounding to zero keep the sign
 * bit, as the format's own conversion does).
 */
uint8_t orc_e4m3_from_f64(double v)
{
    build_e4m3_table();
    if (isnan(v)) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;                 /* saturation */
    int lo = 0, hi = 126;                                /* table[lo] <= a < table[hi] */
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (e4m3_value[mid] <= a) lo = mid; else hi = mid;
    }
    const double dlo = a - e4m3_value[lo], dhi = e4m3_value[hi] - a;
    int code;
    if (dlo < dhi) code = lo;
    else if (dhi < dlo) code = hi;
    else code = (lo & 1) ? hi : lo;                      /* tie: even mantissa */
    return sign | (uint8_t)code;
}

void orc_e4m3_encode(const double *v, uint8_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_f64(v[i]);
}

/* fp32 group scale: amax / 448 in fp32, and 1 where that quotient is zero:
 * an all-zero group, or one whose largest magnitude is below 448 * 2^-150, so
 * that the fp32 quotient underflows (a zero scale would leave the codes
 * undefined).  Both cases keep the all-zero group's convention. */
static float group_scale_f32(float amax)
{
    const float s = amax / 448.0f;
    return s == 0.0f ? 1.0f : s;
}

/* e8m0 group scale byte: clamp(e + 127, 0, 254), e the smallest integer with
 * amax <= 448 * 2^e (0 for an all-zero group). */
static int group_scale_e8m0(float amax)
{
    int e = 0;
    if (amax != 0.0f) {
        e = ilogb((double)amax) - 10;                /* 448 * 2^e < amax here */
        while (!((double)amax <= ldexp(448.0, e))) ++e;
    }
    int byte = e + 127;
    if (byte < 0) byte = 0;
    if (byte > 254) byte = 254;
    return byte;
}

/* The e4m3 code of element v of a group with fp32 scale s (fmt 0) or e8m0
 * byte b (fmt 1). */
static uint8_t group_code(float v, int fmt, float s, int b)
{
    if (fmt == 0) return orc_e4m3_from_f64((double)(v / s));
    return orc_e4m3_from_f64(ldexp((double)v, -(b - 127)));
}

/*
 * 1x128 activation-group quantisation (the recipe the blockwise operation's
 * inputs follow): for row m and group g (elements 128g .. min(128g+128, K)-1)
 *   amax = max |x|
 *   fmt 0: scale = fp32(amax / 448) (1 when that is zero),
 *          q = e4m3_rne(sat(fp32(x / scale)))
 *   fmt 1: e = the smallest integer with amax <= 448 * 2^e, i.e.
 *          ceil(log2(amax / 448)) (0 when amax == 0); byte = clamp(e + 127,
 *          0, 254); q = e4m3_rne(sat(x * 2^-(byte - 127)))
 * x is fp32 here (bf16 inputs widen exactly).  scale_f32 / scale_e8m0 are
 * [M, ceil(K/128)] row-major; q is [M, K] with row stride ldq.
 *   Sources: pytorch issue "torch._scaled_mm with blockwise scaling doesn't
 *   work with torch.compile" (1x128 groups of A with an fp32 scale each,
 *   scale_a [M, K/128]); ROCm/aiter PR "Add opus fp8 mxscale BMM kernels for
 *   gfx950" (e8m0 power-of-two scales per 128-element group).  The amax / 448
 *   scale and the saturating RNE cast are the plain reading of "scaled e4m3":
 *   448 is the largest finite e4m3 magnitude.
 */
int orc_quantize_1x128(const float *x, int64_t M, int64_t K, int64_t ldx, int fmt,
                       uint8_t *q, int64_t ldq, float *scale_f32, uint8_t *scale_e8m0)
{
    if (M < 0 || K < 0 || ldx < K || ldq < K || (fmt != 0 && fmt != 1)) return ORC_ERR_SHAPE;
    const int64_t KB = (K + 127) / 128;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < KB; ++g) {
            const int64_t k0 = 128 * g, k1 = k0 + 128 < K ? k0 + 128 : K;
            float amax = 0.0f;
            for (int64_t k = k0; k < k1; ++k) {
                const float a = fabsf(x[m * ldx + k]);
                if (a > amax) amax = a;
            }
            const float s = group_scale_f32(amax);
            const int b = group_scale_e8m0(amax);
            if (fmt == 0) scale_f32[m * KB + g] = s;
            else scale_e8m0[m * KB + g] = (uint8_t)b;
            for (int64_t k = k0; k < k1; ++k) q[m * ldq + k] = group_code(x[m * ldx + k], fmt, s, b);
        }
    }
    return ORC_OK;
}

/*
 * Quantisation for the backward pass of a blockwise fp8 linear layer: the
 * codes are written transposed, so that the dimension the backward GEMMs
 * contract over (the rows of x) becomes the contiguous one.  x is [R, C]
 * (row stride ldx); q_t is [C, R] (row stride ldq), q_t[c][r] the code of
 * x[r][c].  Groups, with the same scale and code rules as orc_quantize_1x128:
 *   group 0 (128x1): rows 128rb .. min(128rb + 128, R) - 1 of one column c;
 *                    scale[c * RB + rb]  ([C, RB], RB = ceil(R / 128)), i.e.
 *                    the 1x128 groups of x transposed
 *   group 1 (128x128): the block rows 128rb.., columns 128cb..;
 *                    scale[rb * CB + cb]  ([RB, CB], CB = ceil(C / 128))
 *   Sources: pytorch issue "torch._scaled_mm with blockwise scaling doesn't
 *   work with torch.compile" (the forward and backward benchmark of the
 *   blockwise fp8 linear layer; the 1x128 activation groups with scale_a
 *   [M, K/128] and the 128x128 weight blocks with scale_b [K/128, N/128] are
 *   the only two group shapes it fixes, so the backward operands take those
 *   two shapes along their contraction dimension).
 */
int orc_quantize_t(const float *x, int64_t R, int64_t C, int64_t ldx, int group, int fmt,
                   uint8_t *q_t, int64_t ldq, float *scale_f32, uint8_t *scale_e8m0)
{
    if (R < 0 || C < 0 || ldx < C || ldq < R || (fmt != 0 && fmt != 1) || (group != 0 && group != 1))
        return ORC_ERR_SHAPE;
    const int64_t RB = (R + 127) / 128, CB = (C + 127) / 128;
    const int64_t CW = group == 0 ? 1 : 128;          /* columns per group */
    const int64_t NG = group == 0 ? C : CB;            /* groups per row block */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t gi = 0; gi < RB * NG; ++gi) {
        const int64_t rb = gi / NG, g = gi % NG;
        const int64_t r0 = 128 * rb, r1 = r0 + 128 < R ? r0 + 128 : R;
        const int64_t c0 = g * CW, c1 = c0 + CW < C ? c0 + CW : C;
        float amax = 0.0f;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) {
                const float a = fabsf(x[r * ldx + c]);
                if (a > amax) amax = a;
            }
        const float s = group_scale_f32(amax);
        const int b = group_scale_e8m0(amax);
        const int64_t si = group == 0 ? g * RB + rb : rb * CB + g;
        if (fmt == 0) scale_f32[si] = s;
        else scale_e8m0[si] = (uint8_t)b;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) q_t[c * ldq + r] = group_code(x[r * ldx + c], fmt, s, b);
    }
    return ORC_OK;
}

/*
 * 128x128 block quantisation in the input's own orientation, for the forward
 * GEMM's weight operand: a weight W [N, K] (x [R, C], row stride ldx) becomes
 * codes q [R, C] (row stride ldq), q[r][c] the code of x[r][c], with one scale
 * per block of rows 128rb .. min(128rb + 128, R) - 1 and columns
 * 128cb .. min(128cb + 128, C) - 1, scale[rb * CB + cb] ([RB, CB]), and the
 * scale and code rules of orc_quantize_1x128.  For x = W [N, K] the codes are
 * the B_t [N, K] of the blockwise GEMM and the transposed scale matrix is its
 * scale_b [K/128, N/128].
 *   Source: pytorch issue "torch._scaled_mm with blockwise scaling doesn't
 *   work with torch.compile" (128x128 weight blocks with one fp32 scale each,
 *   scale_b (64, 40) for K = 8192, N = 5120).
 */
int orc_quantize_128x128(const float *x, int64_t R, int64_t C, int64_t ldx, int fmt,
                         uint8_t *q, int64_t ldq, float *scale_f32, uint8_t *scale_e8m0)
{
    if (R < 0 || C < 0 || ldx < C || ldq < C || (fmt != 0 && fmt != 1)) return ORC_ERR_SHAPE;
    const int64_t RB = (R + 127) / 128, CB = (C + 127) / 128;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t bi = 0; bi < RB * CB; ++bi) {
        const int64_t rb = bi / CB, cb = bi % CB;
        const int64_t r0 = 128 * rb, r1 = r0 + 128 < R ? r0 + 128 : R;
        const int64_t c0 = 128 * cb, c1 = c0 + 128 < C ? c0 + 128 : C;
        float amax = 0.0f;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) {
                const float a = fabsf(x[r * ldx + c]);
                if (a > amax) amax = a;
            }
        const float s = group_scale_f32(amax);
        const int b = group_scale_e8m0(amax);
        if (fmt == 0) scale_f32[rb * CB + cb] = s;
        else scale_e8m0[rb * CB + cb] = (uint8_t)b;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) q[r * ldq + c] = group_code(x[r * ldx + c], fmt, s, b);
    }
    return ORC_OK;
}

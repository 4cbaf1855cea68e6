/*
 * Oracle for the dense GEMM path -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
 * leg may load this library.  The GPU library never links or calls it, and it
 * shares no code, header or constant table with the GPU path.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *
 *   C[i][j] = sum_{k=0}^{K-1} a(i,k) * b(k,j)            (evaluated in fp64,
 *                                                          natural k order)
 *
 * following the matrix product C_{MxN} = A_{MxK} B_{KxN} of
 * "GPU 执行模型" (wineandchord.com), section "Tile 的容量约束".  B is stored
 * K-major, i.e. as an N x K array: b(k,j) = B[j*ldb + k].  A is row-major:
 * a(i,k) = A[i*lda + k].  The fp64 sum is returned unrounded; the callers
 * round it once to the output type (fp32 or bf16, round-to-nearest-even).
 *
 * The block-scaled variant follows the "块量化 MMA / Block-Scaled MMA" item of
 * "Modern GPU Programming For MLSys - 书籍总结" (omica.com.cn), sections 2.4
 * and 2.6: every element is an FP8 E4M3 code, and every run of 32 consecutive
 * K elements of a row of A (or of a row of the K-major B) shares one E8M0
 * scale byte.  The pages name the mechanism only; the element and scale
 * encodings are the OCP microscaling formats, decoded here from their
 * definitions.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (see build.py).
 * -ffp-contract=off keeps every multiply and add separately rounded, so the
 * k-order sum is exactly the loop as written.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- codecs -- */

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.  It is
 * the top half of an IEEE binary32, decoded here field by field. */
double oracle_bf16_to_f64(uint16_t bits) {
    int sign = (bits >> 15) & 1;
    int e = (bits >> 7) & 0xFF;
    int f = bits & 0x7F;
    double mag;
    if (e == 0xFF) {
        mag = (f == 0) ? INFINITY : NAN;
    } else if (e == 0) {
        mag = ldexp((double)f, -126 - 7);            /* subnormal: 0.f * 2^-126 */
    } else {
        mag = ldexp((double)(128 + f), e - 127 - 7);  /* 1.f * 2^(e-127) */
    }
    return sign ? -mag : mag;
}

/* FP8 E4M3 (OCP "fn" flavour): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; no infinities; S.1111.111 is NaN; max finite 448. */
double oracle_e4m3_to_f64(uint8_t bits) {
    int sign = (bits >> 7) & 1;
    int e = (bits >> 3) & 0xF;
    int m = bits & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) {
        mag = NAN;
    } else if (e == 0) {
        mag = ldexp((double)m, -6 - 3);              /* subnormal: 0.m * 2^-6 */
    } else {
        mag = ldexp((double)(8 + m), e - 7 - 3);     /* 1.m * 2^(e-7) */
    }
    return sign ? -mag : mag;
}

/* E8M0 scale: an unsigned biased exponent, value 2^(e-127); 0xFF is NaN. */
double oracle_e8m0_to_f64(uint8_t bits) {
    if (bits == 0xFF) return NAN;
    return ldexp(1.0, (int)bits - 127);
}

/* Round an fp64 value to the nearest bfloat16, ties to even, directly from
 * fp64 (no intermediate binary32, so there is no double rounding).
 * Overflow goes to infinity, NaN stays NaN (quiet, sign kept). */
uint16_t oracle_f64_to_bf16_rne(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0);
    if (isinf(x)) return (uint16_t)(sign | 0x7F80);
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);                   /* a = f * 2^e2, f in [0.5, 1) */
    int exp_unbiased = e2 - 1;       /* a = 1.xxx * 2^exp_unbiased */
    if (exp_unbiased < -126) exp_unbiased = -126;   /* subnormal range: fixed quantum */
    /* quantum (unit in the last place) of bf16 at this binade: 2^(exp-7) */
    double q = ldexp(1.0, exp_unbiased - 7);
    double n = a / q;                /* exact: power-of-two division */
    double r = nearbyint(n);         /* default rounding mode: nearest, ties to even */
    double v = r * q;                /* exact */
    /* re-encode v (it may have rounded down to zero or up into the next binade) */
    if (v == 0.0) return sign;
    if (v >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    int ve2;
    double vf = frexp(v, &ve2);
    int ve = ve2 - 1;
    if (ve < -126) {
        /* subnormal: fraction field = v / 2^-133 */
        uint16_t frac = (uint16_t)ldexp(v, 133);
        return (uint16_t)(sign | frac);
    }
    uint16_t frac = (uint16_t)(ldexp(vf, 8) - 128.0);   /* vf in [0.5,1): 1.f * 2^7 */
    uint16_t bexp = (uint16_t)(ve + 127);
    return (uint16_t)(sign | (bexp << 7) | frac);
}

/* Round an fp64 value to binary32, ties to even (the C conversion under the
 * default IEEE rounding mode). */
float oracle_f64_to_f32_rne(double x) { return (float)x; }

/* ------------------------------------------------------------ GEMM core -- */

/* C[i*ldc + j] = sum_k A[i*lda + k] * B[j*ldb + k], fp64, natural k order.
 * Rows of C are independent and are split across OpenMP threads; the per
 * element summation order is the plain loop's. */
void oracle_gemm_f64(const double *A, int64_t lda, const double *B, int64_t ldb,
                     double *C, int64_t ldc, int64_t M, int64_t N, int64_t K) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i) {
        const double *a = A + i * lda;
        for (int64_t j = 0; j < N; ++j) {
            const double *b = B + j * ldb;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[k] * b[k];
            C[i * ldc + j] = acc;
        }
    }
}

/* Sum_k |a(i,k) * b(k,j)|: the magnitude that scales the tolerance. */
void oracle_gemm_abs_f64(const double *A, int64_t lda, const double *B, int64_t ldb,
                         double *C, int64_t ldc, int64_t M, int64_t N, int64_t K) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i) {
        const double *a = A + i * lda;
        for (int64_t j = 0; j < N; ++j) {
            const double *b = B + j * ldb;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += fabs(a[k] * b[k]);
            C[i * ldc + j] = acc;
        }
    }
}

/* ------------------------------------------------- decode whole matrices -- */

void oracle_decode_bf16(const uint16_t *src, double *dst, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) dst[i] = oracle_bf16_to_f64(src[i]);
}

void oracle_decode_e4m3(const uint8_t *src, double *dst, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) dst[i] = oracle_e4m3_to_f64(src[i]);
}

/* Block-scaled operand: X is rows x K E4M3 codes with leading dimension ldx;
 * S is rows x (K/32) E8M0 bytes with leading dimension lds.  Output is the
 * dense fp64 value x(r,k) * 2^(S[r][k/32]-127), rows x K, leading dim K.
 * Each product of an E4M3 value and a power of two is exact in fp64. */
void oracle_decode_mx_operand(const uint8_t *X, int64_t ldx, const uint8_t *S, int64_t lds,
                              double *dst, int64_t rows, int64_t K) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            dst[r * K + k] = oracle_e4m3_to_f64(X[r * ldx + k]) *
                             oracle_e8m0_to_f64(S[r * lds + k / 32]);
        }
    }
}

void oracle_round_f32(const double *src, float *dst, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) dst[i] = oracle_f64_to_f32_rne(src[i]);
}

void oracle_round_bf16(const double *src, uint16_t *dst, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) dst[i] = oracle_f64_to_bf16_rne(src[i]);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

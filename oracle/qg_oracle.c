/*
 * qg_oracle.c -- plain CPU oracle for the FP4 quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library under quantize_gemm_b200/csrc.
 *
 * What it computes is the plain definition of the method described in the
 * QbitAI write-up "微软首创FP4训练框架，训练效果媲美BF16" (news.movedaos.com/post/4103,
 * a summary of arXiv 2501.17116, "Optimizing Large Language Model Training
 * Using FP4 Quantization"), cited below as [FP4-writeup] with the paragraph:
 *
 *   [FP4-writeup, E2M1]       the FP4 format: 1 sign, 2 exponent, 1 mantissa bit
 *   [FP4-writeup, granularity] W quantized per column (channel-wise), A per row
 *                              (token-wise)
 *   [FP4-writeup, ScaleShift] scale into [-1, 1], then map onto the FP4 range,
 *                              then round to the nearest FP4 value by table lookup
 *   [FP4-writeup, outliers]   quantile search for the largest |A|, clamp to the
 *                              threshold (A_clamped), sparse compensation
 *                              matrix dA = A - A_clamped
 *
 * Readings where the page is silent (each is listed in the design notes):
 *   - ScaleShift is multiplicative: r = fp32(6 / amax), q = round(fp32(x * r)),
 *     s = fp32(amax / 6), dequantized value = grid(q) * s.
 *   - round-to-nearest ties go to the even code (mantissa bit 0); the sign bit
 *     is the sign bit of the input, so -0.1 encodes as 0x8 (negative zero).
 *   - the quantile is the plain order statistic: sort |A| over the whole
 *     tensor, T = sorted[k], k = ceil(alpha * n) - 1 evaluated in double.
 *   - entries with |a| == T are not clamped; dA is non-zero where |a| > T.
 *   - dA values are kept in double (a - sign(a) * T evaluated in double).
 *   - the correction added to the GEMM is dA * W with W unquantized.
 *   - a row (column) whose amax is 0, or so small that 6 / amax overflows in
 *     fp32, gets r = 0 and s = 0: its codes carry only sign bits.
 *
 * Layouts: A is M x K row-major, W is K x N row-major.  Packed codes hold two
 * E2M1 codes per byte, the even k in the low nibble.  Row codes are M x K/2;
 * column codes are stored transposed, N x K/2 (K contiguous).
 *
 * Floating point: compiled without fast-math and without FMA contraction, so
 * every fp32 operation below is one IEEE correctly rounded operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* [FP4-writeup, E2M1]: magnitudes of the eight codes s=0, eem = 000 .. 111.  */
static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(uint8_t code) {
    double mag = E2M1_GRID[code & 7u];
    return (code & 8u) ? -mag : mag;
}

/* [FP4-writeup, ScaleShift]: "round to the nearest FP4 value by table lookup".
 * Walk the table of midpoints between neighbouring grid values; the first
 * midpoint above |x| gives the code; a value exactly on a midpoint takes the
 * neighbour with the even code.  Past the last midpoint the code saturates
 * at 6.  NaN is rejected before this is called.                             */
uint8_t orc_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 8u : 0u;
    double m = fabs((double)x);
    for (int i = 0; i < 7; ++i) {
        double mid = 0.5 * (E2M1_GRID[i] + E2M1_GRID[i + 1]);
        if (m < mid) return (uint8_t)(sign | (uint8_t)i);
        if (m == mid) return (uint8_t)(sign | (uint8_t)((i % 2 == 0) ? i : i + 1));
    }
    return (uint8_t)(sign | 7u);
}

/* One code per input element (unpacked), for encoder tests. */
void orc_e2m1_encode_array(const float* x, int64_t n, uint8_t* codes) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) codes[i] = orc_e2m1_encode(x[i]);
}

/* Encode the n consecutive fp32 bit patterns start, start+1, ... and pack
 * them two per byte (even index in the low nibble).  n must be even.  Used
 * by the exhaustive encoder sweep over all 2^32 patterns.                   */
void orc_e2m1_encode_bits_packed(uint32_t start, int64_t n, uint8_t* packed) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n / 2; ++j) {
        uint32_t b0 = start + (uint32_t)(2 * j), b1 = b0 + 1u;
        float x0, x1;
        memcpy(&x0, &b0, 4);
        memcpy(&x1, &b1, 4);
        uint8_t c0 = isnan(x0) ? 0u : orc_e2m1_encode(x0);
        uint8_t c1 = isnan(x1) ? 0u : orc_e2m1_encode(x1);
        packed[j] = (uint8_t)(c0 | (c1 << 4));
    }
}

/* ------------------------------------------------------------------------ */
/* [FP4-writeup, outliers]: quantile threshold.  Plain order statistic.      */
int64_t orc_quantile_rank(double alpha, int64_t n) {
    int64_t k = (int64_t)ceil(alpha * (double)n) - 1;
    if (k < 0) k = 0;
    if (k > n - 1) k = n - 1;
    return k;
}

static int cmp_float(const void* a, const void* b) {
    float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

/* T = sorted(|A|)[k] over all n entries of the tensor. */
float orc_threshold(const float* A, int64_t n, double alpha) {
    float* mag = (float*)malloc((size_t)n * sizeof(float));
    if (!mag) return NAN;
    for (int64_t i = 0; i < n; ++i) mag[i] = fabsf(A[i]);
    qsort(mag, (size_t)n, sizeof(float), cmp_float);
    float T = mag[orc_quantile_rank(alpha, n)];
    free(mag);
    return T;
}

/* [FP4-writeup, outliers]: A_clamped = clamp(A, -T, T) and the sparse
 * compensation dA = A - A_clamped in CSR form (rows ascending, columns
 * ascending within a row).  A_c may be NULL.  Returns nnz, or -1 when the
 * capacity is too small.                                                    */
int64_t orc_clamp_compensate(const float* A, int64_t M, int64_t K, float T, float* A_c,
                             int32_t* row_ptr, int32_t* col, double* val, int64_t cap) {
    int64_t nnz = 0;
    row_ptr[0] = 0;
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t k = 0; k < K; ++k) {
            float a = A[i * K + k];
            float ac = (fabsf(a) > T) ? copysignf(T, a) : a;
            if (A_c) A_c[i * K + k] = ac;
            if (fabsf(a) > T) {
                if (nnz >= cap) return -1;
                col[nnz] = (int32_t)k;
                val[nnz] = (double)a - (double)ac;
                ++nnz;
            }
        }
        row_ptr[i + 1] = (int32_t)nnz;
    }
    return nnz;
}

/* ------------------------------------------------------------------------ */
/* [FP4-writeup, ScaleShift]: r maps [-amax, amax] onto [-6, 6]; s undoes it. */
void orc_scale_factors(float amax, float* r_out, float* s_out) {
    float r = 6.0f / amax;
    if (amax == 0.0f || isinf(r)) {
        *r_out = 0.0f;
        *s_out = 0.0f;
    } else {
        *r_out = r;
        *s_out = amax / 6.0f;
    }
}

/* [FP4-writeup, granularity]: token-wise (row) quantization of A.           */
void orc_quantize_rows(const float* A, int64_t M, int64_t K, uint8_t* codes, float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        const float* a = A + i * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            if (fabsf(a[k]) > amax) amax = fabsf(a[k]);
        float r, s;
        orc_scale_factors(amax, &r, &s);
        scales[i] = s;
        for (int64_t k = 0; k < K; k += 2) {
            float x0 = a[k] * r, x1 = a[k + 1] * r;
            codes[i * (K / 2) + k / 2] =
                (uint8_t)(orc_e2m1_encode(x0) | (orc_e2m1_encode(x1) << 4));
        }
    }
}

/* [FP4-writeup, granularity]: channel-wise (column) quantization of W (K x N),
 * codes written transposed as N x K/2 so that the GEMM reads both operands
 * with K contiguous.                                                        */
void orc_quantize_cols(const float* W, int64_t K, int64_t N, uint8_t* codesT, float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            if (fabsf(W[k * N + j]) > amax) amax = fabsf(W[k * N + j]);
        float r, s;
        orc_scale_factors(amax, &r, &s);
        scales[j] = s;
        for (int64_t k = 0; k < K; k += 2) {
            float x0 = W[k * N + j] * r, x1 = W[(k + 1) * N + j] * r;
            codesT[j * (K / 2) + k / 2] =
                (uint8_t)(orc_e2m1_encode(x0) | (orc_e2m1_encode(x1) << 4));
        }
    }
}

/* Fused activation path: threshold, clamp, dA, then row quantization of
 * A_clamped.  A_c scratch is allocated here.  Returns nnz or -1.            */
int64_t orc_quantize_act(const float* A, int64_t M, int64_t K, double alpha, uint8_t* codes,
                         float* scales, int32_t* row_ptr, int32_t* col, double* val,
                         int64_t cap, float* T_out) {
    float T = orc_threshold(A, M * K, alpha);
    float* A_c = (float*)malloc((size_t)(M * K) * sizeof(float));
    if (!A_c) return -1;
    int64_t nnz = orc_clamp_compensate(A, M, K, T, A_c, row_ptr, col, val, cap);
    orc_quantize_rows(A_c, M, K, codes, scales);
    free(A_c);
    *T_out = T;
    return nnz;
}

/* ------------------------------------------------------------------------ */
/* The FP4 product of the codes, acc_ij = sum_k e2m1(qA_ik) * e2m1(qW_jk),
 * in double (every partial sum is a multiple of 0.25 well inside 2^53, so
 * the sum is exact).  Computed for the listed rows only (rows == NULL means
 * all M rows); acc has one row of N per listed row.                         */
void orc_gemm_acc_rows(const uint8_t* codesA, const uint8_t* codesWT, int64_t M, int64_t N,
                       int64_t K, const int64_t* rows, int64_t nrows, double* acc) {
    int64_t R = rows ? nrows : M;
    double* wt = (double*)malloc((size_t)(N * K) * sizeof(double));
    if (!wt) return;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = codesWT[j * (K / 2) + k / 2];
            wt[j * K + k] = orc_e2m1_value((k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 15u));
        }
#pragma omp parallel
    {
        double* arow = (double*)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < R; ++r) {
            int64_t i = rows ? rows[r] : r;
            for (int64_t k = 0; k < K; ++k) {
                uint8_t b = codesA[i * (K / 2) + k / 2];
                arow[k] = orc_e2m1_value((k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 15u));
            }
            for (int64_t j = 0; j < N; ++j) {
                const double* w = wt + j * K;
                double sum = 0.0;
                for (int64_t k = 0; k < K; ++k) sum += arow[k] * w[k];
                acc[r * N + j] = sum;
            }
        }
        free(arow);
    }
    free(wt);
}

/* Y_ij = acc_ij * s_i * t_j + sum_k dA_ik * W_kj, all in double, for the
 * listed rows (rows == NULL: all).  acc holds one row of N per listed row.  */
void orc_linear_y_rows(const double* acc, const float* sA, const float* sW,
                       const int32_t* row_ptr, const int32_t* col, const double* val,
                       const float* W, int64_t M, int64_t N, int64_t K, const int64_t* rows,
                       int64_t nrows, double* Y) {
    (void)K;
    int64_t R = rows ? nrows : M;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        int64_t i = rows ? rows[r] : r;
        double* y = Y + r * N;
        for (int64_t j = 0; j < N; ++j)
            y[j] = acc[r * N + j] * (double)sA[i] * (double)sW[j];
        for (int32_t p = row_ptr[i]; p < row_ptr[i + 1]; ++p) {
            const float* w = W + (int64_t)col[p] * N;
            for (int64_t j = 0; j < N; ++j) y[j] += val[p] * (double)w[j];
        }
    }
}

/* dA * W alone (the correction term), in double, all rows. */
void orc_spmm(const int32_t* row_ptr, const int32_t* col, const double* val, const float* W,
              int64_t M, int64_t N, double* C) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double* c = C + i * N;
        for (int64_t j = 0; j < N; ++j) c[j] = 0.0;
        for (int32_t p = row_ptr[i]; p < row_ptr[i + 1]; ++p) {
            const float* w = W + (int64_t)col[p] * N;
            for (int64_t j = 0; j < N; ++j) c[j] += val[p] * (double)w[j];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4 block-scaled variant.
 *
 * [MX-lecture] "FP4量化训练的硬件挑战：NVIDIA Blackwell架构上的微缩放格式（Micro-
 * scaling）实现" (zyxy.net/?p=24232), section 3 on micro-scaling: split the
 * tensor into small groups, give each group its own scale (max scaling: from
 * the group's largest magnitude), divide the group by its scale and round to
 * FP4, multiply back to dequantize.
 * [LP-survey] (10100.com/article/123065115), custom number formats: micro-
 * scaling pairs a per-block scale, usually E8M0 (a bare power of two), with
 * low-precision elements.
 *
 * Readings: groups are 32 consecutive elements along the contraction
 * dimension (K); the block scale is the smallest power of two X = 2^e with
 * 6 * X >= amax (the block's largest magnitude lands inside the E2M1 range
 * without clipping), e limited to [-127, 127] and stored as the E8M0 byte
 * e + 127; a block whose amax is 0 gets e = -127.  Codes are
 * E2M1(fp32(x * 2^-e)) with the encoder above; the dequantized value of a
 * code is grid(code) * 2^e.                                                 */
int orc_mx_exponent(float amax) {
    int e = -127;
    while (e < 127 && ldexp(6.0, e) < (double)amax) ++e;
    return e;
}

/* One block of n (<= 32) values with stride `stride`: codes into out_codes
 * (unpacked, one per value), the E8M0 byte returned.                        */
static uint8_t mx_block(const float* x, int64_t stride, int n, uint8_t* out_codes) {
    float amax = 0.0f;
    for (int t = 0; t < n; ++t)
        if (fabsf(x[t * stride]) > amax) amax = fabsf(x[t * stride]);
    const int e = orc_mx_exponent(amax);
    const float inv = ldexpf(1.0f, -e);
    for (int t = 0; t < n; ++t) out_codes[t] = orc_e2m1_encode(x[t * stride] * inv);
    return (uint8_t)(e + 127);
}

/* Rows of A (M x K, K % 32 == 0): codes M x K/2, E8M0 scales M x K/32.      */
void orc_mx_quantize_rows(const float* A, int64_t M, int64_t K, uint8_t* codes,
                          uint8_t* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        uint8_t q[32];
        for (int64_t b = 0; b < K / 32; ++b) {
            scales[i * (K / 32) + b] = mx_block(A + i * K + 32 * b, 1, 32, q);
            for (int t = 0; t < 32; t += 2)
                codes[i * (K / 2) + 16 * b + t / 2] = (uint8_t)(q[t] | (q[t + 1] << 4));
        }
    }
}

/* Columns of W (K x N, K % 32 == 0), blocks along K: codes written transposed
 * N x K/2, scales N x K/32.                                                 */
void orc_mx_quantize_cols(const float* W, int64_t K, int64_t N, uint8_t* codesT,
                          uint8_t* scalesT) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
        uint8_t q[32];
        for (int64_t b = 0; b < K / 32; ++b) {
            scalesT[j * (K / 32) + b] = mx_block(W + 32 * b * N + j, N, 32, q);
            for (int t = 0; t < 32; t += 2)
                codesT[j * (K / 2) + 16 * b + t / 2] = (uint8_t)(q[t] | (q[t + 1] << 4));
        }
    }
}

/* Y_ij = sum over blocks b of 2^(eA_ib + eW_jb) * sum_{k in b} e2m1(qA_ik) e2m1(qW_jk),
 * in double, for the listed rows (rows == NULL: all M).                     */
void orc_mx_gemm_rows(const uint8_t* codesA, const uint8_t* sA, const uint8_t* codesWT,
                      const uint8_t* sW, int64_t M, int64_t N, int64_t K, const int64_t* rows,
                      int64_t nrows, double* Y) {
    const int64_t R = rows ? nrows : M;
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const int64_t i = rows ? rows[r] : r;
        for (int64_t j = 0; j < N; ++j) {
            double y = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                double part = 0.0;
                for (int64_t k = 32 * b; k < 32 * b + 32; ++k) {
                    const uint8_t ba = codesA[i * (K / 2) + k / 2];
                    const uint8_t bw = codesWT[j * (K / 2) + k / 2];
                    const uint8_t ca = (k & 1) ? (uint8_t)(ba >> 4) : (uint8_t)(ba & 15u);
                    const uint8_t cw = (k & 1) ? (uint8_t)(bw >> 4) : (uint8_t)(bw & 15u);
                    part += orc_e2m1_value(ca) * orc_e2m1_value(cw);
                }
                y += ldexp(part, ((int)sA[i * nb + b] - 127) + ((int)sW[j * nb + b] - 127));
            }
            Y[r * N + j] = y;
        }
    }
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

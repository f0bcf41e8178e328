/*
 * fp8_oracle.c -- plain, slow CPU oracle for the FP8 (e4m3) dynamic
 * quantization + scaled-GEMM hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline / reference legs may load this library.  The
 * product path (the CUDA library) never calls it, and the two share no code,
 * header, table or helper.
 *
 * What it computes, and the passages it follows:
 *
 *  - FP8 e4m3 is the OCP 8-bit "E4M3" format (1 sign, 4 exponent bits with bias
 *    7, 3 mantissa bits, no infinities, NaN = S.1111.111, largest finite
 *    value 448).  The pages only say "FP8"/"e4m3"; the maximum 448 used by the
 *    scale rule fixes this variant.  Encode/decode below are written from that
 *    format definition, value by value, in fp64.
 *
 *  - Dynamic quantization of one group G (a 1x128 slice, a 128x128 tile, a row
 *    or the whole tensor):  amax = max |x|,  s = 448 / amax (fp32, IEEE
 *    round-to-nearest),  q = e4m3(x * s) rounded to nearest-even and saturated
 *    to +-448,  and the stored scale is the reciprocal 1/s.  Storing the
 *    reciprocal follows pytorch/ao PR #2785 "integrate torch._scaled_mm into
 *    Float8BlockwiseLinear and add bench script" (Summary: the quant kernels
 *    write reciprocal scales directly); column-major scale grids follow the
 *    same Summary ("Compute scales in column major format").  The 1x128 /
 *    128x128 group shapes are the (1,128) and (128,128) block shapes of
 *    pytorch/ao PR #2592 "add more generic kernel for fp8 blockwise scaling"
 *    (Performance table) and the (BlockWise1x128, BlockWise128x128) recipe of
 *    pytorch/ao PR #4209 "[codex] add repro for blockwise _scaled_mm
 *    investigation" (Findings So Far).
 *    Readings where the pages are silent: an all-zero group uses
 *    amax = 1e-12; q is computed from x*s (not x/r); r = 1/s (not amax/448);
 *    the sign of a zero result is kept (0x80).
 *
 *  - Scaled GEMM, C = A . B^T with A (M x K) and B^T (N x K) both K-contiguous:
 *    C[m,n] = sum_kb  rA(m,kb) * rB(n,kb) * sum_{k in kb} D(qA[m,k]) D(qB[n,k]).
 *    This is the explicit "dequantized matmul" of PR #4209 (What Changed: the
 *    repro compares an FP32 reference matmul, an explicit dequantized matmul
 *    and the kernels on the same quantized inputs and reciprocal scales) and
 *    of ROCm/aiter issue #1765 "[Issue]: Does gemm_a8w8 support per-tensor
 *    quant?" (Steps to Reproduce: x_dequant = q*scale, F.linear of the two).
 *    Two evaluations are provided: oracle_gemm dequantizes each element
 *    (D(q) * r in fp64) and accumulates in fp64 in natural k order;
 *    oracle_gemm_blocksum sums each 128-block of integer-valued products
 *    exactly and then multiplies by rA*rB.  Both are the same definition.
 *
 *  - SQNR = 20 log10(||ref|| / ||ref - out||), the quality measure PR #4209
 *    reports (Findings So Far) and PR #2592's review asks for everywhere.
 *
 * Build:  gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math: the
 * fp32 steps of the scale rule must be IEEE single-precision operations).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------- */
/* e4m3 (OCP "E4M3") decode and encode                                        */
/* ------------------------------------------------------------------------- */

/* Value of an e4m3 byte: (-1)^s * 2^(e-7) * (1 + m/8) for e in 1..15 (except
 * the NaN pattern e=15,m=7), and (-1)^s * 2^-6 * (m/8) for e = 0. */
EXPORT double oracle_e4m3_decode(uint8_t b)
{
    int s = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round a non-negative double to the nearest integer, ties to even. */
static double round_half_even(double q)
{
    double f = floor(q);
    double frac = q - f;            /* exact: q has at most 53 significant bits */
    if (frac > 0.5) return f + 1.0;
    if (frac < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Encode a float as e4m3 with round-to-nearest-even and saturation to +-448.
 * The magnitude grid: spacing 2^-9 below 2^-6 (subnormals), spacing
 * 2^(e-3) in the binade [2^e, 2^(e+1)) for e = -6..8.  NaN input maps to the
 * NaN pattern (never exercised: the path takes finite inputs only). */
EXPORT uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    double step, n, r;
    int e;
    if (isnan(v))
        return (uint8_t)(sign | 0x7F);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        step = ldexp(1.0, -9);
    } else {
        frexp(a, &e);               /* a = f * 2^e with f in [0.5, 1) */
        e -= 1;                     /* a in [2^e, 2^(e+1)) */
        step = ldexp(1.0, e - 3);
    }
    n = round_half_even(a / step);  /* a/step exact: step is a power of two */
    r = n * step;                   /* the rounded magnitude, on the grid */
    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -6)) {       /* subnormal: e-field 0, m = r / 2^-9 */
        return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9)));
    }
    frexp(r, &e);
    e -= 1;                         /* r in [2^e, 2^(e+1)), e in -6..8 */
    {
        int mant = (int)((r / ldexp(1.0, e) - 1.0) * 8.0);   /* 0..7, exact */
        return (uint8_t)(sign | ((e + 7) << 3) | mant);
    }
}

EXPORT void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode(v[i]);
}

EXPORT void oracle_e4m3_decode_array(const uint8_t* b, int64_t n, double* out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        out[i] = oracle_e4m3_decode(b[i]);
}

/* ------------------------------------------------------------------------- */
/* Input access: bf16 (raw 16-bit patterns) or fp32, through a strided view.  */
/* ------------------------------------------------------------------------- */

enum { ORACLE_BF16 = 0, ORACLE_F32 = 1 };

/* Element (i, j) of a strided view: x[i*s0 + j*s1], widened exactly to fp32. */
static float load_elem(const void* x, int xt, int64_t i, int64_t j, int64_t s0, int64_t s1)
{
    int64_t off = i * s0 + j * s1;
    if (xt == ORACLE_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t*)x)[off]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return f;
    }
    return ((const float*)x)[off];
}

/* Which scale rule the quantization functions apply (oracle_set_scale_rule):
 * 0, the method's rule: s = 448 / amax in fp32;
 * 1, the power-of-two rule of hardware block scaling (UE8M0 scale factors, an
 *    8-bit exponent and no mantissa): s = the largest power of two not above
 *    fl32(448 / amax), so that x * s is exact and never above 448.  This is
 *    the B200 form of a variant without per-K-block promotion in software (the
 *    tensor core applies power-of-two block scales itself), the counterpart of
 *    the fast-accumulation flag of the scaled-mm template in pytorch/pytorch
 *    issue #159940 (Describe the bug: USE_FAST_ACCUM). */
static int g_scale_rule = 0;

EXPORT void oracle_set_scale_rule(int rule)
{
    g_scale_rule = rule;
}

/* The scale rule for one group with absolute maximum amax. */
static float scale_from_amax(float amax)
{
    float s = 448.0f / fmaxf(amax, 1e-12f);
    if (g_scale_rule == 1) {
        int e;
        (void)frexpf(s, &e);           /* s = m * 2^e, m in [0.5, 1) */
        s = ldexpf(1.0f, e - 1);
    }
    return s;
}

/* ------------------------------------------------------------------------- */
/* Quantization.  The input is the strided view V (rows x cols), element       */
/* (i, j) at x[i*s0 + j*s1].  A row-major matrix is s0 = ld, s1 = 1; its       */
/* transpose is s0 = 1, s1 = ld.                                               */
/* ------------------------------------------------------------------------- */

/* 1x128 groups along the columns of V: group g of row i covers columns
 * [128g, min(128g+128, cols)).  Output row o (o = index into `rows`, or the
 * row itself when rows == NULL) goes to q[o*ldq + j]; its scale for group g
 * goes to sinv[o + g*ld_s] (column-major grid). */
EXPORT void oracle_quant_1x128(const void* x, int xt, int64_t nrow_view, int64_t cols,
                               int64_t s0, int64_t s1,
                               const int64_t* rows, int64_t nrows,
                               uint8_t* q, int64_t ldq, float* sinv, int64_t ld_s)
{
    int64_t G = (cols + 127) / 128;
    int64_t n_out = rows ? nrows : nrow_view;
    int64_t o;
#pragma omp parallel for schedule(dynamic, 4)
    for (o = 0; o < n_out; ++o) {
        int64_t i = rows ? rows[o] : o;
        int64_t g, j;
        for (g = 0; g < G; ++g) {
            int64_t j0 = 128 * g, j1 = j0 + 128 < cols ? j0 + 128 : cols;
            float amax = 0.0f, s;
            for (j = j0; j < j1; ++j) {
                float a = fabsf(load_elem(x, xt, i, j, s0, s1));
                if (a > amax) amax = a;
            }
            s = scale_from_amax(amax);
            for (j = j0; j < j1; ++j)
                q[o * ldq + j] = oracle_e4m3_encode(load_elem(x, xt, i, j, s0, s1) * s);
            sinv[o + g * ld_s] = 1.0f / s;
        }
    }
}

/* 128x128 tiles of V.  Tile (bi, bj) covers rows [128bi, ...) and columns
 * [128bj, ...), clipped at the edges.  Only the row-blocks listed in `rblocks`
 * (or all when NULL) are computed; row-block number o of the list is written
 * to output rows [128o, 128o+128) of q, and its scales to sinv[o + bj*ld_s]. */
EXPORT void oracle_quant_128x128(const void* x, int xt, int64_t nrow_view, int64_t cols,
                                 int64_t s0, int64_t s1,
                                 const int64_t* rblocks, int64_t nrb,
                                 uint8_t* q, int64_t ldq, float* sinv, int64_t ld_s)
{
    int64_t RB = (nrow_view + 127) / 128, CB = (cols + 127) / 128;
    int64_t n_out = rblocks ? nrb : RB;
    int64_t t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < n_out * CB; ++t) {
        int64_t o = t / CB, bj = t % CB;
        int64_t bi = rblocks ? rblocks[o] : o;
        int64_t i0 = 128 * bi, i1 = i0 + 128 < nrow_view ? i0 + 128 : nrow_view;
        int64_t j0 = 128 * bj, j1 = j0 + 128 < cols ? j0 + 128 : cols;
        int64_t i, j;
        float amax = 0.0f, s;
        for (i = i0; i < i1; ++i)
            for (j = j0; j < j1; ++j) {
                float a = fabsf(load_elem(x, xt, i, j, s0, s1));
                if (a > amax) amax = a;
            }
        s = scale_from_amax(amax);
        for (i = i0; i < i1; ++i)
            for (j = j0; j < j1; ++j)
                q[(128 * o + (i - i0)) * ldq + j] =
                    oracle_e4m3_encode(load_elem(x, xt, i, j, s0, s1) * s);
        sinv[o + bj * ld_s] = 1.0f / s;
    }
}

/* One scale per row of V (the group is the whole row). */
EXPORT void oracle_quant_rowwise(const void* x, int xt, int64_t nrow_view, int64_t cols,
                                 int64_t s0, int64_t s1,
                                 const int64_t* rows, int64_t nrows,
                                 uint8_t* q, int64_t ldq, float* sinv)
{
    int64_t n_out = rows ? nrows : nrow_view;
    int64_t o;
#pragma omp parallel for schedule(dynamic, 4)
    for (o = 0; o < n_out; ++o) {
        int64_t i = rows ? rows[o] : o;
        int64_t j;
        float amax = 0.0f, s;
        for (j = 0; j < cols; ++j) {
            float a = fabsf(load_elem(x, xt, i, j, s0, s1));
            if (a > amax) amax = a;
        }
        s = scale_from_amax(amax);
        for (j = 0; j < cols; ++j)
            q[o * ldq + j] = oracle_e4m3_encode(load_elem(x, xt, i, j, s0, s1) * s);
        sinv[o] = 1.0f / s;
    }
}

/* One scale for the whole tensor (n contiguous elements). */
EXPORT void oracle_quant_tensor(const void* x, int xt, int64_t n, uint8_t* q, float* sinv)
{
    float amax = 0.0f, s;
    int64_t i;
    for (i = 0; i < n; ++i) {
        float a = fabsf(load_elem(x, xt, i, 0, 1, 0));
        if (a > amax) amax = a;
    }
    s = scale_from_amax(amax);
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        q[i] = oracle_e4m3_encode(load_elem(x, xt, i, 0, 1, 0) * s);
    *sinv = 1.0f / s;
}

/* ------------------------------------------------------------------------- */
/* Scaled GEMM                                                                */
/* ------------------------------------------------------------------------- */

enum {
    ORACLE_SCALE_TENSOR = 0,            /* rA = sa[0],           rB = sb[0]            */
    ORACLE_SCALE_ROWWISE = 1,           /* rA = sa[m],           rB = sb[n]            */
    ORACLE_SCALE_BLOCK_1x128_128x128 = 2, /* rA = sa[m + kb ld_sa], rB = sb[n/128 + kb ld_sb] */
    ORACLE_SCALE_BLOCK_1x128_1x128 = 3    /* rA = sa[m + kb ld_sa], rB = sb[n + kb ld_sb]     */
};

static double scale_a(int mode, const float* sa, int64_t ld_sa, int64_t m, int64_t kb)
{
    switch (mode) {
    case ORACLE_SCALE_TENSOR:  return (double)sa[0];
    case ORACLE_SCALE_ROWWISE: return (double)sa[m];
    default:                   return (double)sa[m + kb * ld_sa];
    }
}

static double scale_b(int mode, const float* sb, int64_t ld_sb, int64_t n, int64_t kb)
{
    switch (mode) {
    case ORACLE_SCALE_TENSOR:              return (double)sb[0];
    case ORACLE_SCALE_ROWWISE:             return (double)sb[n];
    case ORACLE_SCALE_BLOCK_1x128_128x128: return (double)sb[n / 128 + kb * ld_sb];
    default:                               return (double)sb[n + kb * ld_sb];
    }
}

/* C[o][n] (o-th listed row, or row o when rows == NULL), C row-major M' x N.
 * Each operand element is dequantized, a = D(q) * r in fp64, and the products
 * are accumulated in fp64 in natural k order. */
EXPORT void oracle_gemm(int64_t M, int64_t N, int64_t K,
                        const uint8_t* A, int64_t lda, const uint8_t* Bt, int64_t ldb,
                        const float* sa, int64_t ld_sa, const float* sb, int64_t ld_sb,
                        int mode, const int64_t* rows, int64_t nrows, double* C)
{
    int64_t n_out = rows ? nrows : M;
    int64_t t;
    (void)M;
#pragma omp parallel for schedule(dynamic, 16)
    for (t = 0; t < n_out * N; ++t) {
        int64_t o = t / N, n = t % N;
        int64_t m = rows ? rows[o] : o;
        int64_t k;
        double acc = 0.0;
        for (k = 0; k < K; ++k) {
            int64_t kb = k / 128;
            double a = oracle_e4m3_decode(A[m * lda + k]) * scale_a(mode, sa, ld_sa, m, kb);
            double b = oracle_e4m3_decode(Bt[n * ldb + k]) * scale_b(mode, sb, ld_sb, n, kb);
            acc += a * b;
        }
        C[o * N + n] = acc;
    }
}

/* Same definition, evaluated block by block: for each 128-wide K block the
 * products D(qA) D(qB) are integer multiples of 2^-18 below 2^18 in size, so
 * a block sum of at most 128 of them is exact in fp64; the block sum is then
 * multiplied by rA * rB and added. */
EXPORT void oracle_gemm_blocksum(int64_t M, int64_t N, int64_t K,
                                 const uint8_t* A, int64_t lda, const uint8_t* Bt, int64_t ldb,
                                 const float* sa, int64_t ld_sa, const float* sb, int64_t ld_sb,
                                 int mode, const int64_t* rows, int64_t nrows, double* C)
{
    int64_t n_out = rows ? nrows : M;
    int64_t Kb = (K + 127) / 128;
    int64_t t;
    (void)M;
#pragma omp parallel for schedule(dynamic, 16)
    for (t = 0; t < n_out * N; ++t) {
        int64_t o = t / N, n = t % N;
        int64_t m = rows ? rows[o] : o;
        int64_t kb, k;
        double acc = 0.0;
        for (kb = 0; kb < Kb; ++kb) {
            int64_t k1 = 128 * kb + 128 < K ? 128 * kb + 128 : K;
            double blk = 0.0;
            for (k = 128 * kb; k < k1; ++k)
                blk += oracle_e4m3_decode(A[m * lda + k]) * oracle_e4m3_decode(Bt[n * ldb + k]);
            acc += blk * (scale_a(mode, sa, ld_sa, m, kb) * scale_b(mode, sb, ld_sb, n, kb));
        }
        C[o * N + n] = acc;
    }
}

/* Unquantized reference: C[o][n] = sum_k X[m][k] * Y[n][k] in fp64, X and Y
 * given as bf16 or fp32 strided views (element (i,k) at X[i*xs0 + k*xs1]). */
EXPORT void oracle_matmul_ref(int64_t N, int64_t K,
                              const void* X, int xt, int64_t xs0, int64_t xs1,
                              const void* Y, int yt, int64_t ys0, int64_t ys1,
                              const int64_t* rows, int64_t nrows, double* C)
{
    int64_t t;
#pragma omp parallel for schedule(dynamic, 16)
    for (t = 0; t < nrows * N; ++t) {
        int64_t o = t / N, n = t % N;
        int64_t m = rows[o];
        int64_t k;
        double acc = 0.0;
        for (k = 0; k < K; ++k)
            acc += (double)load_elem(X, xt, m, k, xs0, xs1) * (double)load_elem(Y, yt, n, k, ys0, ys1);
        C[o * N + n] = acc;
    }
}

/* SQNR in dB of `out` against `ref`: 20 log10(||ref||_2 / ||ref - out||_2). */
EXPORT double oracle_sqnr(const double* ref, const double* out, int64_t n)
{
    double s = 0.0, e = 0.0;
    int64_t i;
    for (i = 0; i < n; ++i) {
        double d = ref[i] - out[i];
        s += ref[i] * ref[i];
        e += d * d;
    }
    return 20.0 * log10(sqrt(s) / sqrt(e));
}

/* Round fp64 values to fp32 (RN) and then to bf16 (RNE), returning the bf16
 * bit patterns: the oracle's output conversion for bf16 results. */
EXPORT void oracle_to_bf16(const double* c, int64_t n, uint16_t* out)
{
    int64_t i;
    for (i = 0; i < n; ++i) {
        float f = (float)c[i];
        uint32_t u, lsb;
        memcpy(&u, &f, sizeof u);
        lsb = (u >> 16) & 1u;
        u += 0x7FFFu + lsb;         /* finite inputs only */
        out[i] = (uint16_t)(u >> 16);
    }
}

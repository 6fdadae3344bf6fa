/*
 * CPU oracle for the weight-streaming matmul and the router top-k.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg call into this file.  It shares no code,
 * header, table or helper with the CUDA library; the two sides meet only in
 * the seeded 16-bit input patterns drawn by the separate input generator.
 *
 * What it computes (plain definitions, written out, fp64 throughout):
 *
 *   C[i][j] = sum_{p=0}^{k-1} dec(A[i][p]) * dec(Wt[j][p])      (p ascending)
 *   S[i][j] = sum_{p=0}^{k-1} |dec(A[i][p]) * dec(Wt[j][p])|
 *
 * This is the product C[m,n] = A[m,k] . W[k,n] whose per-row cost the
 * nx_batchscale_kat.nx note times across m, with the weight stored with k
 * contiguous (row j of Wt is column j of W).  The method reaches exactly this
 * product up to rounding order, so the oracle is the definition itself.
 * S is the per-element scale of the error bound |err| <= 1e-5 * S.
 *
 * Top-k (the multi-row top-10 of Strata PR #109, "What", router bullet): for
 * each row, every (value, index) pair is sorted by a total order -- value
 * descending, equal values by index ascending, -0.0 equal to +0.0, any NaN
 * ranked above +inf -- and the first topk pairs are returned.
 *
 * dec() decodes bf16 / f16 bit patterns exactly from their IEEE-754 style
 * fields (sign, biased exponent, fraction), subnormals, infinities and NaN
 * included.
 *
 * Threads: OpenMP splits the output elements only; each element's k loop
 * runs in one thread in ascending order, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F16 = 0, ORC_BF16 = 1 };

/* bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_dec_bf16(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xFF;
    int f = h & 0x7F;
    double v;
    if (e == 0xFF)
        v = f ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)f, -126 - 7);           /* subnormal: f * 2^-133 */
    else
        v = ldexp(1.0 + (double)f / 128.0, e - 127);
    return sign ? -v : v;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_dec_f16(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0x1F)
        v = f ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)f, -14 - 10);            /* subnormal: f * 2^-24 */
    else
        v = ldexp(1.0 + (double)f / 1024.0, e - 15);
    return sign ? -v : v;
}

static double dec(uint16_t h, int fmt)
{
    return fmt == ORC_BF16 ? oracle_dec_bf16(h) : oracle_dec_f16(h);
}

/*
 * C = A . W with W given as Wt[n][k] (k contiguous), plus S = sum |a*w|.
 * A: m rows of k 16-bit patterns, row stride lda elements.
 * C, S: m rows of n doubles, row stride ldc (S may be NULL).
 * Returns 0, or -1 on a bad argument.
 */
int oracle_matmul(const uint16_t *A, int64_t lda, int a_fmt,
                  const uint16_t *Wt, int64_t ldw, int w_fmt,
                  int64_t m, int64_t n, int64_t k,
                  double *C, double *S, int64_t ldc)
{
    if (m < 0 || n < 0 || k < 0 || (m && (!A || !C)) || (n && !Wt))
        return -1;
    if ((a_fmt != ORC_F16 && a_fmt != ORC_BF16) || (w_fmt != ORC_F16 && w_fmt != ORC_BF16))
        return -1;
    int64_t total = m * n;
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < total; ++e) {
        int64_t i = e / n, j = e % n;
        double acc = 0.0, mag = 0.0;
        for (int64_t p = 0; p < k; ++p) {
            double prod = dec(A[i * lda + p], a_fmt) * dec(Wt[j * ldw + p], w_fmt);
            acc += prod;
            mag += fabs(prod);
        }
        C[i * ldc + j] = acc;
        if (S)
            S[i * ldc + j] = mag;
    }
    return 0;
}

/* ---- top-k --------------------------------------------------------------- */

typedef struct {
    float v;
    int32_t i;
} orc_pair;

/* Negative when x ranks before y in the total order. */
static int orc_rank(const void *px, const void *py)
{
    const orc_pair *x = (const orc_pair *)px, *y = (const orc_pair *)py;
    int xn = isnan(x->v), yn = isnan(y->v);
    if (xn != yn)
        return xn ? -1 : 1;                 /* NaN ranks above everything */
    if (!xn) {
        if (x->v > y->v) return -1;         /* larger value first; -0 == +0 */
        if (x->v < y->v) return 1;
    }
    return (x->i < y->i) ? -1 : (x->i > y->i);   /* ties: lower index first */
}

/*
 * For each of m rows of n fp32 logits (row stride ldl), write the topk best
 * (index, value) pairs in rank order to idx / val (row stride ldo; val may be
 * NULL).  Returns 0, or -1 on a bad argument.
 */
int oracle_topk(const float *logits, int64_t ldl, int64_t m, int64_t n, int32_t topk,
                int32_t *idx, float *val, int64_t ldo)
{
    if (m < 0 || n < 1 || topk < 0 || topk > n || (m && (!logits || !idx)))
        return -1;
    orc_pair *buf = (orc_pair *)malloc((size_t)n * sizeof(orc_pair));
    if (!buf)
        return -1;
    for (int64_t r = 0; r < m; ++r) {
        for (int64_t j = 0; j < n; ++j) {
            buf[j].v = logits[r * ldl + j];
            buf[j].i = (int32_t)j;
        }
        qsort(buf, (size_t)n, sizeof(orc_pair), orc_rank);
        for (int32_t t = 0; t < topk; ++t) {
            idx[r * ldo + t] = buf[t].i;
            if (val)
                val[r * ldo + t] = buf[t].v;
        }
    }
    free(buf);
    return 0;
}

/* ---- output-rounding allowance -------------------------------------------- */

/*
 * Spacing of the binary16 / bfloat16 grid at |x|: for a finite |x| in a normal
 * binade [2^e, 2^(e+1)) it is 2^(e - fraction_bits); below the smallest normal
 * it is the subnormal spacing.  A round-to-nearest result is within half of
 * this of the value it rounds.
 */
double oracle_ulp_f16(double x)
{
    double a = fabs(x);
    if (a < ldexp(1.0, -14))
        return ldexp(1.0, -24);
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
    return ldexp(1.0, (e - 1) - 10);
}

double oracle_ulp_bf16(double x)
{
    double a = fabs(x);
    if (a < ldexp(1.0, -126))
        return ldexp(1.0, -133);
    int e;
    frexp(a, &e);
    return ldexp(1.0, (e - 1) - 7);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- bf16 cast and sigmoid gate (adjacent window steps) ------------------ */

/*
 * fp32 -> bf16 with round to nearest, ties to even, from the binary32 bit
 * layout: keep the top 16 bits and round on the 16 dropped ones.  NaN maps to
 * a quiet NaN of the same sign; overflow rounds to infinity like any other
 * carry into the exponent field.  (The bf16 cast of the window's rows in
 * Strata PR #109, "What": one call casts the window's contiguous rows.)
 */
uint16_t oracle_f32_to_bf16(float x)
{
    uint32_t b;
    memcpy(&b, &x, sizeof(b));
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu))
        return (uint16_t)((b >> 16) | 0x0040u);          /* quiet NaN */
    uint32_t upper = b >> 16, lower = b & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;                                      /* carries may reach the exponent */
    return (uint16_t)upper;
}

void oracle_cast_f32_bf16(const float *x, int64_t ldx, uint16_t *y, int64_t ldy, int64_t rows, int64_t cols)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            y[r * ldy + c] = oracle_f32_to_bf16(x[r * ldx + c]);
}

/* The logistic function 1 / (1 + e^-x) in fp64 (the shared expert's scalar gate). */
double oracle_sigmoid(double x)
{
    return 1.0 / (1.0 + exp(-x));
}

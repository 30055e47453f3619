/*
 * nvfp4_oracle.c -- plain, slow, float64 CPU oracle for the NVFP4 decode GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file.  It is used by tests/, by __graft_entry__.smoke()
 * and by bench.py's cpu_baseline / reference legs, and by nothing else.  It
 * shares no code, table or constant generator with the CUDA library.
 *
 * What it computes (ignis, "Models and artifacts", section "The artifact":
 * the body is 4-bit floating point with one scale per 16 values, read by the
 * kernels straight from its weight planes; ignis README, "The decode round":
 * all lanes share one pass over the weights):
 *
 *   Y[m][n] = gscale * sum_k x[m][k] * e2m1(q[n][k]) * e4m3(s[n][k/16])
 *
 * Element and scale codes follow the standard NVFP4 / OCP formats, which the
 * pages do not spell out (readings listed in the design notes):
 *   E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.
 *   E4M3 ("fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
 *         0x7F/0xFF are NaN, no infinities.
 * Canonical planes: q is u8[N][K/2], element 2j of a row in the low nibble
 * of byte j and element 2j+1 in the high nibble; s is u8[N][K/16], scale b
 * covering k in [16b, 16b+15].  X is bf16 [M][K] row-major (raw bits).
 *
 * Every code is decoded through an explicit table built from the format's
 * definition; all arithmetic is double; sums run in plain k order.
 * Parity status: every function here is pinned by tests (tables against
 * closed forms and torch's float8_e4m3fn; GEMM against closed forms and a
 * brute-force loop on tiny shapes; top-k against hand-derived cases, numpy's
 * lexsort / stable argsort and its defining invariants).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* E2M1 value of a 4-bit code, from the format definition. */
static double e2m1_def(unsigned c)
{
    unsigned s = (c >> 3) & 1u, e = (c >> 1) & 3u, m = c & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* E4M3 (OCP "fn") value of a byte, from the format definition. */
static double e4m3_def(unsigned b)
{
    unsigned s = (b >> 7) & 1u, e = (b >> 3) & 15u, m = b & 7u;
    double mag;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

static double E2M1[16];
static double E4M3[256];
static int tables_ready = 0;

static void build_tables(void)
{
    if (tables_ready) return;
    for (unsigned c = 0; c < 16; ++c) E2M1[c] = e2m1_def(c);
    for (unsigned b = 0; b < 256; ++b) E4M3[b] = e4m3_def(b);
    tables_ready = 1;
}

/* bf16 is the top half of an IEEE binary32. */
static double bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static unsigned code_at(const uint8_t* q, int64_t K, int64_t n, int64_t k)
{
    uint8_t byte = q[n * (K / 2) + k / 2];
    return (k & 1) ? (byte >> 4) : (byte & 15u);
}

static unsigned scale_at(const uint8_t* s, int64_t K, int64_t n, int64_t k)
{
    return s[n * (K / 16) + k / 16];
}

int or_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void or_tables(double* e2m1_out, double* e4m3_out)
{
    build_tables();
    memcpy(e2m1_out, E2M1, sizeof E2M1);
    memcpy(e4m3_out, E4M3, sizeof E4M3);
}

/* Number of NaN scale codes (0x7F / 0xFF) in a canonical scale plane. */
int64_t or_count_nan_scales(const uint8_t* s, int64_t N, int64_t K)
{
    int64_t bad = 0;
    for (int64_t i = 0; i < N * (K / 16); ++i)
        if ((s[i] & 0x7Fu) == 0x7Fu) ++bad;
    return bad;
}

/* Dequantised weights: W[n][k] = fp32( e2m1 * e4m3 * gscale ).  The product
 * of the two codes is exact in double; the single rounding is the final
 * conversion to float (round to nearest even). */
void or_dequant(const uint8_t* q, const uint8_t* s, int64_t N, int64_t K, float gscale, float* W)
{
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double w = E2M1[code_at(q, K, n, k)] * E4M3[scale_at(s, K, n, k)];
            W[n * K + k] = (float)(w * (double)gscale);
        }
}

/* The decode GEMM in float64.  Y[m][n] and, for the tolerance,
 * A[m][n] = sum_k |x[m][k] * w[n][k]| with w = fp32 dequantised weight. */
void or_gemm(const uint16_t* X, int M, const uint8_t* q, const uint8_t* s, float gscale,
             int64_t N, int64_t K, double* Y, double* A)
{
    build_tables();
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int m = 0; m < M; ++m) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double w = E2M1[code_at(q, K, n, k)] * E4M3[scale_at(s, K, n, k)];
                double x = bf16_to_double(X[(int64_t)m * K + k]);
                acc += x * w;
                mag += fabs(x * (double)(float)(w * (double)gscale));
            }
            Y[(int64_t)m * N + n] = (double)gscale * acc;
            if (A) A[(int64_t)m * N + n] = mag;
        }
}

/* The same GEMM for a subset of output elements (rows n_idx[i] for every
 * lane), so that very large shapes can be checked on samples. */
void or_gemm_rows(const uint16_t* X, int M, const uint8_t* q, const uint8_t* s, float gscale,
                  int64_t N, int64_t K, const int64_t* n_idx, int64_t count, double* Y, double* A)
{
    build_tables();
    (void)N;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t n = n_idx[i];
        for (int m = 0; m < M; ++m) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double w = E2M1[code_at(q, K, n, k)] * E4M3[scale_at(s, K, n, k)];
                double x = bf16_to_double(X[(int64_t)m * K + k]);
                acc += x * w;
                mag += fabs(x * (double)(float)(w * (double)gscale));
            }
            Y[(int64_t)m * count + i] = (double)gscale * acc;
            if (A) A[(int64_t)m * count + i] = mag;
        }
    }
}

/* Fused MLP front half: g = gate GEMM, u = up GEMM, h = silu(g) * u, with
 * silu(g) = g / (1 + exp(-g)).  Outputs g, u, h and the two magnitude sums. */
void or_gateup_silu(const uint16_t* X, int M,
                    const uint8_t* qg, const uint8_t* sg, float gscale_g,
                    const uint8_t* qu, const uint8_t* su, float gscale_u,
                    int64_t Nff, int64_t K,
                    double* G, double* U, double* H, double* AG, double* AU)
{
    or_gemm(X, M, qg, sg, gscale_g, Nff, K, G, AG);
    or_gemm(X, M, qu, su, gscale_u, Nff, K, U, AU);
    for (int64_t i = 0; i < (int64_t)M * Nff; ++i) {
        double g = G[i];
        H[i] = g / (1.0 + exp(-g)) * U[i];
    }
}

/* ------------------------------------------------------------------------
 * Top-k over rows of FP32 logits (ignis README, "What sets it apart",
 * "Speculative decoding (DFlash2)": the row-split top-k that follows the
 * output head and gives a bit-identical answer).
 *
 * For each row m < M: the k largest of logits[m][0..V) (row stride ldv),
 * written as vals[m][j], idx[m][j] for j = 0..k-1, best first.  "Largest"
 * is IEEE 754 totalOrder except that -0 and +0 count as equal; equal
 * values rank by lower index.  So for numbers (infinities included) it is
 * the numeric order; a NaN with sign 0 ranks above +inf and one with sign 1
 * below -inf; among NaNs of one sign a larger payload is further from the
 * numbers.  The answer is unique.  Plain method: sort every index of the
 * row with that comparison and keep the first k.
 * ---------------------------------------------------------------------- */
#include <stdlib.h>

typedef struct {
    float v;
    int64_t i;
} or_entry;

/* -1 if x ranks before y (x is "larger"), +1 if after, 0 if tied. */
static int or_value_rank(float x, float y)
{
    const int xn = isnan(x), yn = isnan(y);
    if (!xn && !yn) {
        if (x > y) return -1;
        if (x < y) return 1;
        return 0; /* equal numbers, -0 == +0 included */
    }
    uint32_t bx, by;
    memcpy(&bx, &x, 4);
    memcpy(&by, &y, 4);
    /* class: 2 = NaN with sign 0, 1 = a number, 0 = NaN with sign 1 */
    const int cx = xn ? ((bx >> 31) ? 0 : 2) : 1;
    const int cy = yn ? ((by >> 31) ? 0 : 2) : 1;
    if (cx != cy) return cx > cy ? -1 : 1;
    /* two NaNs of the same sign: compare payloads (the 23 fraction bits) */
    const uint32_t px = bx & 0x7FFFFFu, py = by & 0x7FFFFFu;
    if (px == py) return 0;
    if (cx == 2) return px > py ? -1 : 1; /* positive NaNs: larger payload ranks first */
    return px > py ? 1 : -1;              /* negative NaNs: larger payload ranks last */
}

static int or_entry_cmp(const void* a, const void* b)
{
    const or_entry* x = (const or_entry*)a;
    const or_entry* y = (const or_entry*)b;
    const int r = or_value_rank(x->v, y->v);
    if (r != 0) return r;
    return (x->i < y->i) ? -1 : (x->i > y->i ? 1 : 0);
}

/* Returns 0, or -1 on bad arguments (k < 1, k > V, ldv < V) or no memory. */
int or_topk(const float* logits, int M, int64_t V, int64_t ldv, int k, float* vals, int32_t* idx)
{
    if (M < 1 || V < 1 || k < 1 || k > V || ldv < V) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int m = 0; m < M; ++m) {
        or_entry* e = (or_entry*)malloc((size_t)V * sizeof(or_entry));
        if (!e) {
            bad |= 1;
            continue;
        }
        for (int64_t i = 0; i < V; ++i) {
            e[i].v = logits[(int64_t)m * ldv + i];
            e[i].i = i;
        }
        qsort(e, (size_t)V, sizeof(or_entry), or_entry_cmp);
        for (int j = 0; j < k; ++j) {
            vals[(int64_t)m * k + j] = e[j].v;
            idx[(int64_t)m * k + j] = (int32_t)e[j].i;
        }
        free(e);
    }
    return bad ? -1 : 0;
}

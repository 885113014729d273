/*
 * CPU oracle for the LittleBit compressed linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It is deliberately plain and slow: float64 arithmetic,
 * single-threaded loops in the order the method states, no blocking, no
 * fusion, no reordering.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Source (LittleBit: Ultra Low-Bit Quantization via Latent Factorization,
 * NeurIPS 2025, paper notes page, section "Multi-scale compensation"):
 *   W_pri = diag(h) * U_sign * diag(l) * V_sign^T * diag(g),
 * and, section "Residual compensation", W = W_pri + W_res with the residual
 * path of the same form.  The same section of notes states the forward is
 * evaluated as sequential element-wise products and binary matmuls without
 * storing the effective weight; orc_forward follows exactly that order:
 *   t = x (.) g ; z = t . V_sign ; z (.)= l ; s = z . U_sign^T ; y += h (.) s.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - sign(0) = +1; a value is "negative" iff (value < 0), so -0.0 -> +1 and
 *    NaN -> +1 (the comparison is false).
 *  - W is N x K (rows = outputs); U_sign is N x r, V_sign is K x r.
 *  - h, g, l are IEEE binary16; x is bfloat16; both paths have the same rank r
 *    and each path has its own h, g, l.
 *  - Canonical packed layout: word  packed[i * ceil(r/32) + j/32],  bit j%32,
 *    is 1 iff F[i][j] < 0.  Padding bits are 0.
 *
 * Parity pins (all in the CPU test suite): every function here is pinned by
 * something other than itself -- numpy's float16 decoder over all 65536
 * codes, numpy.packbits for the layout, dense reconstruction of W followed by
 * a library matmul, exact rational arithmetic, closed forms for special
 * cases, linearity and rank additivity.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- number formats, decoded from their IEEE / bfloat16 definitions ---- */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_half_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 1024), expo - 25);  /* (1 + frac/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32: 1 sign, 8 exponent (bias
 * 127), 7 fraction bits. */
double orc_bf16_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 7) & 0xff;
    int frac = bits & 0x7f;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -133);                /* subnormal: frac * 2^-133 */
    else if (expo == 255)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 128), expo - 134);  /* (1 + frac/128) * 2^(e-127) */
    return sign ? -v : v;
}

/* ---- sign binarisation and the canonical bit layout ---- */

int64_t orc_packed_words(int64_t rows, int r)
{
    return rows * (int64_t)((r + 31) / 32);
}

/* U_sign = sign(U) (notes page, method step 2).  One bit per element, set
 * iff the element compares below zero.  Written bit by bit. */
void orc_pack_signs(const float *F, int64_t rows, int r, uint32_t *packed)
{
    int64_t wpr = (r + 31) / 32;
    for (int64_t w = 0; w < rows * wpr; ++w)
        packed[w] = 0u;
    for (int64_t i = 0; i < rows; ++i)
        for (int j = 0; j < r; ++j)
            if (F[i * r + j] < 0.0f)
                packed[i * wpr + j / 32] |= (uint32_t)1u << (j % 32);
}

/* The +-1 value the canonical layout stores at (i, j). */
static int sign_at(const uint32_t *packed, int r, int64_t i, int j)
{
    int64_t wpr = (r + 31) / 32;
    uint32_t bit = (packed[i * wpr + j / 32] >> (j % 32)) & 1u;
    return bit ? -1 : +1;
}

void orc_unpack_signs(const uint32_t *packed, int64_t rows, int r, int8_t *s)
{
    for (int64_t i = 0; i < rows; ++i)
        for (int j = 0; j < r; ++j)
            s[i * r + j] = (int8_t)sign_at(packed, r, i, j);
}

/* ---- bits per weight ---- */

/* Storage of npaths paths, each r*(N+K) one-bit signs plus N+K+r 16-bit
 * scales, divided by the N*K weights of the dense layer. */
double orc_bpw(int N, int K, int r, int npaths)
{
    double per_path = (double)r * (double)(N + K) * 1.0 + 16.0 * (double)(N + K + r);
    return npaths * per_path / ((double)N * (double)K);
}

/* ---- one path of the forward, in the order the notes give ---- */

/* Latent vector of one activation row for one path:
 *   zl[j] = l[j] * sum_k V_sign[k][j] * (x[k] * g[k]).                       */
static void latent_row(const uint16_t *xrow, int K, int r, const uint32_t *V,
                       const uint16_t *g, const uint16_t *l, double *zl)
{
    double *t = (double *)malloc(sizeof(double) * (size_t)K);
    for (int k = 0; k < K; ++k)                       /* t = x (.) g          */
        t[k] = orc_bf16_to_double(xrow[k]) * orc_half_to_double(g[k]);
    for (int j = 0; j < r; ++j) {                     /* z = t . V_sign       */
        double z = 0.0;
        for (int k = 0; k < K; ++k)
            z += t[k] * (double)sign_at(V, r, k, j);
        zl[j] = z * orc_half_to_double(l[j]);         /* z (.)= l             */
    }
    free(t);
}

/* Output element of one path:  h[n] * sum_j U_sign[n][j] * zl[j].            */
static double output_elem(const double *zl, int r, const uint32_t *U,
                          const uint16_t *h, int64_t n)
{
    double s = 0.0;
    for (int j = 0; j < r; ++j)                       /* s = zl . U_sign^T    */
        s += zl[j] * (double)sign_at(U, r, n, j);
    return orc_half_to_double(h[n]) * s;              /* h (.) s              */
}

/*
 * y[M x N] (float64, row-major) = sum over paths of the path output.
 * x is [M x K] bfloat16 bits, row-major.  U[p] / V[p] are canonical packed
 * signs of path p (N x r and K x r); h[p] (N), g[p] (K), l[p] (r) are binary16.
 */
void orc_forward(int M, int N, int K, int r, int npaths,
                 const uint16_t *x,
                 const uint32_t *const *U, const uint32_t *const *V,
                 const uint16_t *const *h, const uint16_t *const *g,
                 const uint16_t *const *l, double *y)
{
    double *zl = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
    for (int64_t e = 0; e < (int64_t)M * N; ++e)
        y[e] = 0.0;
    for (int m = 0; m < M; ++m)
        for (int p = 0; p < npaths; ++p) {            /* W = W_pri + W_res    */
            latent_row(x + (int64_t)m * K, K, r, V[p], g[p], l[p], zl);
            for (int64_t n = 0; n < N; ++n)
                y[(int64_t)m * N + n] += output_elem(zl, r, U[p], h[p], n);
        }
    free(zl);
}

/*
 * Same result as orc_forward, for the selected rows ms[0..nm) and output
 * columns ns[0..nn) only:  out[a * nn + b] = y[ms[a]][ns[b]].  Used to check
 * full-size layers one sampled element at a time.
 */
void orc_forward_sampled(int M, int N, int K, int r, int npaths,
                         const uint16_t *x,
                         const uint32_t *const *U, const uint32_t *const *V,
                         const uint16_t *const *h, const uint16_t *const *g,
                         const uint16_t *const *l,
                         const int *ms, int nm, const int64_t *ns, int nn,
                         double *out)
{
    (void)M;
    (void)N;
    double *zl = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
    for (int64_t e = 0; e < (int64_t)nm * nn; ++e)
        out[e] = 0.0;
    for (int a = 0; a < nm; ++a)
        for (int p = 0; p < npaths; ++p) {
            latent_row(x + (int64_t)ms[a] * K, K, r, V[p], g[p], l[p], zl);
            for (int b = 0; b < nn; ++b)
                out[(int64_t)a * nn + b] += output_elem(zl, r, U[p], h[p], ns[b]);
        }
    free(zl);
}

/*
 * Brute force: the dense effective weight
 *   W[n][k] = sum_p h[n] * sum_j U_sign[n][j] * l[j] * V_sign[k][j] * g[k]
 * written out as an N x K float64 matrix (row-major).
 */
void orc_dense_weight(int N, int K, int r, int npaths,
                      const uint32_t *const *U, const uint32_t *const *V,
                      const uint16_t *const *h, const uint16_t *const *g,
                      const uint16_t *const *l, double *W)
{
    for (int64_t e = 0; e < (int64_t)N * K; ++e)
        W[e] = 0.0;
    for (int p = 0; p < npaths; ++p)
        for (int64_t n = 0; n < N; ++n)
            for (int k = 0; k < K; ++k) {
                double acc = 0.0;
                for (int j = 0; j < r; ++j)
                    acc += (double)sign_at(U[p], r, n, j) * orc_half_to_double(l[p][j]) *
                           (double)sign_at(V[p], r, k, j);
                W[n * K + k] += orc_half_to_double(h[p][n]) * acc * orc_half_to_double(g[p][k]);
            }
}

// Dual-SVID + residual initialisation of a LittleBit layer from a dense weight
// (LittleBit paper notes page, "Dual-SVID initialisation" and "Residual
// compensation"), all in binary64 on the device.
//
// Per path, with A = W (K <= N) or A = W^T (K > N), so that A is mA x nA with
// nA = min(N, K):
//   1. truncated SVD by randomised subspace iteration: Q (nA x L) random,
//      then `iters` times Z = orth(A Q), Q = orth(A^T Z), each orth a
//      Cholesky QR (Gram matrix, blocked Cholesky, triangular solve through
//      the inverses of its 64 x 64 diagonal blocks; columns whose orthogonal
//      part vanishes are dropped).  L = nA makes Q the identity and the SVD
//      exact.  Rayleigh-Ritz: P = A Q, T = P^T P = Z_T diag(lambda) Z_T^T by
//      Jacobi, the r largest lambda give s = sqrt(lambda), right vectors Q Z_r
//      and left vectors P Z_r / s;
//   2. U' = U_r sqrt(s), V' = V_r sqrt(s), each pair signed so that the
//      largest-magnitude entry of the U' column is positive; the sign bits
//      (set <=> < 0) are packed in the canonical layout;
//   3. rank-1 SVD of |U'| and |V'|: the top eigenpair of the r x r Gram matrix
//      (Jacobi) gives s_A^2 and b (signed to sum >= 0), a = |U'| b / s_A;
//      h = a_u, g = a_v, l = s_u s_v (b_u (.) b_v);
//   4. the residual path repeats 1-3 on W - diag(h) U_sign diag(l) V_sign^T diag(g).
#include "littlebit_init.h"
#include "lb_linalg.cuh"

#include <algorithm>
#include <math.h>

namespace lb {
namespace {

constexpr int kPanel = 64;
constexpr int kMaxSweeps = 40;
constexpr double kDepTol = 1e-13;      // pivot / column norm^2 below which a column counts as dependent
constexpr int kT = 256;
constexpr int kCholSmem = 2 * kPanel * (kPanel + 1) * (int)sizeof(double);

long even(long x) { return (x + 1) & ~1L; }
size_t up32(size_t x) { return (x + 31) & ~size_t(31); }

struct InitPlan {
    int N, K, r, nA, mA, L, npan;
    bool trans;               // A = W^T
    long ldK, ldL, ldr;
    size_t o_Wd, o_Q, o_Z, o_S, o_dg, o_inv, o_T, o_Vt, o_G, o_E, o_F, o_Up, o_Vp, o_M, o_Mv, o_vec, o_side, o_part;
    size_t o_int;             // int region (in doubles from the base)
    size_t total;             // doubles
};

InitPlan make_plan(int N, int K, int r)
{
    InitPlan P{};
    P.N = N;
    P.K = K;
    P.r = r;
    P.trans = K > N;
    P.nA = std::min(N, K);
    P.mA = std::max(N, K);
    const int want = std::max(64, (2 * r + 63) / 64 * 64);
    P.L = std::min(P.nA, want);
    P.npan = (P.L + kPanel - 1) / kPanel;
    P.ldK = even(K);
    P.ldL = even(P.L);
    P.ldr = even(r);
    size_t o = 0;
    auto take = [&](size_t n) { const size_t at = o; o = up32(o + n); return at; };
    P.o_Wd = take((size_t)N * P.ldK);
    P.o_Q = take((size_t)P.nA * P.ldL);
    P.o_Z = take((size_t)P.mA * P.ldL);
    P.o_S = take((size_t)P.L * P.ldL);
    P.o_dg = take((size_t)P.L);
    P.o_inv = take((size_t)P.npan * kPanel * kPanel);
    P.o_T = take((size_t)P.L * P.ldL);
    P.o_Vt = take((size_t)P.L * P.ldL);
    P.o_G = take((size_t)r * P.ldL);
    P.o_E = take((size_t)P.nA * P.ldr);
    P.o_F = take((size_t)P.mA * P.ldr);
    P.o_Up = take((size_t)N * P.ldr);
    P.o_Vp = take((size_t)K * P.ldr);
    P.o_M = take((size_t)r * P.ldr);
    P.o_Mv = take((size_t)r * P.ldr);
    P.o_vec = take((size_t)5 * r + 2 * (size_t)N + 2 * (size_t)K + 8);   // s, bu, bv, ls, misc | au, hs | av, gs
    P.o_side = take((size_t)3 * (P.L + 1));
    P.o_part = take(kDgemmPartElems);
    P.o_int = take((size_t)(2 * r + 16) / 2 + 1);                          // ints: bar[2], err, ord[r], flip[r]
    P.total = o;
    return P;
}

int grid_for(long n) { return (int)std::max<long>(1, std::min<long>((n + kT - 1) / kT, 148L * 8)); }

// ---------------------------------------------------------------------------
// element-wise and small kernels
// ---------------------------------------------------------------------------
__global__ void f32_to_f64_kernel(const float *__restrict__ W, int N, int K, double *Wd, long ld)
{
    const long total = (long)N * K;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x)
        Wd[(e / K) * ld + e % K] = (double)W[e];
}

__device__ __forceinline__ uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// start block of the subspace iteration: uniform entries in [-1, 1) from a counter-based generator
__global__ void random_fill_kernel(double *X, int rows, int cols, long ld, uint64_t seed)
{
    const long total = (long)rows * cols;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const uint64_t z = mix64(seed + (uint64_t)(e + 1) * 0x9E3779B97F4A7C15ull);
        X[(e / cols) * ld + e % cols] = (double)(z >> 11) * 0x1.0p-52 - 1.0;
    }
}

__global__ void identity_kernel(double *X, int n, long ld)
{
    const long total = (long)n * n;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x)
        X[(e / n) * ld + e % n] = (e / n == e % n) ? 1.0 : 0.0;
}

__global__ void copy_diag_kernel(const double *S, int n, long ld, double *dg)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) dg[i] = S[(long)i * ld + i];
}

// Cholesky of the diagonal block S[k0:k0+nb, k0:k0+nb] (lower triangle) in shared memory: L is written back in
// place, its inverse to Inv (64 x 64, ld 64, zero outside nb x nb).  A pivot at or below kDepTol times the
// column's original squared norm marks a dependent column: it is dropped (L column = e_j, inverse row j = 0).
__global__ void __launch_bounds__(kT) chol_diag_kernel(double *S, long ld, int k0, int nb, const double *__restrict__ dg,
                                                       double *Inv)
{
    extern __shared__ __align__(16) unsigned char csm[];
    double(*D)[kPanel + 1] = reinterpret_cast<double(*)[kPanel + 1]>(csm);
    double(*X)[kPanel + 1] = D + kPanel;
    __shared__ int dep[kPanel];
    const int tid = threadIdx.x;
    for (int e = tid; e < kPanel * kPanel; e += kT) {
        const int i = e / kPanel, j = e % kPanel;
        D[i][j] = (i < nb && j <= i) ? S[(long)(k0 + i) * ld + k0 + j] : 0.0;
        X[i][j] = 0.0;
    }
    __syncthreads();
    for (int j = 0; j < nb; ++j) {
        if (tid == 0) {
            const double d = D[j][j];
            const bool bad = !(d > kDepTol * dg[k0 + j]) || !(d > 0.0);
            dep[j] = bad;
            D[j][j] = bad ? 1.0 : sqrt(d);
        }
        __syncthreads();
        for (int i = j + 1 + tid; i < nb; i += kT) D[i][j] = dep[j] ? 0.0 : D[i][j] / D[j][j];
        __syncthreads();
        const int w = nb - j - 1;
        for (int e = tid; e < w * w; e += kT) {
            const int i = j + 1 + e / w, m = j + 1 + e % w;
            if (m <= i) D[i][m] -= D[i][j] * D[m][j];
        }
        __syncthreads();
    }
    // inverse of the lower-triangular D, one column per thread (forward substitution)
    for (int c = tid; c < nb; c += kT) {
        X[c][c] = 1.0 / D[c][c];
        for (int i = c + 1; i < nb; ++i) {
            double acc = 0.0;
            for (int m = c; m < i; ++m) acc += D[i][m] * X[m][c];
            X[i][c] = -acc / D[i][i];
        }
    }
    __syncthreads();
    for (int e = tid; e < kPanel * kPanel; e += kT) {
        const int i = e / kPanel, j = e % kPanel;
        Inv[e] = (i < nb && j < nb && !dep[i]) ? X[i][j] : 0.0;
        if (i < nb && j <= i) S[(long)(k0 + i) * ld + k0 + j] = D[i][j];
    }
}

// the r largest diagonal entries of T (eigenvalues after Jacobi), in decreasing order (first index on ties)
__global__ void select_top_kernel(const double *T, int n, long ld, int r, int *ord, double *sig)
{
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < n; j += gridDim.x * blockDim.x) {
        const double lj = T[(long)j * ld + j];
        int rank = 0;
        for (int i = 0; i < n; ++i) {
            const double li = T[(long)i * ld + i];
            rank += (li > lj) || (li == lj && i < j);
        }
        if (rank < r) {
            ord[rank] = j;
            sig[rank] = sqrt(fmax(lj, 0.0));
        }
    }
}

__global__ void gather_rows_kernel(const double *Vt, long ldv, const int *__restrict__ ord, int r, int n, double *G,
                                   long ldg)
{
    const long total = (long)r * n;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const int j = (int)(e / n), c = (int)(e % n);
        G[(long)j * ldg + c] = Vt[(long)ord[j] * ldv + c];
    }
}

// out[:, j] = X[:, j] * sqrt(s_j) (up) or / sqrt(s_j) (!up); zero where s_j == 0
__global__ void col_scale_kernel(const double *X, int rows, int r, long ldx, const double *__restrict__ sig, int up,
                                 double *out, long ldo)
{
    const long total = (long)rows * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const long i = e / r;
        const int j = (int)(e % r);
        const double s = sig[j];
        const double f = s > 0.0 ? (up ? sqrt(s) : 1.0 / sqrt(s)) : 0.0;
        out[i * ldo + j] = X[i * ldx + j] * f;
    }
}

// flip[j] = 1 if the largest-magnitude entry of column j (first index on ties) is negative; one warp per column
__global__ void col_sign_kernel(const double *X, int rows, int r, long ld, int *flip)
{
    const int lane = threadIdx.x & 31;
    for (int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; j < r; j += (gridDim.x * blockDim.x) >> 5) {
        double best = -1.0;
        int bi = 0x7fffffff;
        for (int i = lane; i < rows; i += 32) {
            const double v = fabs(X[(long)i * ld + j]);
            if (v > best) {       // rows are visited in increasing order: keeps the first index of a tie
                best = v;
                bi = i;
            }
        }
        for (int o = 16; o; o >>= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ob > best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
            }
        }
        if (lane == 0) flip[j] = (bi < rows && X[(long)bi * ld + j] < 0.0) ? 1 : 0;
    }
}

__global__ void col_flip_kernel(double *X, int rows, int r, long ld, const int *__restrict__ flip)
{
    const long total = (long)rows * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const int j = (int)(e % r);
        if (flip[j]) X[(e / r) * ld + j] = -X[(e / r) * ld + j];
    }
}

// canonical sign words (bit j % 32 of word [i, j / 32] set <=> X[i, j] < 0); then X = |X|
__global__ void pack_abs_kernel(double *X, int rows, int r, long ld, uint32_t *words)
{
    const int wpr = (r + 31) / 32;
    const long total = (long)rows * wpr;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const long i = e / wpr;
        const int w = (int)(e % wpr);
        uint32_t bits = 0;
        for (int b = 0; b < 32 && 32 * w + b < r; ++b) {
            double *x = X + i * ld + 32 * w + b;
            const double v = *x;
            bits |= (uint32_t)(v < 0.0) << b;
            *x = fabs(v);
        }
        words[e] = bits;
    }
}

// top eigenpair of an r x r Gram matrix after Jacobi: s = sqrt(lambda_max), b = its eigenvector with sum >= 0
// (zero when s == 0).  One CTA.
__global__ void __launch_bounds__(kT) top1_kernel(const double *M, const double *Mv, int r, long ld, double *b,
                                                  double *s_out)
{
    __shared__ double bv[kT];
    __shared__ int bi[kT];
    __shared__ double sum[kT];
    const int tid = threadIdx.x;
    double best = -INFINITY;
    int idx = 0x7fffffff;
    for (int j = tid; j < r; j += kT) {
        const double v = M[(long)j * ld + j];
        if (v > best) {
            best = v;
            idx = j;
        }
    }
    bv[tid] = best;
    bi[tid] = idx;
    __syncthreads();
    for (int o = kT / 2; o; o >>= 1) {
        if (tid < o && (bv[tid + o] > bv[tid] || (bv[tid + o] == bv[tid] && bi[tid + o] < bi[tid]))) {
            bv[tid] = bv[tid + o];
            bi[tid] = bi[tid + o];
        }
        __syncthreads();
    }
    const int top = bi[0];
    const double s = sqrt(fmax(bv[0], 0.0));
    double part = 0.0;
    for (int j = tid; j < r; j += kT) part += Mv[(long)top * ld + j];
    sum[tid] = part;
    __syncthreads();
    for (int o = kT / 2; o; o >>= 1) {
        if (tid < o) sum[tid] += sum[tid + o];
        __syncthreads();
    }
    const double sg = sum[0] < 0.0 ? -1.0 : 1.0;
    for (int j = tid; j < r; j += kT) b[j] = s > 0.0 ? sg * Mv[(long)top * ld + j] : 0.0;
    if (tid == 0) *s_out = s;
}

__global__ void vec_div_kernel(double *a, int n, const double *s)
{
    const double v = *s;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) a[i] = v > 0.0 ? a[i] / v : 0.0;
}

// l = s_u s_v (b_u (.) b_v); float32 copies of h, g, l and the singular values
__global__ void scales_out_kernel(const double *au, int N, const double *av, int K, const double *bu, const double *bv,
                                  const double *su, const double *sv, const double *sig, int r, double *ls, float *h,
                                  float *g, float *l, float *sigma)
{
    const double f = *su * *sv;
    const int n = max(max(N, K), r);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        if (i < N) h[i] = (float)au[i];
        if (i < K) g[i] = (float)av[i];
        if (i < r) {
            const double v = f * (bu[i] * bv[i]);
            ls[i] = v;
            l[i] = (float)v;
            if (sigma) sigma[i] = (float)sig[i];
        }
    }
}

// rows of a scaled sign factor from its packed words: out[i, j] = row_scale[i] * col_scale[j] * (+-1)
__global__ void signed_factor_kernel(const uint32_t *__restrict__ words, int rows, int r, const double *row_scale,
                                     const double *col_scale, double *out, long ld)
{
    const int wpr = (r + 31) / 32;
    const long total = (long)rows * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const long i = e / r;
        const int j = (int)(e % r);
        const bool neg = (words[i * wpr + j / 32] >> (j % 32)) & 1u;
        const double v = row_scale[i] * (col_scale ? col_scale[j] : 1.0);
        out[i * ld + j] = neg ? -v : v;
    }
}

// ---------------------------------------------------------------------------
// host steps
// ---------------------------------------------------------------------------
struct Ctx {
    const InitPlan &P;
    double *base;
    double *part;
    cudaStream_t s;
    double *at(size_t o) const { return base + o; }
    void gemm(bool ta, bool tb, int m, int n, int k, double alpha, const double *A, long lda, const double *B, long ldb,
              double beta, double *C, long ldc) const
    {
        dgemm(ta, tb, m, n, k, alpha, A, lda, B, ldb, beta, C, ldc, part, kDgemmPartElems, s);
    }
};

// X (rows x L, ld ldL) <- X R^{-1} with X^T X = R^T R (Cholesky QR); dependent columns become zero
void cholqr(const Ctx &c, double *X, int rows)
{
    const InitPlan &P = c.P;
    const int L = P.L;
    const long ld = P.ldL;
    double *S = c.at(P.o_S), *dg = c.at(P.o_dg), *inv = c.at(P.o_inv);
    c.gemm(true, false, L, L, rows, 1.0, X, ld, X, ld, 0.0, S, ld);
    copy_diag_kernel<<<grid_for(L), kT, 0, c.s>>>(S, L, ld, dg);
    for (int p = 0; p < P.npan; ++p) {
        const int k0 = p * kPanel, nb = std::min(kPanel, L - k0), rest = L - k0 - nb;
        double *ip = inv + (size_t)p * kPanel * kPanel;
        chol_diag_kernel<<<1, kT, kCholSmem, c.s>>>(S, ld, k0, nb, dg, ip);
        if (rest > 0) {
            double *L21 = S + (long)(k0 + nb) * ld + k0;
            c.gemm(false, true, rest, nb, nb, 1.0, L21, ld, ip, kPanel, 0.0, L21, ld);
            c.gemm(false, true, rest, rest, nb, -1.0, L21, ld, L21, ld, 1.0, S + (long)(k0 + nb) * ld + k0 + nb, ld);
        }
    }
    for (int p = 0; p < P.npan; ++p) {
        const int k0 = p * kPanel, nb = std::min(kPanel, L - k0);
        if (k0 > 0) c.gemm(false, true, rows, nb, k0, -1.0, X, ld, S + (long)k0 * ld, ld, 1.0, X + k0, ld);
        c.gemm(false, true, rows, nb, nb, 1.0, X + k0, ld, inv + (size_t)p * kPanel * kPanel, kPanel, 0.0, X + k0, ld);
    }
}

// Z = A X (X: nA x L) and its transpose product, with A = W or W^T
void apply_A(const Ctx &c, const double *X, double *Y)
{
    const InitPlan &P = c.P;
    if (!P.trans) c.gemm(false, false, P.N, P.L, P.K, 1.0, c.at(P.o_Wd), P.ldK, X, P.ldL, 0.0, Y, P.ldL);
    else c.gemm(true, false, P.K, P.L, P.N, 1.0, c.at(P.o_Wd), P.ldK, X, P.ldL, 0.0, Y, P.ldL);
}
void apply_At(const Ctx &c, const double *X, double *Y)
{
    const InitPlan &P = c.P;
    if (!P.trans) c.gemm(true, false, P.K, P.L, P.N, 1.0, c.at(P.o_Wd), P.ldK, X, P.ldL, 0.0, Y, P.ldL);
    else c.gemm(false, false, P.N, P.L, P.K, 1.0, c.at(P.o_Wd), P.ldK, X, P.ldL, 0.0, Y, P.ldL);
}

// rank-1 SVD of the non-negative X (rows x r, ld ldr): a (rows) = X b / s, b (r), s
cudaError_t rank1(const Ctx &c, const double *X, int rows, double *a, double *b, double *s, unsigned *bar, int *err)
{
    const InitPlan &P = c.P;
    const int r = P.r;
    double *M = c.at(P.o_M), *Mv = c.at(P.o_Mv);
    c.gemm(true, false, r, r, rows, 1.0, X, P.ldr, X, P.ldr, 0.0, M, P.ldr);
    cudaError_t e = jacobi_eig(M, r, P.ldr, Mv, P.ldr, c.at(P.o_side), bar, err, kMaxSweeps, c.s);
    if (e != cudaSuccess) return e;
    top1_kernel<<<1, kT, 0, c.s>>>(M, Mv, r, P.ldr, b, s);
    c.gemm(false, false, rows, 1, r, 1.0, X, P.ldr, b, 1, 0.0, a, 1);
    vec_div_kernel<<<grid_for(rows), kT, 0, c.s>>>(a, rows, s);
    return cudaGetLastError();
}

cudaError_t one_path(const Ctx &c, int iters, uint64_t seed, uint32_t *Uw, uint32_t *Vw, float *h, float *g, float *l,
                     float *sigma, bool residual_next, unsigned *bar, int *err, int *ord, int *flip)
{
    const InitPlan &P = c.P;
    const int N = P.N, K = P.K, r = P.r, L = P.L;
    double *Q = c.at(P.o_Q), *Z = c.at(P.o_Z), *T = c.at(P.o_T), *Vt = c.at(P.o_Vt), *G = c.at(P.o_G);
    double *E = c.at(P.o_E), *F = c.at(P.o_F), *Up = c.at(P.o_Up), *Vp = c.at(P.o_Vp);
    double *vec = c.at(P.o_vec);
    double *sig = vec, *bu = vec + r, *bv = vec + 2 * r, *ls = vec + 3 * r, *misc = vec + 4 * r;
    double *au = vec + 5 * r + 8, *av = au + 2 * (size_t)N;
    double *su = misc, *sv = misc + 1;

    // 1. truncated SVD
    if (L == P.nA) {
        identity_kernel<<<grid_for((long)L * L), kT, 0, c.s>>>(Q, L, P.ldL);
    } else {
        random_fill_kernel<<<grid_for((long)P.nA * L), kT, 0, c.s>>>(Q, P.nA, L, P.ldL, seed);
        cholqr(c, Q, P.nA);
        for (int it = 0; it < iters; ++it) {
            apply_A(c, Q, Z);
            cholqr(c, Z, P.mA);
            apply_At(c, Z, Q);
            cholqr(c, Q, P.nA);
        }
        cholqr(c, Q, P.nA);
    }
    apply_A(c, Q, Z);                                                   // P = A Q
    c.gemm(true, false, L, L, P.mA, 1.0, Z, P.ldL, Z, P.ldL, 0.0, T, P.ldL);
    cudaError_t e = jacobi_eig(T, L, P.ldL, Vt, P.ldL, c.at(P.o_side), bar, err, kMaxSweeps, c.s);
    if (e != cudaSuccess) return e;
    select_top_kernel<<<grid_for(L), kT, 0, c.s>>>(T, L, P.ldL, r, ord, sig);
    gather_rows_kernel<<<grid_for((long)r * L), kT, 0, c.s>>>(Vt, P.ldL, ord, r, L, G, P.ldL);
    c.gemm(false, true, P.nA, r, L, 1.0, Q, P.ldL, G, P.ldL, 0.0, E, P.ldr);   // right vectors of A
    c.gemm(false, true, P.mA, r, L, 1.0, Z, P.ldL, G, P.ldL, 0.0, F, P.ldr);   // left vectors of A times s

    // 2. U', V' (balanced), canonical pair signs, packed signs, magnitudes
    if (!P.trans) {
        col_scale_kernel<<<grid_for((long)N * r), kT, 0, c.s>>>(F, N, r, P.ldr, sig, 0, Up, P.ldr);
        col_scale_kernel<<<grid_for((long)K * r), kT, 0, c.s>>>(E, K, r, P.ldr, sig, 1, Vp, P.ldr);
    } else {
        col_scale_kernel<<<grid_for((long)N * r), kT, 0, c.s>>>(E, N, r, P.ldr, sig, 1, Up, P.ldr);
        col_scale_kernel<<<grid_for((long)K * r), kT, 0, c.s>>>(F, K, r, P.ldr, sig, 0, Vp, P.ldr);
    }
    col_sign_kernel<<<grid_for(32L * r), kT, 0, c.s>>>(Up, N, r, P.ldr, flip);
    col_flip_kernel<<<grid_for((long)N * r), kT, 0, c.s>>>(Up, N, r, P.ldr, flip);
    col_flip_kernel<<<grid_for((long)K * r), kT, 0, c.s>>>(Vp, K, r, P.ldr, flip);
    const int wpr = (r + 31) / 32;
    pack_abs_kernel<<<grid_for((long)N * wpr), kT, 0, c.s>>>(Up, N, r, P.ldr, Uw);
    pack_abs_kernel<<<grid_for((long)K * wpr), kT, 0, c.s>>>(Vp, K, r, P.ldr, Vw);

    // 3. rank-1 SVDs of the magnitudes -> h, g, l
    if ((e = rank1(c, Up, N, au, bu, su, bar, err)) != cudaSuccess) return e;
    if ((e = rank1(c, Vp, K, av, bv, sv, bar, err)) != cudaSuccess) return e;
    scales_out_kernel<<<grid_for(std::max(std::max(N, K), r)), kT, 0, c.s>>>(au, N, av, K, bu, bv, su, sv, sig, r, ls,
                                                                             h, g, l, sigma);

    // 4. target of the next path: W - diag(h) U_sign diag(l) V_sign^T diag(g)
    if (residual_next) {
        signed_factor_kernel<<<grid_for((long)N * r), kT, 0, c.s>>>(Uw, N, r, au, ls, F, P.ldr);
        signed_factor_kernel<<<grid_for((long)K * r), kT, 0, c.s>>>(Vw, K, r, av, nullptr, Z, P.ldr);
        c.gemm(false, true, N, K, r, -1.0, F, P.ldr, Z, P.ldr, 1.0, c.at(P.o_Wd), P.ldK);
    }
    return cudaGetLastError();
}

}  // namespace
}  // namespace lb

extern "C" LB_API size_t lb_dual_svid_workspace_bytes(int N, int K, int r)
{
    if (N < 1 || K < 1 || r < 1 || r > std::min(N, K) || r > LB_MAX_RANK) return 0;
    return lb::make_plan(N, K, r).total * sizeof(double);
}

extern "C" LB_API lb_status lb_dual_svid_init(const float *W, int N, int K, int r, int npaths, int iters,
                                              uint32_t *const *U, uint32_t *const *V, float *const *h,
                                              float *const *g, float *const *l, float *sigma, void *workspace,
                                              size_t workspace_bytes, void *stream)
{
    using namespace lb;
    if (N < 1 || K < 1 || r < 1 || r > std::min(N, K) || r > LB_MAX_RANK) return LB_ERR_INVALID_ARG;
    if (npaths != 1 && npaths != 2) return LB_ERR_UNSUPPORTED;
    if (!W || ((uintptr_t)W & 3) || iters < 0 || iters > 1000) return LB_ERR_INVALID_ARG;
    if (!U || !V || !h || !g || !l) return LB_ERR_INVALID_ARG;
    for (int p = 0; p < npaths; ++p)
        if (!U[p] || !V[p] || !h[p] || !g[p] || !l[p]) return LB_ERR_INVALID_ARG;
    const InitPlan P = make_plan(N, K, r);
    if (!workspace || ((uintptr_t)workspace & 255) || workspace_bytes < P.total * sizeof(double))
        return LB_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return LB_ERR_CUDA;

    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCholSmem) != cudaSuccess)
            return LB_ERR_CUDA;
        attr = true;
    }
    double *base = (double *)workspace;
    const Ctx c{P, base, base + P.o_part, s};
    int *ints = reinterpret_cast<int *>(base + P.o_int);
    unsigned *bar = reinterpret_cast<unsigned *>(ints);
    int *err = ints + 2, *ord = ints + 3, *flip = ints + 3 + r;
    if ((e = cudaMemsetAsync(err, 0, sizeof(int), s)) != cudaSuccess) return LB_ERR_CUDA;
    f32_to_f64_kernel<<<grid_for((long)N * K), kT, 0, s>>>(W, N, K, c.at(P.o_Wd), P.ldK);
    for (int p = 0; p < npaths && e == cudaSuccess; ++p)
        e = one_path(c, iters, 0x4C42495453564944ull + (uint64_t)p, U[p], V[p], h[p], g[p], l[p],
                     sigma ? sigma + (size_t)p * r : nullptr, p + 1 < npaths, bar, err, ord, flip);
    if (e != cudaSuccess) return LB_ERR_CUDA;
    int herr = 0;
    if (cudaMemcpyAsync(&herr, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LB_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LB_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return LB_ERR_CUDA;
    return herr ? LB_ERR_TIMEOUT : LB_OK;
}

// Dual-SVID + residual initialisation of a LittleBit layer from a dense weight
// (LittleBit paper notes page, "Dual-SVID initialisation" and "Residual
// compensation"), all in binary64 on the device.
//
// Per path, with A = W (K <= N) or A = W^T (K > N), so that A is mA x nA with
// nA = min(N, K):
//   1. truncated SVD by randomised subspace iteration: Q (nA x L) random,
//      then `iters` times Q = orth(A^T (A Q)), each orth a Cholesky QR (Gram
//      matrix; Cholesky factor and its inverse in one cooperative launch; one
//      GEMM; columns whose orthogonal part vanishes are dropped).  The Gram
//      matrix then has condition (s_1 / s_L)^4, inside binary64 for the
//      spectra of weight matrices; a second Cholesky QR pass at the end makes
//      Q orthonormal to working precision.  L = nA makes Q the identity and
//      the SVD exact.  Rayleigh-Ritz: P = A Q, T = P^T P = Z_T diag(lambda) Z_T^T by
//      Jacobi, the r largest lambda give s = sqrt(lambda), right vectors Q Z_r
//      and left vectors P Z_r / s;
//   2. U' = U_r sqrt(s), V' = V_r sqrt(s), each pair signed so that the
//      largest-magnitude entry of the U' column is positive; the sign bits
//      (set <=> < 0) are packed in the canonical layout;
//   3. rank-1 SVD of |U'| and |V'|: the top eigenpair of the r x r Gram matrix
//      (power iteration from the all-ones vector, which cannot be orthogonal
//      to the non-negative Perron vector) gives s_A^2 and b (signed to sum
//      >= 0), a = |U'| b / s_A;
//      h = a_u, g = a_v, l = s_u s_v (b_u (.) b_v);
//   4. the residual path repeats 1-3 on W - diag(h) U_sign diag(l) V_sign^T diag(g).
//
// LittleBit-2 (wiki page on LittleBit and LittleBit-2, section 1: latent
// rotation by joint iterative quantisation before QAT, initialisation only)
// inserts between 1 and 2 a rotation R of the latent space, which leaves
// U' V'^T unchanged: X = [U' / rho_u ; V' / rho_v] (each factor scaled to
// unit RMS entry), then `itq_iters` alternations of B = sign(X R) and
// R = polar(X^T B) (orthogonal Procrustes; the polar factor by Newton-Schulz
// iteration in one launch: one thread-block cluster for r <= 96, else a
// cooperative grid), and U' <- U' R, V' <- V' R before
// the signs.
#include "littlebit_init.h"
#include "lb_coop.cuh"
#include "lb_internal.cuh"
#include "lb_linalg.cuh"

#include <cooperative_groups.h>

#include <algorithm>
#include <math.h>

namespace lb {
namespace {

constexpr int kMaxSweeps = 40;
constexpr int kT = 256;
constexpr uint64_t kSeed = 0x4C42495453564944ull;   // start block of the primary path (the residual path adds 1)
constexpr int kPowerIters = 5000;       // bound of the rank-1 power iteration (converges in tens for such data)

long even(long x) { return (x + 1) & ~1L; }
size_t up32(size_t x) { return (x + 31) & ~size_t(31); }

struct InitPlan {
    int N, K, r, nA, mA, L;
    bool trans;               // A = W^T
    long ldK, ldL, ldr;
    size_t o_Wd, o_Q, o_Q2, o_Z, o_Z2, o_S, o_dg, o_Lf, o_Li, o_T, o_Vt, o_G, o_E, o_F, o_Up, o_Vp, o_M, o_vec, o_side,
        o_part;
    size_t o_X, o_Y, o_R, o_C, o_P0, o_P1, o_NS, o_red;   // Joint-ITQ (LittleBit-2) only
    bool itq;
    size_t o_int;             // int region (in doubles from the base)
    size_t total;             // doubles
};

constexpr int kRedBlocks = 296;        // CTAs of the fixed-order reductions (two per SM)
constexpr int kPolarMaxSteps = 60;     // Newton-Schulz steps at most: enough for sigma_min / ||C||_F down to ~1e-9
constexpr double kPolarStop = 1e-9;    // an update below this makes the new iterate exact to rounding (error squares)

InitPlan make_plan(int N, int K, int r, bool itq = false)
{
    InitPlan P{};
    P.itq = itq;
    P.N = N;
    P.K = K;
    P.r = r;
    P.trans = K > N;
    P.nA = std::min(N, K);
    P.mA = std::max(N, K);
    const int want = std::max(64, (2 * r + 63) / 64 * 64);
    P.L = std::min(P.nA, want);
    P.ldK = even(K);
    P.ldL = even(P.L);
    P.ldr = even(r);
    size_t o = 0;
    auto take = [&](size_t n) { const size_t at = o; o = up32(o + n); return at; };
    P.o_Wd = take((size_t)N * P.ldK);
    P.o_Q = take((size_t)P.nA * P.ldL);
    P.o_Q2 = take((size_t)P.nA * P.ldL);
    P.o_Z = take((size_t)P.mA * P.ldL);
    P.o_Z2 = take((size_t)P.mA * P.ldL);
    P.o_S = take((size_t)P.L * P.ldL);
    P.o_dg = take((size_t)P.L);
    P.o_Lf = take((size_t)P.L * P.ldL);
    P.o_Li = take((size_t)P.L * P.ldL);
    P.o_T = take((size_t)P.L * P.ldL);
    P.o_Vt = take((size_t)P.L * P.ldL);
    P.o_G = take((size_t)r * P.ldL);
    P.o_E = take((size_t)P.nA * P.ldr);
    P.o_F = take((size_t)P.mA * P.ldr);
    P.o_Up = take((size_t)N * P.ldr);
    P.o_Vp = take((size_t)K * P.ldr);
    P.o_M = take((size_t)r * P.ldr);
    P.o_vec = take((size_t)5 * r + 2 * (size_t)N + 2 * (size_t)K + 8);   // s, bu, bv, ls, misc | au, hs | av, gs
    P.o_side = take((size_t)3 * (P.L + 1));
    P.o_part = take(kDgemmPartElems);
    if (itq) {
        P.o_X = take((size_t)(N + K) * P.ldr);
        P.o_Y = take((size_t)(N + K) * P.ldr);
        P.o_R = take((size_t)r * P.ldr);
        P.o_C = take((size_t)r * P.ldr);
        P.o_P0 = take((size_t)r * P.ldr);
        P.o_P1 = take((size_t)r * P.ldr);
        P.o_NS = take((size_t)r * P.ldr);
        P.o_red = take((size_t)kRedBlocks + 8);
    }
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

// Leading eigenpair of the r x r Gram matrix M of a non-negative matrix by power iteration from the all-ones
// vector (not orthogonal to the non-negative Perron vector): b_{k+1} = M b_k / |M b_k| until no entry moves by more
// than 2e-15.  s = sqrt(b^T M b); b is signed to sum >= 0; M = 0 gives b = 0, s = 0.  One CTA, b in shared memory.
__global__ void __launch_bounds__(512) rank1_power_kernel(const double *__restrict__ M, int r, long ld, double *b,
                                                          double *s_out, int max_iter)
{
    extern __shared__ __align__(16) double pw[];
    double *bv = pw, *yv = pw + r;
    __shared__ double red[16];
    __shared__ double bcast;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    // block-wide sum (op = 0) or max (op = 1) of one value per thread
    auto reduce = [&](double v, int op) {
        for (int o = 16; o; o >>= 1) {
            const double w = __shfl_xor_sync(0xffffffffu, v, o);
            v = op ? fmax(v, w) : v + w;
        }
        __syncthreads();
        if (lane == 0) red[warp] = v;
        __syncthreads();
        if (tid == 0) {
            double a = red[0];
            for (int i = 1; i < nw; ++i) a = op ? fmax(a, red[i]) : a + red[i];
            bcast = a;
        }
        __syncthreads();
        return bcast;
    };
    // yv = M bv, one warp per row
    auto matvec = [&]() {
        for (int i = warp; i < r; i += nw) {
            double acc = 0.0;
            for (int j = lane; j < r; j += 32) acc += M[(long)i * ld + j] * bv[j];
            for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) yv[i] = acc;
        }
        __syncthreads();
    };
    for (int i = tid; i < r; i += blockDim.x) bv[i] = rsqrt((double)r);
    __syncthreads();
    bool zero = false;
    for (int it = 0; it < max_iter; ++it) {
        matvec();
        double loc = 0.0;
        for (int i = tid; i < r; i += blockDim.x) loc += yv[i] * yv[i];
        const double nrm2 = reduce(loc, 0);
        if (!(nrm2 > 0.0)) {
            zero = true;
            break;
        }
        const double inv = 1.0 / sqrt(nrm2);
        double diff = 0.0;
        for (int i = tid; i < r; i += blockDim.x) {
            const double v = yv[i] * inv;
            diff = fmax(diff, fabs(v - bv[i]));
            bv[i] = v;
        }
        if (reduce(diff, 1) <= 2e-15) break;
    }
    if (zero) {
        for (int i = tid; i < r; i += blockDim.x) b[i] = 0.0;
        if (tid == 0) *s_out = 0.0;
        return;
    }
    matvec();
    double q = 0.0, sm = 0.0;
    for (int i = tid; i < r; i += blockDim.x) {
        q += bv[i] * yv[i];
        sm += bv[i];
    }
    const double lam = reduce(q, 0);
    const double sg = reduce(sm, 0) < 0.0 ? -1.0 : 1.0;
    for (int i = tid; i < r; i += blockDim.x) b[i] = sg * bv[i];
    if (tid == 0) *s_out = sqrt(fmax(lam, 0.0));
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
// Joint-ITQ kernels (LittleBit-2)
// ---------------------------------------------------------------------------
// block-wide sum of one value per thread (kT threads); the result is valid in thread 0
__device__ double block_sum(double v)
{
    __shared__ double red[kT / 32];
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0)
        for (int w = 1; w < kT / 32; ++w) v += red[w];
    return v;
}

// part[b] = sum of X[i, j]^2 over this CTA's strided share of the entries (grid kRedBlocks x kT)
__global__ void __launch_bounds__(kT) sumsq_kernel(const double *X, int rows, int r, long ld, double *part)
{
    double acc = 0.0;
    const long total = (long)rows * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const double v = X[(e / r) * ld + e % r];
        acc += v * v;
    }
    acc = block_sum(acc);
    if (threadIdx.x == 0) part[blockIdx.x] = acc;
}

// out = scale * (part[0] + ... + part[n - 1]), summed in index order (one thread: deterministic)
__global__ void finalize_sum_kernel(const double *part, int n, double scale, double *out)
{
    double a = 0.0;
    for (int i = 0; i < n; ++i) a += part[i];
    *out = a * scale;
}

// 1 / RMS entry of a rows x r factor from its sum of squares (1 for a zero factor)
__device__ __forceinline__ double inv_rms(double ss, long n) { return ss > 0.0 ? 1.0 / sqrt(ss / (double)n) : 1.0; }

// X = [U' / rho_u ; V' / rho_v] ((N + K) x r, ld); ss = the two sums of squares
__global__ void itq_stack_kernel(const double *Up, int N, const double *Vp, int K, int r, long ld,
                                 const double *__restrict__ ss, double *X)
{
    const double fu = inv_rms(ss[0], (long)N * r), fv = inv_rms(ss[1], (long)K * r);
    const long total = (long)(N + K) * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const long i = e / r;
        const int j = (int)(e % r);
        X[i * ld + j] = i < N ? Up[i * ld + j] * fu : Vp[(i - N) * ld + j] * fv;
    }
}

// U' = rho_u Y[0 .. N), V' = rho_v Y[N .. N + K): the rotated factors at their own scale
__global__ void itq_unstack_kernel(const double *Y, int N, int K, int r, long ld, const double *__restrict__ ss,
                                   double *Up, double *Vp)
{
    const double fu = 1.0 / inv_rms(ss[0], (long)N * r), fv = 1.0 / inv_rms(ss[1], (long)K * r);
    const long total = (long)(N + K) * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        const long i = e / r;
        const int j = (int)(e % r);
        if (i < N) Up[i * ld + j] = Y[i * ld + j] * fu;
        else Vp[(i - N) * ld + j] = Y[i * ld + j] * fv;
    }
}

// part[b] = this CTA's share of sum (sign(Y) - Y)^2 (sign(0) = +1); with `write`, Y <- sign(Y)
__global__ void __launch_bounds__(kT) itq_sign_kernel(double *Y, int rows, int r, long ld, int write, double *part)
{
    double acc = 0.0;
    const long total = (long)rows * r;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        double *y = Y + (e / r) * ld + e % r;
        const double v = *y, b = v < 0.0 ? -1.0 : 1.0;
        acc += (b - v) * (b - v);
        if (write) *y = b;
    }
    acc = block_sum(acc);
    if (threadIdx.x == 0) part[blockIdx.x] = acc;
}

// block-wide max of one value per thread (kT threads); the result is valid in thread 0
__device__ double block_max(double v)
{
    __shared__ double red[kT / 32];
    for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0)
        for (int w = 1; w < kT / 32; ++w) v = fmax(v, red[w]);
    return v;
}

// Polar factor of C (r x r, ld) by Newton-Schulz iteration in one cooperative launch: X_0 = C / ||C||_F (all
// singular values in (0, 1]; C = 0 gives the identity), X_{k+1} = X_k (3 I - X_k^T X_k) / 2, until an update moves no
// entry by more than kPolarStop (the error of the new iterate is then ~the square of that: exact to rounding) or
// kPolarMaxSteps.  X, Xn, T: r x r scratch (ld); side: gridDim.x doubles; the result goes to R (ld).  Every CTA
// takes the same decisions from the same fixed-order sums, so all pass the same grid barriers.
__global__ void __launch_bounds__(kT) polar_ns_kernel(const double *C, int r, long ld, double *X, double *Xn,
                                                      double *T, double *side, double *R, unsigned *bar, int *err)
{
    __shared__ double sh;
    unsigned gen = 0;
    const long n2 = (long)r * r;
    const long tid = blockIdx.x * (long)blockDim.x + threadIdx.x, nth = (long)gridDim.x * blockDim.x;
    double acc = 0.0;
    for (long e = tid; e < n2; e += nth) {
        const double v = C[(e / r) * ld + e % r];
        acc += v * v;
    }
    acc = block_sum(acc);
    if (threadIdx.x == 0) side[blockIdx.x] = acc;
    if (!grid_barrier(bar, gen, err)) return;
    if (threadIdx.x == 0) {
        double a = 0.0;
        for (int b = 0; b < (int)gridDim.x; ++b) a += side[b];
        sh = sqrt(a);
    }
    __syncthreads();
    const double nrm = sh;
    for (long e = tid; e < n2; e += nth) {
        const long i = e / r, j = e % r;
        X[i * ld + j] = nrm > 0.0 ? C[i * ld + j] / nrm : (i == j ? 1.0 : 0.0);
    }
    if (!grid_barrier(bar, gen, err)) return;
    for (int k = 0; k < kPolarMaxSteps; ++k) {
        // T = (3 I - X^T X) / 2
        for (long e = tid; e < n2; e += nth) {
            const long i = e / r, j = e % r;
            double a = 0.0;
            for (int l = 0; l < r; ++l) a = fma(X[l * ld + i], X[l * ld + j], a);
            T[i * ld + j] = (i == j ? 1.5 : 0.0) - 0.5 * a;
        }
        if (!grid_barrier(bar, gen, err)) return;
        // X_{k+1} = X T and the largest change of an entry
        double dmax = 0.0;
        for (long e = tid; e < n2; e += nth) {
            const long i = e / r, j = e % r;
            double a = 0.0;
            for (int l = 0; l < r; ++l) a = fma(X[i * ld + l], T[l * ld + j], a);
            Xn[i * ld + j] = a;
            dmax = fmax(dmax, fabs(a - X[i * ld + j]));
        }
        dmax = block_max(dmax);
        if (threadIdx.x == 0) side[blockIdx.x] = dmax;
        if (!grid_barrier(bar, gen, err)) return;
        if (threadIdx.x == 0) {
            double m = 0.0;
            for (int b = 0; b < (int)gridDim.x; ++b) m = fmax(m, side[b]);
            sh = m;
        }
        __syncthreads();
        const double d = sh;
        double *t = X;
        X = Xn;
        Xn = t;
        if (d <= kPolarStop) break;
    }
    for (long e = tid; e < n2; e += nth) R[(e / r) * ld + e % r] = X[(e / r) * ld + e % r];
}

// The same iteration for small r in one thread-block cluster: kPolarCtas CTAs of kPolarThreads threads, the
// hardware cluster barrier in place of the grid barrier (all CTAs of a cluster are scheduled together).
constexpr int kPolarCtas = 8;           // portable cluster size
constexpr int kPolarThreads = 1024;
constexpr int kPolarClusterMaxR = 96;   // above this the grid-wide kernel (more SMs for the r^3 steps) is faster

// block-wide sum / max of one value per thread (any multiple of 32 threads up to 1024); valid in thread 0
__device__ double block_reduce_any(double v, bool is_max)
{
    __shared__ double red[32];
    for (int o = 16; o; o >>= 1) {
        const double w = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmax(v, w) : v + w;
    }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0)
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) v = is_max ? fmax(v, red[w]) : v + red[w];
    return v;
}

__global__ void __cluster_dims__(kPolarCtas, 1, 1) __launch_bounds__(kPolarThreads)
    polar_ns_cluster_kernel(const double *C, int r, long ld, double *X, double *Xn, double *T, double *side, double *R)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    __shared__ double sh;
    const long n2 = (long)r * r;
    const int rank = (int)cl.block_rank();
    const long tid = rank * (long)blockDim.x + threadIdx.x, nth = (long)kPolarCtas * blockDim.x;
    auto sync = [&]() {
        __threadfence();
        cl.sync();
    };
    double acc = 0.0;
    for (long e = tid; e < n2; e += nth) {
        const double v = C[(e / r) * ld + e % r];
        acc += v * v;
    }
    acc = block_reduce_any(acc, false);
    if (threadIdx.x == 0) side[rank] = acc;
    sync();
    if (threadIdx.x == 0) {
        double a = 0.0;
        for (int b = 0; b < kPolarCtas; ++b) a += side[b];
        sh = sqrt(a);
    }
    __syncthreads();
    const double nrm = sh;
    for (long e = tid; e < n2; e += nth) {
        const long i = e / r, j = e % r;
        X[i * ld + j] = nrm > 0.0 ? C[i * ld + j] / nrm : (i == j ? 1.0 : 0.0);
    }
    sync();
    for (int k = 0; k < kPolarMaxSteps; ++k) {
        for (long e = tid; e < n2; e += nth) {
            const long i = e / r, j = e % r;
            double a = 0.0;
            for (int l = 0; l < r; ++l) a = fma(X[l * ld + i], X[l * ld + j], a);
            T[i * ld + j] = (i == j ? 1.5 : 0.0) - 0.5 * a;
        }
        sync();
        double dmax = 0.0;
        for (long e = tid; e < n2; e += nth) {
            const long i = e / r, j = e % r;
            double a = 0.0;
            for (int l = 0; l < r; ++l) a = fma(X[i * ld + l], T[l * ld + j], a);
            Xn[i * ld + j] = a;
            dmax = fmax(dmax, fabs(a - X[i * ld + j]));
        }
        dmax = block_reduce_any(dmax, true);
        if (threadIdx.x == 0) side[rank] = dmax;
        sync();
        if (threadIdx.x == 0) {
            double m = 0.0;
            for (int b = 0; b < kPolarCtas; ++b) m = fmax(m, side[b]);
            sh = m;
        }
        __syncthreads();
        const double d = sh;
        double *t = X;
        X = Xn;
        Xn = t;
        if (d <= kPolarStop) break;
    }
    for (long e = tid; e < n2; e += nth) R[(e / r) * ld + e % r] = X[(e / r) * ld + e % r];
}

__global__ void copy_square_kernel(const double *src, int r, long lds, double *dst, long ldd)
{
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < r * r; e += gridDim.x * blockDim.x)
        dst[(long)(e / r) * ldd + e % r] = src[(long)(e / r) * lds + e % r];
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

// Xout = X R^{-1} with X^T X = R^T R (Cholesky QR; X and Xout rows x L, ld ldL); dependent columns become zero
cudaError_t cholqr(const Ctx &c, const double *X, int rows, double *Xout, unsigned *bar, int *err)
{
    const InitPlan &P = c.P;
    const int L = P.L;
    const long ld = P.ldL;
    double *S = c.at(P.o_S), *Lf = c.at(P.o_Lf), *Li = c.at(P.o_Li);
    c.gemm(true, false, L, L, rows, 1.0, X, ld, X, ld, 0.0, S, ld);
    cudaError_t e = chol_inverse(S, L, ld, Lf, Li, ld, c.at(P.o_dg), bar, err, c.s);
    if (e != cudaSuccess) return e;
    c.gemm(false, true, rows, L, L, 1.0, X, ld, Li, ld, 0.0, Xout, ld);
    return cudaSuccess;
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
void rank1(const Ctx &c, const double *X, int rows, double *a, double *b, double *s)
{
    const InitPlan &P = c.P;
    const int r = P.r;
    double *M = c.at(P.o_M);
    c.gemm(true, false, r, r, rows, 1.0, X, P.ldr, X, P.ldr, 0.0, M, P.ldr);
    rank1_power_kernel<<<1, 512, 2 * r * sizeof(double), c.s>>>(M, r, P.ldr, b, s, kPowerIters);
    c.gemm(false, false, rows, 1, r, 1.0, X, P.ldr, b, 1, 0.0, a, 1);
    vec_div_kernel<<<grid_for(rows), kT, 0, c.s>>>(a, rows, s);
}

// Joint-ITQ options of lb_littlebit2_init (none for lb_dual_svid_init)
struct ItqArgs {
    int iters = 0;
    const double *const *R0 = nullptr;   // host array of device r x r (ld r) starts, or null (identity)
    double *loss = nullptr;              // device [npaths][iters + 1], or null
    double *const *Rout = nullptr;       // host array of device r x r (ld r) outputs, or null
};

int sm_count_init()
{
    int n = 0;
    if (sm_count_of_current(&n) != cudaSuccess || n <= 0) n = 148;
    return n;
}

// R = polar factor of C (r x r, ld): one cooperative launch of polar_ns_kernel
cudaError_t polar(const Ctx &c, const double *C, double *R, double *X, double *Xn, double *T, double *side,
                  unsigned *bar, int *err)
{
    const InitPlan &P = c.P;
    const int r = P.r;
    long ld = P.ldr;
    if (r <= kPolarClusterMaxR) {
        polar_ns_cluster_kernel<<<kPolarCtas, kPolarThreads, 0, c.s>>>(C, r, ld, X, Xn, T, side, R);
        return cudaGetLastError();
    }
    const int grid = (int)std::max<long>(1, std::min<long>(std::min(sm_count_init(), kRedBlocks),
                                                           ((long)r * r + kT - 1) / kT));
    cudaError_t e = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned), c.s);
    if (e != cudaSuccess) return e;
    int rr = r;
    void *args[] = {(void *)&C, &rr, &ld, &X, &Xn, &T, &side, &R, &bar, &err};
    return cudaLaunchCooperativeKernel((const void *)polar_ns_kernel, dim3(grid), dim3(kT), args, 0, c.s);
}

// Rotate U', V' (N x r and K x r, ld ldr) by the Joint-ITQ rotation of path p (LittleBit-2).
cudaError_t joint_itq(const Ctx &c, const ItqArgs &a, int p, double *Up, double *Vp, unsigned *bar, int *err)
{
    const InitPlan &P = c.P;
    const int N = P.N, K = P.K, r = P.r, rows = N + K;
    const long ld = P.ldr;
    double *X = c.at(P.o_X), *Y = c.at(P.o_Y), *R = c.at(P.o_R), *C = c.at(P.o_C), *T = c.at(P.o_NS);
    double *Pa = c.at(P.o_P0), *Pb = c.at(P.o_P1);
    double *red = c.at(P.o_red), *ss = red + kRedBlocks, *scratch = ss + 2;
    sumsq_kernel<<<kRedBlocks, kT, 0, c.s>>>(Up, N, r, ld, red);
    finalize_sum_kernel<<<1, 1, 0, c.s>>>(red, kRedBlocks, 1.0, ss);
    sumsq_kernel<<<kRedBlocks, kT, 0, c.s>>>(Vp, K, r, ld, red);
    finalize_sum_kernel<<<1, 1, 0, c.s>>>(red, kRedBlocks, 1.0, ss + 1);
    itq_stack_kernel<<<grid_for((long)rows * r), kT, 0, c.s>>>(Up, N, Vp, K, r, ld, ss, X);
    if (a.R0 && a.R0[p]) copy_square_kernel<<<grid_for((long)r * r), kT, 0, c.s>>>(a.R0[p], r, r, R, ld);
    else identity_kernel<<<grid_for((long)r * r), kT, 0, c.s>>>(R, r, ld);
    const double inv_n = 1.0 / ((double)rows * r);
    for (int t = 0;; ++t) {
        const bool last = t == a.iters;
        c.gemm(false, false, rows, r, r, 1.0, X, ld, R, ld, 0.0, Y, ld);          // Y = X R
        itq_sign_kernel<<<kRedBlocks, kT, 0, c.s>>>(Y, rows, r, ld, last ? 0 : 1, red);
        finalize_sum_kernel<<<1, 1, 0, c.s>>>(red, kRedBlocks, inv_n,
                                              a.loss ? a.loss + (size_t)p * (a.iters + 1) + t : scratch);
        if (last) break;
        c.gemm(true, false, r, r, rows, 1.0, X, ld, Y, ld, 0.0, C, ld);           // C = X^T B
        cudaError_t e = polar(c, C, R, Pa, Pb, T, red, bar, err);                 // R = polar factor of C
        if (e != cudaSuccess) return e;
    }
    // Y = X R with the final R: back to each factor's own scale
    itq_unstack_kernel<<<grid_for((long)rows * r), kT, 0, c.s>>>(Y, N, K, r, ld, ss, Up, Vp);
    if (a.Rout && a.Rout[p]) copy_square_kernel<<<grid_for((long)r * r), kT, 0, c.s>>>(R, r, ld, a.Rout[p], r);
    return cudaGetLastError();
}

cudaError_t one_path(const Ctx &c, int iters, uint64_t seed, uint32_t *Uw, uint32_t *Vw, float *h, float *g, float *l,
                     float *sigma, bool residual_next, unsigned *bar, int *err, int *ord, int *flip,
                     const ItqArgs *itq = nullptr, int path = 0)
{
    const InitPlan &P = c.P;
    const int N = P.N, K = P.K, r = P.r, L = P.L;
    double *Q = c.at(P.o_Q), *Q2 = c.at(P.o_Q2), *Z = c.at(P.o_Z), *Z2 = c.at(P.o_Z2);
    double *T = c.at(P.o_T), *Vt = c.at(P.o_Vt), *G = c.at(P.o_G);
    double *E = c.at(P.o_E), *F = c.at(P.o_F), *Up = c.at(P.o_Up), *Vp = c.at(P.o_Vp);
    double *vec = c.at(P.o_vec);
    double *sig = vec, *bu = vec + r, *bv = vec + 2 * r, *ls = vec + 3 * r, *misc = vec + 4 * r;
    double *au = vec + 5 * r + 8, *av = au + 2 * (size_t)N;
    double *su = misc, *sv = misc + 1;

    // 1. truncated SVD (Q2, Z2: products before orthonormalisation)
    cudaError_t e = cudaSuccess;
    if (L == P.nA) {
        identity_kernel<<<grid_for((long)L * L), kT, 0, c.s>>>(Q, L, P.ldL);
    } else {
        random_fill_kernel<<<grid_for((long)P.nA * L), kT, 0, c.s>>>(Q2, P.nA, L, P.ldL, seed);
        if ((e = cholqr(c, Q2, P.nA, Q, bar, err)) != cudaSuccess) return e;
        for (int it = 0; it < iters; ++it) {
            // timing hook (primary path, first iteration): events 0 | A Q | 1 | A^T (A Q) | 2
            const bool mark = seed == kSeed && it == 0;
            if (mark) profile_mark(0, c.s);
            apply_A(c, Q, Z2);
            if (mark) profile_mark(1, c.s);
            apply_At(c, Z2, Q2);
            if (mark) profile_mark(2, c.s);
            if ((e = cholqr(c, Q2, P.nA, Q, bar, err)) != cudaSuccess) return e;
        }
        // a second pass: orthonormal to working precision for the Rayleigh-Ritz step
        if ((e = cholqr(c, Q, P.nA, Q2, bar, err)) != cudaSuccess) return e;
        std::swap(Q, Q2);
    }
    apply_A(c, Q, Z);                                                   // P = A Q
    c.gemm(true, false, L, L, P.mA, 1.0, Z, P.ldL, Z, P.ldL, 0.0, T, P.ldL);
    e = jacobi_eig(T, L, P.ldL, Vt, P.ldL, c.at(P.o_side), bar, err, kMaxSweeps, c.s);
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
    if (itq) {
        // LittleBit-2 latent rotation, started from the canonically signed factors
        col_sign_kernel<<<grid_for(32L * r), kT, 0, c.s>>>(Up, N, r, P.ldr, flip);
        col_flip_kernel<<<grid_for((long)N * r), kT, 0, c.s>>>(Up, N, r, P.ldr, flip);
        col_flip_kernel<<<grid_for((long)K * r), kT, 0, c.s>>>(Vp, K, r, P.ldr, flip);
        if ((e = joint_itq(c, *itq, path, Up, Vp, bar, err)) != cudaSuccess) return e;
    }
    col_sign_kernel<<<grid_for(32L * r), kT, 0, c.s>>>(Up, N, r, P.ldr, flip);
    col_flip_kernel<<<grid_for((long)N * r), kT, 0, c.s>>>(Up, N, r, P.ldr, flip);
    col_flip_kernel<<<grid_for((long)K * r), kT, 0, c.s>>>(Vp, K, r, P.ldr, flip);
    const int wpr = (r + 31) / 32;
    pack_abs_kernel<<<grid_for((long)N * wpr), kT, 0, c.s>>>(Up, N, r, P.ldr, Uw);
    pack_abs_kernel<<<grid_for((long)K * wpr), kT, 0, c.s>>>(Vp, K, r, P.ldr, Vw);

    // 3. rank-1 SVDs of the magnitudes -> h, g, l
    rank1(c, Up, N, au, bu, su);
    rank1(c, Vp, K, av, bv, sv);
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

namespace lb {
namespace {

lb_status run_init(const float *W, int N, int K, int r, int npaths, int iters, uint32_t *const *U, uint32_t *const *V,
                   float *const *h, float *const *g, float *const *l, float *sigma, void *workspace,
                   size_t workspace_bytes, void *stream, const ItqArgs *itq)
{
    if (N < 1 || K < 1 || r < 1 || r > std::min(N, K) || r > LB_MAX_RANK) return LB_ERR_INVALID_ARG;
    if (npaths != 1 && npaths != 2) return LB_ERR_UNSUPPORTED;
    if (!W || ((uintptr_t)W & 3) || iters < 0 || iters > 1000) return LB_ERR_INVALID_ARG;
    if (!U || !V || !h || !g || !l) return LB_ERR_INVALID_ARG;
    for (int p = 0; p < npaths; ++p)
        if (!U[p] || !V[p] || !h[p] || !g[p] || !l[p]) return LB_ERR_INVALID_ARG;
    const InitPlan P = make_plan(N, K, r, itq != nullptr);
    if (!workspace || ((uintptr_t)workspace & 255) || workspace_bytes < P.total * sizeof(double))
        return LB_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return LB_ERR_CUDA;

    double *base = (double *)workspace;
    const Ctx c{P, base, base + P.o_part, s};
    int *ints = reinterpret_cast<int *>(base + P.o_int);
    unsigned *bar = reinterpret_cast<unsigned *>(ints);
    int *err = ints + 2, *ord = ints + 3, *flip = ints + 3 + r;
    if ((e = cudaMemsetAsync(err, 0, sizeof(int), s)) != cudaSuccess) return LB_ERR_CUDA;
    f32_to_f64_kernel<<<grid_for((long)N * K), kT, 0, s>>>(W, N, K, c.at(P.o_Wd), P.ldK);
    for (int p = 0; p < npaths && e == cudaSuccess; ++p)
        e = one_path(c, iters, kSeed + (uint64_t)p, U[p], V[p], h[p], g[p], l[p],
                     sigma ? sigma + (size_t)p * r : nullptr, p + 1 < npaths, bar, err, ord, flip, itq, p);
    if (e != cudaSuccess) return LB_ERR_CUDA;
    int herr = 0;
    if (cudaMemcpyAsync(&herr, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LB_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LB_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return LB_ERR_CUDA;
    return herr ? LB_ERR_TIMEOUT : LB_OK;
}

}  // namespace
}  // namespace lb

extern "C" LB_API lb_status lb_dual_svid_init(const float *W, int N, int K, int r, int npaths, int iters,
                                              uint32_t *const *U, uint32_t *const *V, float *const *h,
                                              float *const *g, float *const *l, float *sigma, void *workspace,
                                              size_t workspace_bytes, void *stream)
{
    return lb::run_init(W, N, K, r, npaths, iters, U, V, h, g, l, sigma, workspace, workspace_bytes, stream, nullptr);
}

extern "C" LB_API size_t lb_littlebit2_workspace_bytes(int N, int K, int r)
{
    if (N < 1 || K < 1 || r < 1 || r > std::min(N, K) || r > LB_MAX_RANK) return 0;
    return lb::make_plan(N, K, r, true).total * sizeof(double);
}

extern "C" LB_API lb_status lb_littlebit2_init(const float *W, int N, int K, int r, int npaths, int iters,
                                               int itq_iters, const double *const *R0, uint32_t *const *U,
                                               uint32_t *const *V, float *const *h, float *const *g,
                                               float *const *l, float *sigma, double *itq_loss, double *const *R_out,
                                               void *workspace, size_t workspace_bytes, void *stream)
{
    if (itq_iters < 0 || itq_iters > 1000) return LB_ERR_INVALID_ARG;
    if (npaths == 1 || npaths == 2) {
        for (int p = 0; p < npaths; ++p) {
            if (R0 && R0[p] && ((uintptr_t)R0[p] & 7)) return LB_ERR_INVALID_ARG;
            if (R_out && R_out[p] && ((uintptr_t)R_out[p] & 7)) return LB_ERR_INVALID_ARG;
        }
    }
    if ((uintptr_t)itq_loss & 7) return LB_ERR_INVALID_ARG;
    lb::ItqArgs a;
    a.iters = itq_iters;
    a.R0 = R0;
    a.loss = itq_loss;
    a.Rout = R_out;
    return lb::run_init(W, N, K, r, npaths, iters, U, V, h, g, l, sigma, workspace, workspace_bytes, stream, &a);
}

// Cholesky factor and its inverse in one cooperative launch, for the Cholesky
// QR of the initialisation path: given the Gram matrix S = X^T X (n x n) it
// returns Linv = L^{-1} with S = L L^T, so that X Linv^T has orthonormal
// columns (one GEMM).
//
// Right-looking blocked algorithm, 64-wide panels; per panel k:
//   A. one CTA factors the diagonal block (its Schur complement) in shared
//      memory and inverts the factor, both blocked in 16-wide sub-panels; a
//      pivot at or below kDepTol times the column's original squared norm
//      marks a dependent column: its factor column becomes e_j and its row of
//      the inverse zero, i.e. the column is dropped;
//   B. all CTAs: the panel below, L21 = S21 Inv_kk^T (64-row tiles);
//   C. all CTAs: the trailing update S22 -= L21 L21^T (64 x 64 tiles of the
//      lower triangle);
// then the off-diagonal blocks of the inverse, one block row at a time:
//   D. Linv_ij = -Inv_ii sum_{k=j}^{i-1} L_ik Linv_kj.
// Phases are separated by grid-wide barriers with bounded waits.
#include "lb_linalg.cuh"
#include "lb_coop.cuh"

#include <algorithm>
#include <math.h>

namespace lb {
namespace {

constexpr int kB = 64, kCT = 256;
constexpr int kLd = kB + 1;
constexpr double kDepTol = 1e-13;
// shared memory: three 64 x 65 tiles
constexpr size_t kCholSmem = 3 * kB * kLd * sizeof(double);

using Tile = double[kLd];

// T (rows x cols, zero outside) = the rows x cols block at src, or with `trans` the transpose of the
// cols x rows block at src
__device__ void load_tile(Tile *T, const double *src, long ld, int rows, int cols, bool trans)
{
    // all 16 loads of a thread are issued before the first store
    constexpr int kPer = kB * kB / kCT;
    double v[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int e = threadIdx.x + q * kCT, i = e / kB, j = e % kB;
        const bool in = trans ? (i < cols && j < rows) : (i < rows && j < cols);
        v[q] = in ? __ldcg(src + (long)i * ld + j) : 0.0;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int e = threadIdx.x + q * kCT, i = e / kB, j = e % kB;
        if (trans) T[j][i] = v[q];
        else T[i][j] = v[q];
    }
}

// acc (this thread's rows ty + 16a, cols tx + 16b) += A[64 x 64] B[64 x 64]
__device__ __forceinline__ void tile_mma(double (&acc)[4][4], const Tile *A, const Tile *B)
{
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 4
    for (int k = 0; k < kB; ++k) {
        double a[4], b[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            a[q] = A[ty + 16 * q][k];
            b[q] = B[k][tx + 16 * q];
        }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[p][q] = fma(a[p], b[q], acc[p][q]);
    }
}

__device__ __forceinline__ void zero_acc(double (&acc)[4][4])
{
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = 0.0;
}

// Cholesky factor F (lower) of the nb x nb block whose lower triangle is in D (overwritten), and X = F^{-1},
// in 16-wide sub-panels: (a) one warp factors the 16 x 16 diagonal sub-block (a lane per row), (b) the rows below
// are solved against it, (c) the trailing part of D is updated; then X by inverting the 16 x 16 diagonal blocks
// (a warp each, a lane per column) and block rows X_ij = -X_ii sum_k F_ik X_kj.  A pivot at or below kDepTol
// times the column's original squared norm (dgs) marks a dependent column: factor column e_j, inverse row 0.
__device__ void factor_invert(Tile *D, Tile *F, Tile *X, int nb, const double *dgs, int *dep, double *rdg)
{
    constexpr int kS = 16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int sp = 0; sp < nb; sp += kS) {
        const int w = min(kS, nb - sp);
        if (warp == 0) {                                     // (a)
            const int i = sp + lane;
            for (int j = sp; j < sp + w; ++j) {
                const double d = D[j][j];
                const bool bad = !(d > kDepTol * dgs[j]) || !(d > 0.0);
                const double sd = bad ? 1.0 : sqrt(d);
                const double rsd = 1.0 / sd;
                if (lane < w && i > j) {
                    const double dij = D[i][j];
                    F[i][j] = bad ? 0.0 : dij * rsd;
                    if (!bad) {
                        const double lij = dij / d;       // one division per row and step, none in the loop
                        for (int m = j + 1; m <= i; ++m) D[i][m] -= lij * D[m][j];
                    }
                }
                if (lane == 0) {
                    F[j][j] = sd;
                    rdg[j] = bad ? 0.0 : rsd;             // reciprocal diagonal; 0 drops a dependent column
                    dep[j] = bad;
                }
                __syncwarp();
            }
        }
        __syncthreads();
        for (int i = sp + w + tid; i < nb; i += kCT) {       // (b)
            for (int c = 0; c < w; ++c) {
                const int jc = sp + c;
                double acc = D[i][jc];
                for (int m = 0; m < c; ++m) acc -= F[i][sp + m] * F[jc][sp + m];
                F[i][jc] = acc * rdg[jc];
            }
        }
        __syncthreads();
        const int r0 = sp + w, nr = nb - r0;                 // (c) lower triangle of the trailing block
        for (int e2 = tid; e2 < nr * nr; e2 += kCT) {
            const int i = r0 + e2 / nr, m = r0 + e2 % nr;
            if (m > i) continue;
            double acc = 0.0;
#pragma unroll 4
            for (int c = 0; c < w; ++c) acc += F[i][sp + c] * F[m][sp + c];
            D[i][m] -= acc;
        }
        __syncthreads();
    }
    // inverse: diagonal 16 x 16 blocks
    const int nsub = (nb + kS - 1) / kS;
    if (warp < nsub && lane < kS) {
        const int b0 = warp * kS, w = min(kS, nb - b0), c = lane;
        if (c < w)
            for (int i = c; i < w; ++i) {
                double acc = 0.0;
                for (int m = c; m < i; ++m) acc += F[b0 + i][b0 + m] * X[b0 + m][b0 + c];
                X[b0 + i][b0 + c] = ((i == c ? 1.0 : 0.0) - acc) * rdg[b0 + i];
            }
    }
    __syncthreads();
    // off-diagonal blocks, one block row at a time; D (no longer needed) holds the sums
    for (int bi = 1; bi < nsub; ++bi) {
        const int i0 = bi * kS, wi = min(kS, nb - i0);
        for (int e2 = tid; e2 < bi * kS * kS; e2 += kCT) {
            const int bj = e2 / (kS * kS), r = (e2 / kS) % kS, c = e2 % kS;
            double acc = 0.0;
            if (r < wi)
                for (int q = bj * kS; q < i0; ++q) acc += F[i0 + r][q] * X[q][bj * kS + c];
            D[r][bj * kS + c] = acc;
        }
        __syncthreads();
        for (int e2 = tid; e2 < bi * kS * kS; e2 += kCT) {
            const int bj = e2 / (kS * kS), r = (e2 / kS) % kS, c = e2 % kS;
            if (r >= wi) continue;
            double acc = 0.0;
            for (int q = 0; q <= r; ++q) acc += X[i0 + r][i0 + q] * D[q][bj * kS + c];
            X[i0 + r][bj * kS + c] = -acc;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kCT, 1)
    chol_inv_kernel(double *S, int n, long ldS, double *Lf, double *Linv, long ldI, double *dg, unsigned *bar, int *err)
{
    extern __shared__ __align__(16) unsigned char smem[];
    Tile *T0 = reinterpret_cast<Tile *>(smem);
    Tile *T1 = T0 + kB;
    Tile *T2 = T1 + kB;
    __shared__ int dep[kB];
    __shared__ double dgs[kB];
    __shared__ double rdg[kB];

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int npan = (n + kB - 1) / kB;
    unsigned gen = 0;
    const long gtid = blockIdx.x * (long)kCT + tid, gstride = (long)gridDim.x * kCT;
    for (long e = gtid; e < (long)n * n; e += gstride) {
        const long i = e / n, j = e % n;
        Linv[i * ldI + j] = 0.0;
        Lf[i * ldI + j] = 0.0;
        if (i == j) dg[i] = S[i * ldS + i];
    }
    if (!grid_barrier(bar, gen, err)) return;

    for (int k = 0; k < npan; ++k) {
        const int k0 = k * kB, nb = min(kB, n - k0), rest = n - k0 - nb;
        // ---- A: factor and invert the diagonal block (CTA 0)
        if (blockIdx.x == 0) {
            Tile *D = T0, *F = T1, *X = T2;
            for (int e2 = tid; e2 < kB * kB; e2 += kCT) {
                const int i = e2 / kB, j = e2 % kB;
                D[i][j] = (i < nb && j <= i) ? __ldcg(S + (long)(k0 + i) * ldS + k0 + j) : 0.0;
                F[i][j] = 0.0;
                X[i][j] = 0.0;
            }
            for (int i = tid; i < nb; i += kCT) dgs[i] = __ldcg(dg + k0 + i);
            __syncthreads();
            factor_invert(D, F, X, nb, dgs, dep, rdg);
            for (int e2 = tid; e2 < kB * kB; e2 += kCT) {
                const int i = e2 / kB, j = e2 % kB;
                if (i < nb && j <= i) {
                    Lf[(long)(k0 + i) * ldI + k0 + j] = F[i][j];
                    Linv[(long)(k0 + i) * ldI + k0 + j] = X[i][j];
                }
            }
        }
        if (!grid_barrier(bar, gen, err)) return;
        if (rest > 0) {
            // ---- B: L21 = S21 Inv_kk^T, one 64-row tile per CTA
            const int tiles = (rest + kB - 1) / kB;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
                const int r0 = k0 + nb + t * kB, rows = min(kB, n - r0);
                load_tile(T0, S + (long)r0 * ldS + k0, ldS, rows, nb, false);
                load_tile(T1, Linv + (long)k0 * ldI + k0, ldI, nb, nb, true);     // Inv_kk^T
                __syncthreads();
                double acc[4][4];
                zero_acc(acc);
                tile_mma(acc, T0, T1);
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i = ty + 16 * p, j = tx + 16 * q;
                        if (i < rows && j < nb) Lf[(long)(r0 + i) * ldI + k0 + j] = acc[p][q];
                    }
                __syncthreads();
            }
            if (!grid_barrier(bar, gen, err)) return;
            // ---- C: S22 -= L21 L21^T on the lower-triangle tiles
            const int tp = tiles * (tiles + 1) / 2;
            for (int t = blockIdx.x; t < tp; t += gridDim.x) {
                int bi = 0;
                while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
                const int bj = t - bi * (bi + 1) / 2;
                const int i0 = k0 + nb + bi * kB, j0 = k0 + nb + bj * kB;
                const int ri = min(kB, n - i0), rj = min(kB, n - j0);
                load_tile(T0, Lf + (long)i0 * ldI + k0, ldI, ri, nb, false);
                load_tile(T1, Lf + (long)j0 * ldI + k0, ldI, nb, rj, true);    // (L21 rows of block j)^T
                __syncthreads();
                double acc[4][4];
                zero_acc(acc);
                tile_mma(acc, T0, T1);
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i = ty + 16 * p, j = tx + 16 * q;
                        if (i < ri && j < rj && j0 + j <= i0 + i) {
                            double *s = S + (long)(i0 + i) * ldS + j0 + j;
                            *s = __ldcg(s) - acc[p][q];
                        }
                    }
                __syncthreads();
            }
            if (!grid_barrier(bar, gen, err)) return;
        }
    }
    // ---- D: off-diagonal blocks of the inverse, block row by block row
    for (int bi = 1; bi < npan; ++bi) {
        const int i0 = bi * kB, ri = min(kB, n - i0);
        for (int bj = blockIdx.x; bj < bi; bj += gridDim.x) {
            const int j0 = bj * kB;
            double acc[4][4];
            zero_acc(acc);
            for (int bk = bj; bk < bi; ++bk) {
                const int k0 = bk * kB;
                load_tile(T0, Lf + (long)i0 * ldI + k0, ldI, ri, kB, false);
                load_tile(T1, Linv + (long)k0 * ldI + j0, ldI, kB, kB, false);
                __syncthreads();
                tile_mma(acc, T0, T1);
                __syncthreads();
            }
            // T2 = the sum; Linv_ij = -Inv_ii T2
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) T2[ty + 16 * p][tx + 16 * q] = acc[p][q];
            load_tile(T0, Linv + (long)i0 * ldI + i0, ldI, ri, ri, false);
            __syncthreads();
            zero_acc(acc);
            tile_mma(acc, T0, T2);
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = ty + 16 * p, j = tx + 16 * q;
                    if (i < ri) Linv[(long)(i0 + i) * ldI + j0 + j] = -acc[p][q];
                }
            __syncthreads();
        }
        if (!grid_barrier(bar, gen, err)) return;
    }
}

int sm_count_c()
{
    int n = 0;
    if (sm_count_of_current(&n) != cudaSuccess || n <= 0) n = 148;
    return n;
}

}  // namespace

cudaError_t chol_inverse(double *S, int n, long ldS, double *Lf, double *Linv, long ldI, double *dg, unsigned *bar,
                         int *err, cudaStream_t s)
{
    if (n < 1) return cudaErrorInvalidValue;
    {
        const cudaError_t e = ensure_dyn_smem((const void *)chol_inv_kernel, kCholSmem);
        if (e != cudaSuccess) return e;
    }
    const int npan = (n + kB - 1) / kB;
    const int tiles = std::max(1, npan - 1);
    const int grid = std::max(1, std::min(sm_count_c(), tiles * (tiles + 1) / 2));
    cudaError_t e = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    void *args[] = {&S, &n, &ldS, &Lf, &Linv, &ldI, &dg, &bar, &err};
    return cudaLaunchCooperativeKernel((const void *)chol_inv_kernel, dim3(grid), dim3(kCT), args, kCholSmem, s);
}

}  // namespace lb

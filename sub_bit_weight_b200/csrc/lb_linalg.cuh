// Internal dense binary64 linear algebra of the initialisation path (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lb {

// Shared with the rest of the library (defined with the layer code): raise a kernel's dynamic shared-memory
// limit on the current device (per device and kernel, thread-safe), and the current device's SM count.
cudaError_t ensure_dyn_smem(const void *fn, size_t bytes);
cudaError_t sm_count_of_current(int *sms);

// Row-major matrix view: element (i, j) at p[i * ld + j].
struct DView {
    double *p;
    long ld;
};

// C = alpha * op(A) * op(B) + beta * C, all row-major binary64; op(A) is m x k,
// op(B) is k x n (ta / tb: the stored matrix is the transpose).  beta == 0
// does not read C.  `part` (may be null) is scratch of `part_elems` doubles
// that lets the k range be split over CTAs; with it the sum is formed in a
// fixed order (deterministic).  C may alias A only when n <= 64 (each CTA then
// owns whole rows of C and reads only those rows of A before writing).
void dgemm(bool ta, bool tb, int m, int n, int k, double alpha, const double *A, long lda, const double *B,
           long ldb, double beta, double *C, long ldc, double *part, size_t part_elems, cudaStream_t s);

// Scratch (doubles) dgemm uses at most for its split-k partial sums.
constexpr size_t kDgemmPartElems = size_t(20) << 20;

// Symmetric eigendecomposition by cyclic Jacobi rotations (one cooperative
// launch, one CTA per SM, grid-wide barriers with bounded waits).  A (n x n,
// full symmetric storage, ld lda) is overwritten: its diagonal holds the
// eigenvalues.  Vt (n x n, ld ldv) receives the eigenvectors as ROWS, in the
// order of the diagonal.  `side` is 3 * (n + 1) doubles and `bar` 2 unsigned
// of device scratch; `err` gets a nonzero code if a barrier wait gave up.
// n <= kJacobiMaxN.
constexpr int kJacobiMaxN = 4096;
cudaError_t jacobi_eig(double *A, int n, long lda, double *Vt, long ldv, double *side, unsigned *bar, int *err,
                       int max_sweeps, cudaStream_t s);

// Cholesky factor of the Gram matrix S (n x n, lower triangle read and
// overwritten) and its inverse, in one cooperative launch: Linv (n x n, ld
// ldI, lower triangular) = L^{-1} with S = L L^T, so X Linv^T has orthonormal
// columns when S = X^T X.  A column whose pivot falls to 1e-13 times its
// original squared norm or below counts as dependent and is dropped (its row
// of Linv is zero).  Lf (n x n, ld ldI) and dg (n) are scratch.
cudaError_t chol_inverse(double *S, int n, long ldS, double *Lf, double *Linv, long ldI, double *dg, unsigned *bar,
                         int *err, cudaStream_t s);

}  // namespace lb

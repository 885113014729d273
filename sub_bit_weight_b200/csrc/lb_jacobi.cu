// Symmetric eigendecomposition by parallel cyclic Jacobi (two-sided rotations),
// for the small dense problems of the initialisation path (the Rayleigh-Ritz
// matrix of the truncated SVD and the Gram matrices of the rank-1 SVDs).
//
// Rotation of the pair (p, q) (Golub & Van Loan, "Matrix Computations",
// symmetric Schur decomposition): tau = (a_qq - a_pp) / (2 a_pq),
// t = sign(tau) / (|tau| + sqrt(1 + tau^2)), c = 1 / sqrt(1 + t^2), s = t c;
// with J = [[c, s], [-s, c]] on (p, q), (J^T A J)_pq = 0, a_pp -= t a_pq,
// a_qq += t a_pq.  A rotation is skipped when |a_pq| <= tol sqrt(|a_pp a_qq|)
// (the threshold that gives eigenvalues to high relative accuracy); the
// iteration stops after a sweep whose rotations all had |a_pq| <= 1e-12
// sqrt(|a_pp a_qq|) (convergence is quadratic, so the next sweep would leave
// off-diagonal entries of order 1e-24 of the diagonal over the eigenvalue gaps).
//
// Parallel ordering: the round-robin ("circle") tournament, n/2 disjoint
// pairs per round, n-1 rounds per sweep.  Position 0 is fixed, positions
// 1..n-1 rotate by one each round; pair k of round t joins the indices at
// positions k and n-1-k.  Within a round all rotations commute, so each 2x2
// block A[{p_i, q_i}, {p_j, q_j}] becomes J_i^T B J_j independently: one
// thread per block, every element written exactly once.  The eigenvectors are
// accumulated as rows of Vt <- J^T Vt.  Every CTA computes all rotations of a
// round itself (into shared memory) from copies of the round's pivot
// elements that the previous round wrote to a double-buffered side array, so
// a round needs a single grid-wide barrier; the barrier waits are bounded and
// report through `err`.
#include "lb_linalg.cuh"
#include "lb_coop.cuh"

#include <algorithm>
#include <math.h>

namespace lb {
namespace {

constexpr int kJThreads = 512;
constexpr double kJTol = 1e-15;
constexpr double kJStop = 1e-12;

__device__ __forceinline__ int circle_index(int pos, int t, int np)
{
    return pos == 0 ? 0 : 1 + (pos - 1 + t) % (np - 1);
}

__global__ void __launch_bounds__(kJThreads, 1)
    jacobi_kernel(double *A, int n, long lda, double *Vt, long ldv, double *side, unsigned *bar, int *err,
                  int max_sweeps)
{
    extern __shared__ __align__(16) unsigned char jsm[];
    const int np = n + (n & 1), H = np / 2;
    double *cs = reinterpret_cast<double *>(jsm);
    double *sn = cs + H;
    double *tv = sn + H;
    int *P = reinterpret_cast<int *>(tv + H);
    int *Q = P + H;
    int *nq = Q + H;          // next round: partner q of index x when x is the p side of a pair, else -1
    int *nk = nq + np;        // next round: pair number of that pair
    // The rotations of a round are computed from copies of its pivot elements (the diagonal and the round's
    // pair entries A[p][q]), written by the previous round into the other half of `side`; A itself is updated
    // in place while other CTAs may still be computing their rotations.
    double *dgs[2] = {side, side + np};
    double *ods[2] = {side + 2 * np, side + 2 * np + H};

    unsigned gen = 0;
    const long gtid = blockIdx.x * (long)blockDim.x + threadIdx.x, gstride = (long)gridDim.x * blockDim.x;
    for (long e = gtid; e < (long)n * n; e += gstride) {
        const long i = e / n, j = e % n;
        Vt[i * ldv + j] = i == j ? 1.0 : 0.0;
    }
    for (long x = gtid; x < np; x += gstride) dgs[0][x] = x < n ? A[x * lda + x] : 0.0;
    for (long k = gtid; k < H; k += gstride) {
        const int p = circle_index((int)k, 0, np), q = circle_index(np - 1 - (int)k, 0, np);
        ods[0][k] = (p < n && q < n) ? A[p * lda + q] : 0.0;
    }
    if (!grid_barrier(bar, gen, err)) return;

    const int nblocks = H * H, nvt = H * n;     // 2x2 blocks of A, row-pair entries of Vt (< 2^31 for n <= 4096)
    const int gt = (int)gtid, gs = (int)gstride;
    int b = 0;
    for (int sweep = 0; sweep < max_sweeps; ++sweep) {
        double worst = 0.0;      // largest |a_pq| / sqrt(|a_pp a_qq|) rotated in this sweep
        for (int t = 0; t < np - 1; ++t) {
            const int tn = (t + 1) % (np - 1);
            const double *dgc = dgs[b], *odc = ods[b];
            double *dgn = dgs[b ^ 1], *odn = ods[b ^ 1];
            for (int k = threadIdx.x; k < H; k += blockDim.x) {
                const int p = circle_index(k, t, np), q = circle_index(np - 1 - k, t, np);
                double c = 1.0, s = 0.0, tt = 0.0;
                if (p < n && q < n) {
                    const double app = __ldcg(dgc + p), aqq = __ldcg(dgc + q), apq = __ldcg(odc + k);
                    if (apq != 0.0 && !(fabs(apq) <= kJTol * sqrt(fabs(app) * fabs(aqq)))) {
                        const double tau = (aqq - app) / (2.0 * apq);
                        const double sg = tau >= 0.0 ? 1.0 : -1.0;
                        tt = fabs(tau) > 1e150 ? 0.5 / tau : sg / (fabs(tau) + sqrt(1.0 + tau * tau));
                        c = 1.0 / sqrt(1.0 + tt * tt);
                        s = tt * c;
                        const double den = sqrt(fabs(app) * fabs(aqq));
                        worst = fmax(worst, den > 0.0 ? fabs(apq) / den : INFINITY);
                    }
                }
                cs[k] = c;
                sn[k] = s;
                tv[k] = tt;
                P[k] = p;
                Q[k] = q;
            }
            for (int x = threadIdx.x; x < np; x += blockDim.x) nq[x] = -1;
            __syncthreads();
            for (int k = threadIdx.x; k < H; k += blockDim.x) {
                const int p = circle_index(k, tn, np);
                nq[p] = circle_index(np - 1 - k, tn, np);
                nk[p] = k;
            }
            __syncthreads();
            // copy an element the next round pivots on
            auto note = [&](int x, int y, double v) {
                if (x == y) dgn[x] = v;
                else if (nq[x] == y) odn[nk[x]] = v;
            };
            for (int e = gt; e < nblocks; e += gs) {
                const int i = e / H, j = e - (e / H) * H;
                const double ci = cs[i], si = sn[i], cj = cs[j], sj = sn[j];
                const int pi = P[i], qi = Q[i], pj = P[j], qj = Q[j];
                const bool vp = pi < n, vq = qi < n, wp = pj < n, wq = qj < n;
                if (si == 0.0 && sj == 0.0) {          // unchanged: copy what the next round pivots on
                    if (vp && wp && (pi == pj || nq[pi] == pj)) note(pi, pj, __ldcg(A + pi * lda + pj));
                    if (vp && wq && (pi == qj || nq[pi] == qj)) note(pi, qj, __ldcg(A + pi * lda + qj));
                    if (vq && wp && (qi == pj || nq[qi] == pj)) note(qi, pj, __ldcg(A + qi * lda + pj));
                    if (vq && wq && (qi == qj || nq[qi] == qj)) note(qi, qj, __ldcg(A + qi * lda + qj));
                    continue;
                }
                if (i == j) {
                    // diagonal block: the closed form keeps the off-diagonal exactly zero
                    const double t = tv[i], apq = __ldcg(odc + i);
                    const double npp = __ldcg(dgc + pi) - t * apq, nqq = __ldcg(dgc + qi) + t * apq;
                    A[pi * lda + pi] = npp;
                    A[qi * lda + qi] = nqq;
                    A[pi * lda + qi] = 0.0;
                    A[qi * lda + pi] = 0.0;
                    note(pi, pi, npp);
                    note(qi, qi, nqq);
                    note(pi, qi, 0.0);
                    note(qi, pi, 0.0);
                    continue;
                }
                const double b00 = vp && wp ? __ldcg(A + pi * lda + pj) : 0.0;
                const double b01 = vp && wq ? __ldcg(A + pi * lda + qj) : 0.0;
                const double b10 = vq && wp ? __ldcg(A + qi * lda + pj) : 0.0;
                const double b11 = vq && wq ? __ldcg(A + qi * lda + qj) : 0.0;
                const double r00 = ci * b00 - si * b10, r01 = ci * b01 - si * b11;
                const double r10 = si * b00 + ci * b10, r11 = si * b01 + ci * b11;
                const double n00 = cj * r00 - sj * r01, n01 = sj * r00 + cj * r01;
                const double n10 = cj * r10 - sj * r11, n11 = sj * r10 + cj * r11;
                if (vp && wp) { A[pi * lda + pj] = n00; note(pi, pj, n00); }
                if (vp && wq) { A[pi * lda + qj] = n01; note(pi, qj, n01); }
                if (vq && wp) { A[qi * lda + pj] = n10; note(qi, pj, n10); }
                if (vq && wq) { A[qi * lda + qj] = n11; note(qi, qj, n11); }
            }
            for (int f = gt; f < nvt; f += gs) {
                const int i = f / n, col = f - (f / n) * n;
                const double ci = cs[i], si = sn[i];
                if (si == 0.0) continue;
                double *rp = Vt + P[i] * ldv + col, *rq = Vt + Q[i] * ldv + col;
                const double vpv = __ldcg(rp), vqv = __ldcg(rq);
                *rp = ci * vpv - si * vqv;
                *rq = si * vpv + ci * vqv;
            }
            if (!grid_barrier(bar, gen, err)) return;
            b ^= 1;
        }
        // every CTA saw the same rotations, so all CTAs take the same decision.  Convergence is quadratic: once
        // every rotation of a sweep was below kJStop, what is left off the diagonal is of order kJStop^2
        if (!__syncthreads_or(worst > kJStop)) break;
    }
}

int sm_count_j()
{
    int n = 0;
    if (sm_count_of_current(&n) != cudaSuccess || n <= 0) n = 148;
    return n;
}

}  // namespace

cudaError_t jacobi_eig(double *A, int n, long lda, double *Vt, long ldv, double *side, unsigned *bar, int *err,
                       int max_sweeps, cudaStream_t s)
{
    if (n < 1 || n > kJacobiMaxN) return cudaErrorInvalidValue;
    const int np = n + (n & 1), H = np / 2;
    const size_t smem = (size_t)H * (3 * sizeof(double) + 2 * sizeof(int)) + (size_t)2 * np * sizeof(int);
    cudaError_t e = ensure_dyn_smem((const void *)jacobi_kernel,
                                    (size_t)(kJacobiMaxN / 2) * (3 * sizeof(double) + 2 * sizeof(int)) +
                                        (size_t)2 * kJacobiMaxN * sizeof(int));
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, jacobi_kernel, kJThreads, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    const long items = std::max((long)H * H, (long)H * n);
    const int grid = (int)std::max<long>(1, std::min<long>((long)sm_count_j(), (items + kJThreads - 1) / kJThreads));
    e = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    void *args[] = {&A, &n, &lda, &Vt, &ldv, &side, &bar, &err, &max_sweeps};
    return cudaLaunchCooperativeKernel((const void *)jacobi_kernel, dim3(grid), dim3(kJThreads), args, smem, s);
}

}  // namespace lb

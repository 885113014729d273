// Binary64 GEMM on the CUDA cores for the initialisation path.
//
// B200 issues 64 FP64 FMAs per clock per SM, on the CUDA cores as on its
// FP64 matrix path (tcgen05 has no binary64 kind), so a register-blocked SIMT
// kernel is the binary64 contraction here.  CTA tile 128 x 64, k-step 16,
// 256 threads with an 8 x 4 block of C each; operands staged through
// registers into double-buffered shared memory (one __syncthreads per
// k-step), fragments double-buffered in registers.  A warp is 4 rows x 8
// columns of threads, so every LDS.128 of an operand is one shared-memory
// wavefront, and the staging stores are conflict-free.  Small output grids
// split k over CTAs (the split that fills whole waves) and add the partial
// sums in a fixed order.
#include "lb_linalg.cuh"

#include <algorithm>
#include <math.h>

namespace lb {
namespace {

constexpr int BM = 128, BN = 64, BK = 16, kThreads = 256;

template <bool TA, bool TB>
__global__ void __launch_bounds__(kThreads, 1)
    dgemm_kernel(int m, int n, int k, int kchunk, double alpha, const double *A, long lda, const double *B,
                 long ldb, double beta, double *C, long ldc, double *part, int vec)
{
    __shared__ __align__(16) double As[2][BK][BM];
    __shared__ __align__(16) double Bs[2][BK][BN];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ty = (warp >> 1) * 4 + (lane >> 3);    // 0..15: rows ty*4 + {0..3} and 64 + ty*4 + {0..3}
    const int tx = (warp & 1) * 8 + (lane & 7);      // 0..15: cols tx*2 + {0, 1} and 32 + tx*2 + {0, 1}
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int kbeg = blockIdx.z * kchunk, kend = min(k, kbeg + kchunk);

    double ra[8], rb[4];
    // global -> registers for the k-step starting at k0 (zeros outside the matrix)
    auto load = [&](int k0) {
        if (!TA) {                                   // A is m x k: a thread takes 8 consecutive k of one row
            const int row = tid & (BM - 1), ks = (tid >> 7) * 8, gi = m0 + row, gk = k0 + ks;
            if (gi < m && vec && gk + 8 <= kend) {
                const double2 *src = reinterpret_cast<const double2 *>(A + (long)gi * lda + gk);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const double2 v = src[e];
                    ra[2 * e] = v.x;
                    ra[2 * e + 1] = v.y;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) ra[e] = (gi < m && gk + e < kend) ? A[(long)gi * lda + gk + e] : 0.0;
            }
        } else {                                     // A is k x m: rows 2t, 2t+1 (+32e) of one k
            const int kk = tid >> 4, mo = 2 * (tid & 15), gk = k0 + kk;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int gi = m0 + mo + 32 * e;
                if (gk < kend && vec && gi + 2 <= m) {
                    const double2 v = *reinterpret_cast<const double2 *>(A + (long)gk * lda + gi);
                    ra[2 * e] = v.x;
                    ra[2 * e + 1] = v.y;
                } else {
                    ra[2 * e] = (gk < kend && gi < m) ? A[(long)gk * lda + gi] : 0.0;
                    ra[2 * e + 1] = (gk < kend && gi + 1 < m) ? A[(long)gk * lda + gi + 1] : 0.0;
                }
            }
        }
        if (!TB) {                                   // B is k x n: columns 2t, 2t+1 (+32e) of one k
            const int kk = tid >> 4, no = 2 * (tid & 15), gk = k0 + kk;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int gj = n0 + no + 32 * e;
                if (gk < kend && vec && gj + 2 <= n) {
                    const double2 v = *reinterpret_cast<const double2 *>(B + (long)gk * ldb + gj);
                    rb[2 * e] = v.x;
                    rb[2 * e + 1] = v.y;
                } else {
                    rb[2 * e] = (gk < kend && gj < n) ? B[(long)gk * ldb + gj] : 0.0;
                    rb[2 * e + 1] = (gk < kend && gj + 1 < n) ? B[(long)gk * ldb + gj + 1] : 0.0;
                }
            }
        } else {                                     // B is n x k: 4 consecutive k of one column
            const int col = tid & (BN - 1), ks = (tid >> 6) * 4, gj = n0 + col, gk = k0 + ks;
            if (gj < n && vec && gk + 4 <= kend) {
                const double2 *src = reinterpret_cast<const double2 *>(B + (long)gj * ldb + gk);
                const double2 v0 = src[0], v1 = src[1];
                rb[0] = v0.x; rb[1] = v0.y; rb[2] = v1.x; rb[3] = v1.y;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) rb[e] = (gj < n && gk + e < kend) ? B[(long)gj * ldb + gk + e] : 0.0;
            }
        }
    };
    // registers -> shared stage `b` (both operands k-major: As[k][m], Bs[k][n])
    auto store = [&](int b) {
        if (!TA) {
            const int row = tid & (BM - 1), ks = (tid >> 7) * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) As[b][ks + e][row] = ra[e];
        } else {
            const int kk = tid >> 4, mo = 2 * (tid & 15);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                *reinterpret_cast<double2 *>(&As[b][kk][mo + 32 * e]) = make_double2(ra[2 * e], ra[2 * e + 1]);
        }
        if (!TB) {
            const int kk = tid >> 4, no = 2 * (tid & 15);
#pragma unroll
            for (int e = 0; e < 2; ++e)
                *reinterpret_cast<double2 *>(&Bs[b][kk][no + 32 * e]) = make_double2(rb[2 * e], rb[2 * e + 1]);
        } else {
            const int col = tid & (BN - 1), ks = (tid >> 6) * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e) Bs[b][ks + e][col] = rb[e];
        }
    };

    double acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;

    const int nsteps = (kend - kbeg + BK - 1) / BK;
    if (nsteps > 0) {
        load(kbeg);
        store(0);
        __syncthreads();
    }
    for (int st = 0; st < nsteps; ++st) {
        const int b = st & 1;
        if (st + 1 < nsteps) load(kbeg + (st + 1) * BK);
        // operand fragments of step kk + 1 are read while step kk's FMAs issue
        double2 fa[2][4], fb[2][2];
        auto frag = [&](int s, int kk) {
            fa[s][0] = *reinterpret_cast<const double2 *>(&As[b][kk][ty * 4]);
            fa[s][1] = *reinterpret_cast<const double2 *>(&As[b][kk][ty * 4 + 2]);
            fa[s][2] = *reinterpret_cast<const double2 *>(&As[b][kk][64 + ty * 4]);
            fa[s][3] = *reinterpret_cast<const double2 *>(&As[b][kk][64 + ty * 4 + 2]);
            fb[s][0] = *reinterpret_cast<const double2 *>(&Bs[b][kk][tx * 2]);
            fb[s][1] = *reinterpret_cast<const double2 *>(&Bs[b][kk][32 + tx * 2]);
        };
        frag(0, 0);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const int s = kk & 1;
            if (kk + 1 < BK) frag(s ^ 1, kk + 1);
            const double av[8] = {fa[s][0].x, fa[s][0].y, fa[s][1].x, fa[s][1].y,
                                  fa[s][2].x, fa[s][2].y, fa[s][3].x, fa[s][3].y};
            const double bv[4] = {fb[s][0].x, fb[s][0].y, fb[s][1].x, fb[s][1].y};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
        }
        if (st + 1 < nsteps) store(b ^ 1);
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int gi = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
        if (gi >= m) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gj = n0 + (j < 2 ? tx * 2 + j : 32 + tx * 2 + j - 2);
            if (gj >= n) continue;
            if (part) {
                part[((long)blockIdx.z * m + gi) * n + gj] = acc[i][j];
            } else {
                double *c = C + (long)gi * ldc + gj;
                *c = beta == 0.0 ? alpha * acc[i][j] : fma(alpha, acc[i][j], beta * *c);
            }
        }
    }
}

// C = alpha * sum_z part[z] + beta * C, the slices added in order
__global__ void dgemm_reduce_kernel(int m, int n, int S, double alpha, const double *__restrict__ part, double beta,
                                    double *C, long ldc)
{
    const long total = (long)m * n;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        double acc = 0.0;
        for (int z = 0; z < S; ++z) acc += part[(long)z * total + e];
        double *c = C + (e / n) * ldc + e % n;
        *c = beta == 0.0 ? alpha * acc : fma(alpha, acc, beta * *c);
    }
}

__global__ void dscale_kernel(int m, int n, double beta, double *C, long ldc)
{
    const long total = (long)m * n;
    for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total; e += (long)gridDim.x * blockDim.x) {
        double *c = C + (e / n) * ldc + e % n;
        *c = beta == 0.0 ? 0.0 : beta * *c;
    }
}

int sm_count()
{
    int n = 0;
    if (sm_count_of_current(&n) != cudaSuccess || n <= 0) n = 148;
    return n;
}

}  // namespace

void dgemm(bool ta, bool tb, int m, int n, int k, double alpha, const double *A, long lda, const double *B,
           long ldb, double beta, double *C, long ldc, double *part, size_t part_elems, cudaStream_t s)
{
    if (m <= 0 || n <= 0) return;
    const int sms = sm_count();
    if (k <= 0) {
        const long total = (long)m * n;
        dscale_kernel<<<(int)std::min<long>((total + 255) / 256, 4L * sms), 256, 0, s>>>(m, n, beta, C, ldc);
        return;
    }
    const long tiles = (long)((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    // split k so that the grid fills whole waves of one CTA per SM (and at most 16 slices of >= 256)
    int S = 1;
    if (part && tiles < 4L * sms) {
        double best = -1.0;
        const int smax = (int)std::min<long>(16, std::max(1, k / 256));
        for (int c = 1; c <= smax; ++c) {
            if ((size_t)c * m * n > part_elems) break;
            const long ctas = tiles * c;
            const double waves = (double)ctas / sms;
            const double eff = waves / std::ceil(waves);     // busy fraction of the SMs over the launch
            if (eff > best + 0.02) {
                best = eff;
                S = c;
            }
        }
    }
    int kchunk = ((k + S - 1) / S + BK - 1) / BK * BK;
    S = (k + kchunk - 1) / kchunk;
    const int vec = !(((uintptr_t)A | (uintptr_t)B) & 15) && !(lda & 1) && !(ldb & 1);
    const dim3 grid((n + BN - 1) / BN, (m + BM - 1) / BM, S);
    double *pp = S > 1 ? part : nullptr;
    if (!ta && !tb) dgemm_kernel<false, false><<<grid, kThreads, 0, s>>>(m, n, k, kchunk, alpha, A, lda, B, ldb, beta, C, ldc, pp, vec);
    else if (ta && !tb) dgemm_kernel<true, false><<<grid, kThreads, 0, s>>>(m, n, k, kchunk, alpha, A, lda, B, ldb, beta, C, ldc, pp, vec);
    else if (!ta && tb) dgemm_kernel<false, true><<<grid, kThreads, 0, s>>>(m, n, k, kchunk, alpha, A, lda, B, ldb, beta, C, ldc, pp, vec);
    else dgemm_kernel<true, true><<<grid, kThreads, 0, s>>>(m, n, k, kchunk, alpha, A, lda, B, ldb, beta, C, ldc, pp, vec);
    if (S > 1) {
        const long total = (long)m * n;
        dgemm_reduce_kernel<<<(int)std::min<long>((total + 255) / 256, 4L * sms), 256, 0, s>>>(m, n, S, alpha, part,
                                                                                                beta, C, ldc);
    }
}

}  // namespace lb

// Backward pass of a LittleBit layer for quantisation-aware training
// (LittleBit paper notes page, "Multi-scale compensation" and "Loss /
// training strategy": SmoothSign, forward sign and backward tanh(100 u)).
//
// Per path, with ds = dy (.) h:
//   dzl = ds U_s            = latent contraction of the transposed layer (U <-> V, h <-> g) applied to dy
//   dx  = sum_p g (.) (dz V_s^T), dz = dzl (.) l
//                           = output contraction of the transposed layer applied to dz
//   z   = (x (.) g) V_s     = latent contraction of the forward layer with l = 1
//   dl  = sum_m dzl (.) z,  zl = z (.) l
//   G_U = dy^T zl, dh = sum_j U_s (.) G_U, dU = h (.) G_U (.) 100 (1 - tanh^2(100 U))
//   G_V = x^T dz,  dg = sum_j V_s (.) G_V, dV = g (.) G_V (.) 100 (1 - tanh^2(100 V))
// The contractions run on the tcgen05 kernels of the forward pass (two helper
// layers with l = 1): z and dzl, which are independent, in one launch whose
// output tiles are split over k into units of even length (their fp32 partial
// sums are added in place), dx on the output kernel.  G_U and G_V are plain
// fp16 GEMMs on the library's tcgen05 kernel (lb_gemm.cu), both operands read
// MN-major as stored.  dy is
// multiplied by one power of two 2^E, chosen on the device so that dy 2^E and
// dzl 2^E (and dz 2^E) stay below 2^14, and divided out exactly at the end.
#include "littlebit_backward.h"
#include "lb_internal.cuh"
#include "lb_prefill.cuh"

#include <cuda_fp16.h>
#include <algorithm>
#include <math.h>
#include <new>

struct lb_backward {
    int N = 0, K = 0, r = 0, npaths = 0, r8 = 0, K2 = 0;
    lb_layer *Lf = nullptr;        // forward layer with l = 1: its latent contraction gives z
    lb_layer *Lt = nullptr;        // transposed layer with l = 1: latent gives dzl, output gives dx from dz
    float *lcat = nullptr;         // [K2] l per latent column j' = p*r8 + j (0 on padding)
    float *h32 = nullptr;          // [npaths][N]
    float *g32 = nullptr;          // [npaths][K]
    float *hmax = nullptr;         // [N] max_p |h_p|
    uint32_t *Uw = nullptr;        // [npaths][N][wpr] canonical packed signs
    uint32_t *Vw = nullptr;        // [npaths][K][wpr]
    float *dl_acc = nullptr;       // [K2]
    float *stat = nullptr;         // [0] bound (float bits, atomic max), [1] 2^E, [2] 2^-E, [3] max l, [4] 0
    int M = 0;                     // rows the scratch below holds
    __half *dy16 = nullptr;        // [M][N]
    __half *x16 = nullptr;         // [M][K]
    float *zpart = nullptr;        // [M][K2] z from the k-split latent contraction (fp32)
    float *dzpart = nullptr;       // [M][K2] dzl 2^E, likewise
    lb::PfJobState *jobs = nullptr;   // the one-launch latent contractions (tensor maps, unit records)
    float *GU = nullptr;           // [N][K2]
    float *GV = nullptr;           // [K][K2]
    int *gerr = nullptr;           // error slot of the G_U / G_V GEMM kernel (bounded waits)
    cudaStream_t side = nullptr;   // G_U, G_V and the factor gradients run here, beside dx
    cudaEvent_t fork = nullptr, join = nullptr;
};

namespace lb {
namespace {

constexpr int kT = 256;

int grid_for(long n) { return (int)std::max<long>(1, std::min<long>((n + kT - 1) / kT, 148L * 16)); }

__global__ void half_ones_kernel(uint16_t *o, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) o[i] = 0x3C00;
}

// float32 copies of binary16 scales; l laid out per latent column; max_p |h_p| per row
__global__ void scales_kernel(const uint16_t *h0, const uint16_t *h1, const uint16_t *g0, const uint16_t *g1,
                              const uint16_t *l0, const uint16_t *l1, int npaths, int N, int K, int r, int r8,
                              int K2, float *h32, float *g32, float *hmax, float *lcat, float *stat)
{
    const int n = max(max(N, K), K2);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        if (i < N) {
            const float a = __half2float(__ushort_as_half(h0[i]));
            const float b = npaths > 1 ? __half2float(__ushort_as_half(h1[i])) : 0.0f;
            h32[i] = a;
            if (npaths > 1) h32[N + i] = b;
            hmax[i] = fmaxf(fabsf(a), fabsf(b));
        }
        if (i < K) {
            g32[i] = __half2float(__ushort_as_half(g0[i]));
            if (npaths > 1) g32[K + i] = __half2float(__ushort_as_half(g1[i]));
        }
        if (i < K2) {
            const int p = i / r8, j = i - p * r8;
            float v = 0.0f;
            if (p < npaths && j < r) v = __half2float(__ushort_as_half(p ? l1[j] : l0[j]));
            lcat[i] = v;
            if (v != 0.0f) atomicMax(reinterpret_cast<int *>(stat + 3), __float_as_int(fabsf(v)));
        }
    }
}

// bound = max over rows of max(max_n |dy|, sum_n |dy| hmax[n]) (atomic max on the float's bits: non-negative);
// one CTA per row, float4 loads (N is a multiple of 8)
__global__ void __launch_bounds__(kT) dy_bound_kernel(const float *__restrict__ dy, int M, int N,
                                                      const float *__restrict__ hmax, float *stat)
{
    __shared__ float smx[kT / 32], sl1[kT / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n4 = N / 4;
    const float4 *hm = reinterpret_cast<const float4 *>(hmax);
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const float4 *row = reinterpret_cast<const float4 *>(dy + (size_t)m * N);
        float mx = 0.0f, l1 = 0.0f;
#pragma unroll 4
        for (int q = threadIdx.x; q < n4; q += kT) {
            const float4 a = __ldg(row + q), h = __ldg(hm + q);
            mx = fmaxf(fmaxf(fmaxf(mx, fabsf(a.x)), fmaxf(fabsf(a.y), fabsf(a.z))), fabsf(a.w));
            l1 += fabsf(a.x) * h.x + fabsf(a.y) * h.y + fabsf(a.z) * h.z + fabsf(a.w) * h.w;
        }
        for (int o = 16; o; o >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
        if (lane == 0) {
            smx[warp] = mx;
            sl1[warp] = l1;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 1; w < kT / 32; ++w) {
                mx = fmaxf(mx, smx[w]);
                l1 += sl1[w];
            }
            atomicMax(reinterpret_cast<int *>(stat), __float_as_int(fmaxf(mx, l1)));
        }
        __syncthreads();
    }
}

// 2^E with bound * max(1, max l) * 2^E < 2^14 (E = 0 for a zero or non-finite bound)
__global__ void exponent_kernel(float *stat)
{
    const float b = stat[0] * fmaxf(1.0f, stat[3]);
    int e = 0;
    if (b > 0.0f && isfinite(b)) {
        frexpf(b, &e);                  // b < 2^e
        e = 14 - e;
        e = max(-120, min(120, e));
    } else {
        e = 0;
    }
    stat[1] = ldexpf(1.0f, e);
    stat[2] = ldexpf(1.0f, -e);
}

// dy16 = fp16(dy 2^E), x16 = fp16(x); four elements per thread (N and K are multiples of 8)
__global__ void convert_kernel(const float *__restrict__ dy, long ndy, const uint16_t *__restrict__ x, long nx,
                               const float *__restrict__ stat, __half *dy16, __half *x16)
{
    const float sc = stat[1];
    const long n = max(ndy, nx) / 4;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        if (4 * i < ndy) {
            const float4 a = reinterpret_cast<const float4 *>(dy)[i];
            __half2 *o = reinterpret_cast<__half2 *>(dy16) + 2 * i;
            o[0] = __floats2half2_rn(a.x * sc, a.y * sc);
            o[1] = __floats2half2_rn(a.z * sc, a.w * sc);
        }
        if (4 * i < nx) {
            const uint2 b = reinterpret_cast<const uint2 *>(x)[i];
            __half2 *o = reinterpret_cast<__half2 *>(x16) + 2 * i;
            o[0] = __floats2half2_rn(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u));
            o[1] = __floats2half2_rn(__uint_as_float(b.y << 16), __uint_as_float(b.y & 0xFFFF0000u));
        }
    }
}

// dl_acc[j'] += sum_m dzl[m][j'] z[m][j'] over this CTA's rows; dz = fp16(dzl l), zl = fp16(z l).  dzl and z are
// the fp32 sums of the k-split latent contraction.  Four columns per thread (ncols and ld are multiples of 4), a
// slice of rows per CTA (blockIdx.y).
__global__ void latent_mix_kernel(const float *__restrict__ dzl, const float *__restrict__ z, int M, int ncols, int ld,
                                  const float *__restrict__ lcat, float *dl_acc, __half *dz, __half *zl, int rows_per)
{
    const int j = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (j >= ncols) return;
    const int m0 = blockIdx.y * rows_per, m1 = min(M, m0 + rows_per);
    const float4 l = *reinterpret_cast<const float4 *>(lcat + j);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int m = m0; m < m1; ++m) {
        const size_t o = (size_t)m * ld + j;
        const float4 a = __ldg(reinterpret_cast<const float4 *>(dzl + o));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(z + o));
        acc.x = fmaf(a.x, b.x, acc.x);
        acc.y = fmaf(a.y, b.y, acc.y);
        acc.z = fmaf(a.z, b.z, acc.z);
        acc.w = fmaf(a.w, b.w, acc.w);
        __half2 *pd = reinterpret_cast<__half2 *>(dz + o), *pz = reinterpret_cast<__half2 *>(zl + o);
        pd[0] = __floats2half2_rn(a.x * l.x, a.y * l.y);
        pd[1] = __floats2half2_rn(a.z * l.z, a.w * l.w);
        pz[0] = __floats2half2_rn(b.x * l.x, b.y * l.y);
        pz[1] = __floats2half2_rn(b.z * l.z, b.w * l.w);
    }
    atomicAdd(dl_acc + j, acc.x);
    atomicAdd(dl_acc + j + 1, acc.y);
    atomicAdd(dl_acc + j + 2, acc.z);
    atomicAdd(dl_acc + j + 3, acc.w);
}

__global__ void dl_out_kernel(const float *__restrict__ dl_acc, int r, int r8, const float *__restrict__ stat,
                              float *dl0, float *dl1)
{
    const float sc = stat[2];
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < r; j += gridDim.x * blockDim.x) {
        dl0[j] = dl_acc[j] * sc;
        if (dl1) dl1[j] = dl_acc[r8 + j] * sc;
    }
}

// factor gradients of all paths: one warp per row i of G (rows x K2; path p's columns at p r8 .. p r8 + r):
// dF_p[i][j] = s_p[i] G[i][p r8 + j] 100 (1 - tanh^2(100 F_p[i][j])),  dsc_p[i] = sum_j sign_pij G[i][p r8 + j].
// 100 (1 - tanh^2(a)) is evaluated as 400 e^{-2|a|} / (1 + e^{-2|a|})^2 (no cancellation for large |a|).
struct FactorArgs {
    const float *s[2];
    const uint32_t *words[2];
    const float *F[2];
    float *dF[2];
    float *dsc[2];
};

// 100 (1 - tanh^2(100 f))
__device__ __forceinline__ float smooth_sign_grad(float f)
{
    const float ea = __expf(-200.0f * fabsf(f));
    const float d1 = 1.0f + ea;
    return 400.0f * ea / (d1 * d1);
}

// as factor_grad_kernel, four latent columns per lane (r a multiple of 4: rows of F, dF and G 16-byte aligned)
template <int P>
__global__ void __launch_bounds__(kT) factor_grad4_kernel(const float *__restrict__ G, int rows, int K2, int r, int r8,
                                                          const FactorArgs a)
{
    const int lane = threadIdx.x & 31, wpr = (r + 31) / 32, r4 = r / 4;
    for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < rows; i += (gridDim.x * blockDim.x) >> 5) {
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const float si = a.s[p][i];
            const float4 *__restrict__ g = reinterpret_cast<const float4 *>(G + (size_t)i * K2 + p * r8);
            const uint32_t *__restrict__ w = a.words[p] + (size_t)i * wpr;
            const float4 *__restrict__ f = reinterpret_cast<const float4 *>(a.F[p] + (size_t)i * r);
            float4 *__restrict__ df = reinterpret_cast<float4 *>(a.dF[p] + (size_t)i * r);
            float acc = 0.0f;
#pragma unroll 2
            for (int q = lane; q < r4; q += 32) {
                const float4 gv = __ldg(g + q), fv = __ldg(f + q);
                const uint32_t bits = __ldg(w + (q >> 3)) >> ((4 * q) & 31);
                acc += (bits & 1u ? -gv.x : gv.x) + (bits & 2u ? -gv.y : gv.y) + (bits & 4u ? -gv.z : gv.z) +
                       (bits & 8u ? -gv.w : gv.w);
                float4 o;
                o.x = si * gv.x * smooth_sign_grad(fv.x);
                o.y = si * gv.y * smooth_sign_grad(fv.y);
                o.z = si * gv.z * smooth_sign_grad(fv.z);
                o.w = si * gv.w * smooth_sign_grad(fv.w);
                __stcs(df + q, o);
            }
            for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) a.dsc[p][i] = acc;
        }
    }
}

template <int P>
__global__ void __launch_bounds__(kT) factor_grad_kernel(const float *__restrict__ G, int rows, int K2, int r, int r8,
                                                         const FactorArgs a)
{
    const int lane = threadIdx.x & 31, wpr = (r + 31) / 32;
    for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < rows; i += (gridDim.x * blockDim.x) >> 5) {
#pragma unroll
        for (int p = 0; p < P; ++p) {
            const float si = a.s[p][i];
            const float *__restrict__ g = G + (size_t)i * K2 + p * r8;
            const uint32_t *__restrict__ w = a.words[p] + (size_t)i * wpr;
            const float *__restrict__ f = a.F[p] + (size_t)i * r;
            float *__restrict__ df = a.dF[p] + (size_t)i * r;
            float acc = 0.0f;
#pragma unroll 4
            for (int j = lane; j < r; j += 32) {
                const float gv = __ldg(g + j);
                acc += ((__ldg(w + (j >> 5)) >> (j & 31)) & 1u) ? -gv : gv;
                const float ea = __expf(-200.0f * fabsf(__ldg(f + j)));
                const float d1 = 1.0f + ea;
                df[j] = si * gv * (400.0f * ea / (d1 * d1));
            }
            for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) a.dsc[p][i] = acc;
        }
    }
}

lb_status grow(lb_backward *B, int M, cudaStream_t s)
{
    if (M <= B->M) return LB_OK;
    if (B->M) cudaStreamSynchronize(s);
    cudaFree(B->dy16);
    cudaFree(B->x16);
    cudaFree(B->zpart);
    cudaFree(B->dzpart);
    B->dy16 = nullptr;
    B->x16 = nullptr;
    B->zpart = B->dzpart = nullptr;
    B->M = 0;
    if (cudaMalloc(&B->dy16, (size_t)M * B->N * sizeof(__half)) != cudaSuccess ||
        cudaMalloc(&B->x16, (size_t)M * B->K * sizeof(__half)) != cudaSuccess ||
        cudaMalloc(&B->zpart, (size_t)M * B->K2 * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&B->dzpart, (size_t)M * B->K2 * sizeof(float)) != cudaSuccess)
        return LB_ERR_OOM;
    B->M = M;
    return LB_OK;
}

}  // namespace
}  // namespace lb

using namespace lb;

extern "C" {

void lb_backward_destroy(lb_backward *B)
{
    if (!B) return;
    lb_layer_destroy(B->Lf);
    lb_layer_destroy(B->Lt);
    prefill_jobs_free(B->jobs);
    for (void *p : {(void *)B->lcat, (void *)B->h32, (void *)B->g32, (void *)B->hmax, (void *)B->Uw, (void *)B->Vw,
                    (void *)B->dl_acc, (void *)B->stat, (void *)B->dy16, (void *)B->x16, (void *)B->zpart,
                    (void *)B->dzpart, (void *)B->GU, (void *)B->GV, (void *)B->gerr})
        cudaFree(p);
    if (B->fork) cudaEventDestroy(B->fork);
    if (B->join) cudaEventDestroy(B->join);
    if (B->side) cudaStreamDestroy(B->side);
    delete B;
}

lb_status lb_backward_create(lb_backward **out, int N, int K, int r, int npaths, const uint32_t *const *U,
                             const uint32_t *const *V, const uint16_t *const *h, const uint16_t *const *g,
                             const uint16_t *const *l, void *stream)
{
    if (!out) return LB_ERR_INVALID_ARG;
    *out = nullptr;
    if (N < 1 || K < 1 || r < 1 || r > LB_MAX_RANK) return LB_ERR_INVALID_ARG;
    if (npaths != 1 && npaths != 2) return LB_ERR_UNSUPPORTED;
    if (!U || !V || !h || !g || !l) return LB_ERR_INVALID_ARG;
    for (int p = 0; p < npaths; ++p)
        if (!U[p] || !V[p] || !h[p] || !g[p] || !l[p]) return LB_ERR_INVALID_ARG;
    if (N % 8 || K % 8) return LB_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    lb_backward *B = new (std::nothrow) lb_backward();
    if (!B) return LB_ERR_OOM;
    B->N = N;
    B->K = K;
    B->r = r;
    B->npaths = npaths;
    B->r8 = (r + 7) / 8 * 8;
    const int N1p = (npaths * B->r8 + 15) / 16 * 16;
    B->K2 = (N1p + 63) / 64 * 64;
    const int wpr = (r + 31) / 32;
    lb_status st = LB_OK;
    uint16_t *ones = nullptr;
    auto fail = [&](lb_status e) {
        cudaFree(ones);
        lb_backward_destroy(B);
        return e;
    };
    if (cudaMalloc(&ones, (size_t)r * sizeof(uint16_t)) != cudaSuccess) return fail(LB_ERR_OOM);
    half_ones_kernel<<<grid_for(r), kT, 0, s>>>(ones, r);
    const uint16_t *ones2[2] = {ones, ones};
    const uint32_t *Ut[2] = {V[0], npaths > 1 ? V[1] : V[0]};
    const uint32_t *Vt[2] = {U[0], npaths > 1 ? U[1] : U[0]};
    if ((st = lb_layer_create(&B->Lf, N, K, r, npaths, U, V, h, g, ones2, stream)) != LB_OK) return fail(st);
    if ((st = lb_layer_create(&B->Lt, K, N, r, npaths, Ut, Vt, g, h, ones2, stream)) != LB_OK) return fail(st);
    auto alloc = [&](void **p, size_t bytes) { return cudaMalloc(p, bytes) == cudaSuccess; };
    if (!alloc((void **)&B->lcat, (size_t)B->K2 * 4) || !alloc((void **)&B->h32, (size_t)npaths * N * 4) ||
        !alloc((void **)&B->g32, (size_t)npaths * K * 4) || !alloc((void **)&B->hmax, (size_t)N * 4) ||
        !alloc((void **)&B->Uw, (size_t)npaths * N * wpr * 4) || !alloc((void **)&B->Vw, (size_t)npaths * K * wpr * 4) ||
        !alloc((void **)&B->dl_acc, (size_t)B->K2 * 4) || !alloc((void **)&B->stat, 8 * 4) ||
        !alloc((void **)&B->GU, (size_t)N * B->K2 * 4) || !alloc((void **)&B->GV, (size_t)K * B->K2 * 4))
        return fail(LB_ERR_OOM);
    cudaMemsetAsync(B->stat, 0, 8 * 4, s);
    scales_kernel<<<grid_for(std::max(std::max(N, K), B->K2)), kT, 0, s>>>(
        h[0], npaths > 1 ? h[1] : h[0], g[0], npaths > 1 ? g[1] : g[0], l[0], npaths > 1 ? l[1] : l[0], npaths, N, K, r,
        B->r8, B->K2, B->h32, B->g32, B->hmax, B->lcat, B->stat);
    for (int p = 0; p < npaths; ++p) {
        cudaMemcpyAsync(B->Uw + (size_t)p * N * wpr, U[p], (size_t)N * wpr * 4, cudaMemcpyDeviceToDevice, s);
        cudaMemcpyAsync(B->Vw + (size_t)p * K * wpr, V[p], (size_t)K * wpr * 4, cudaMemcpyDeviceToDevice, s);
    }
    if (!alloc((void **)&B->gerr, sizeof(int))) return fail(LB_ERR_OOM);
    cudaMemsetAsync(B->gerr, 0, sizeof(int), s);
    if (cudaStreamCreateWithFlags(&B->side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&B->fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&B->join, cudaEventDisableTiming) != cudaSuccess)
        return fail(LB_ERR_CUDA);
    if (cudaStreamSynchronize(s) != cudaSuccess) return fail(LB_ERR_CUDA);
    cudaFree(ones);
    ones = nullptr;
    if (cudaGetLastError() != cudaSuccess) return fail(LB_ERR_CUDA);
    *out = B;
    return LB_OK;
}

lb_status lb_layer_backward(lb_backward *B, const uint16_t *x, const float *dy, int M, const float *const *U_lat,
                            const float *const *V_lat, float *dx, float *const *dh, float *const *dg,
                            float *const *dl, float *const *dU, float *const *dV, void *stream)
{
    set_launch_count(0);
    if (!B || M < 1 || !x || !dy || !dx || !U_lat || !V_lat || !dh || !dg || !dl || !dU || !dV)
        return LB_ERR_INVALID_ARG;
    if (((uintptr_t)x | (uintptr_t)dy | (uintptr_t)dx) & 15) return LB_ERR_INVALID_ARG;
    for (int p = 0; p < B->npaths; ++p)
        if (!U_lat[p] || !V_lat[p] || !dh[p] || !dg[p] || !dl[p] || !dU[p] || !dV[p]) return LB_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaGetLastError() != cudaSuccess) return LB_ERR_CUDA;
    lb_status st = grow(B, M, s);
    if (st != LB_OK) return st;
    const int N = B->N, K = B->K, r = B->r, K2 = B->K2;
    int launches = 0;

    // timing hook (littlebit.h): events 0 | scaling | 1 | z and dzl (one launch) | 2, 3 | dl, dz, zl | 4, then
    // dx | 5 on this stream and, from 4 on the side stream, G_U and G_V (one launch) | 6, 7 | factor gradients | 8
    profile_mark(0, s);
    // dy scale (device-side exponent), fp16 copies of dy 2^E and x
    cudaMemsetAsync(B->stat, 0, sizeof(float), s);
    cudaMemsetAsync(B->dl_acc, 0, (size_t)K2 * 4, s);
    dy_bound_kernel<<<std::min(M, 148 * 8), kT, 0, s>>>(dy, M, N, B->hmax, B->stat);
    exponent_kernel<<<1, 1, 0, s>>>(B->stat);
    convert_kernel<<<grid_for((long)M * std::max(N, K)), kT, 0, s>>>(dy, (long)M * N, x, (long)M * K, B->stat, B->dy16,
                                                                      B->x16);
    launches += 3;
    profile_mark(1, s);

    // z (forward latent, l = 1) and dzl 2^E (transposed latent, l = 1), both in one launch with k-split units
    // adding into zeroed fp32 buffers.  The two helpers' plans are set up first (no launch): they own the fp16
    // buffers of zl and dz and the maps of the dx contraction.  The y map of the forward helper is never used (its
    // output contraction is not run); dx only stands in for a well-aligned pointer there.
    const uint16_t *xs[1] = {x};
    const uint16_t *dys[1] = {reinterpret_cast<const uint16_t *>(B->dy16)};
    float *ys[1] = {dx};
    if ((st = prefill_forward(B->Lf->self->plan, &B->Lf, xs, ys, M, s, &launches, 0, false, false)) != LB_OK) return st;
    if ((st = prefill_forward(B->Lt->self->plan, &B->Lt, dys, ys, M, s, &launches, 0, true, false, B->stat + 2)) !=
        LB_OK)
        return st;
    __half *zf = prefill_zl(B->Lf->self->plan, 0), *dz = prefill_zl(B->Lt->self->plan, 0);
    if (!zf || !dz) return LB_ERR_CUDA;
    cudaMemsetAsync(B->zpart, 0, (size_t)M * K2 * sizeof(float), s);
    cudaMemsetAsync(B->dzpart, 0, (size_t)M * K2 * sizeof(float), s);
    const PfLatentJob jobs[2] = {{B->Lf, x, false, B->zpart, K2}, {B->Lt, B->dy16, true, B->dzpart, K2}};
    if ((st = prefill_latent_jobs(&B->jobs, jobs, 2, M, s, &launches)) != LB_OK) return st;
    profile_mark(2, s);
    profile_mark(3, s);

    // dl, dz = dzl l, zl = z l
    const int ncols = B->npaths * B->r8, rows_per = 16, mix_t = 128;
    latent_mix_kernel<<<dim3((ncols / 4 + mix_t - 1) / mix_t, (M + rows_per - 1) / rows_per), mix_t, 0, s>>>(
        B->dzpart, B->zpart, M, ncols, K2, B->lcat, B->dl_acc, dz, zf, rows_per);
    dl_out_kernel<<<grid_for(r), kT, 0, s>>>(B->dl_acc, r, B->r8, B->stat, dl[0], B->npaths > 1 ? dl[1] : nullptr);
    profile_mark(4, s);
    // from here two streams: dx here; G_U, G_V and the factor gradients on the side stream (they read dz, zl, dy16
    // and x16, which are complete), so the side work fills the SMs that the tail of the dx tiles leaves idle
    if (cudaEventRecord(B->fork, s) != cudaSuccess || cudaStreamWaitEvent(B->side, B->fork, 0) != cudaSuccess)
        return LB_ERR_CUDA;
    cudaStream_t s2 = B->side;
    // a failure from here on joins the side stream back into the caller's before returning
    auto joined = [&](lb_status e) {
        cudaEventRecord(B->join, s2);
        cudaStreamWaitEvent(s, B->join, 0);
        return e;
    };
    // dx = 2^-E sum_p g (.) (dz 2^E V_s^T): the output contraction's epilogue multiplies by 2^-E (stat[2])
    if ((st = prefill_forward(B->Lt->self->plan, &B->Lt, dys, ys, M, s, &launches, 2, true, false, B->stat + 2)) !=
        LB_OK)
        return joined(st);
    launches += 2;
    profile_mark(5, s);

    // G_U = 2^-E (dy 2^E)^T zl [N][K2], G_V = 2^-E x^T (dz 2^E) [K][K2]: contracted over the M batch rows
    // (one launch: G_V's tiles fill the last wave of G_U's)
    const float *alpha = B->stat + 2;
    const GemmDesc gd[2] = {{B->dy16, N, zf, K2, B->GU, K2, M, N, K2, alpha}, {B->x16, K, dz, K2, B->GV, K2, M, K, K2, alpha}};
    if ((st = gemm_at_b_batch(gd, 2, B->gerr, s2)) != LB_OK) return joined(st);
    profile_mark(6, s2);
    profile_mark(7, s2);
    launches += 1;
    const int wpr = (r + 31) / 32;
    FactorArgs fu{}, fv{};
    for (int p = 0; p < B->npaths; ++p) {
        fu.s[p] = B->h32 + (size_t)p * N;
        fu.words[p] = B->Uw + (size_t)p * N * wpr;
        fu.F[p] = U_lat[p];
        fu.dF[p] = dU[p];
        fu.dsc[p] = dh[p];
        fv.s[p] = B->g32 + (size_t)p * K;
        fv.words[p] = B->Vw + (size_t)p * K * wpr;
        fv.F[p] = V_lat[p];
        fv.dF[p] = dV[p];
        fv.dsc[p] = dg[p];
    }
    bool vec4 = r % 4 == 0;
    for (int p = 0; p < B->npaths; ++p)
        vec4 = vec4 && !(((uintptr_t)U_lat[p] | (uintptr_t)V_lat[p] | (uintptr_t)dU[p] | (uintptr_t)dV[p]) & 15);
    if (vec4) {
        if (B->npaths == 2) {
            factor_grad4_kernel<2><<<grid_for(32L * N), kT, 0, s2>>>(B->GU, N, K2, r, B->r8, fu);
            factor_grad4_kernel<2><<<grid_for(32L * K), kT, 0, s2>>>(B->GV, K, K2, r, B->r8, fv);
        } else {
            factor_grad4_kernel<1><<<grid_for(32L * N), kT, 0, s2>>>(B->GU, N, K2, r, B->r8, fu);
            factor_grad4_kernel<1><<<grid_for(32L * K), kT, 0, s2>>>(B->GV, K, K2, r, B->r8, fv);
        }
    } else if (B->npaths == 2) {
        factor_grad_kernel<2><<<grid_for(32L * N), kT, 0, s2>>>(B->GU, N, K2, r, B->r8, fu);
        factor_grad_kernel<2><<<grid_for(32L * K), kT, 0, s2>>>(B->GV, K, K2, r, B->r8, fv);
    } else {
        factor_grad_kernel<1><<<grid_for(32L * N), kT, 0, s2>>>(B->GU, N, K2, r, B->r8, fu);
        factor_grad_kernel<1><<<grid_for(32L * K), kT, 0, s2>>>(B->GV, K, K2, r, B->r8, fv);
    }
    launches += 2;
    profile_mark(8, s2);
    if (cudaEventRecord(B->join, s2) != cudaSuccess || cudaStreamWaitEvent(s, B->join, 0) != cudaSuccess)
        return LB_ERR_CUDA;
    set_launch_count(launches);
    return cudaGetLastError() == cudaSuccess ? LB_OK : LB_ERR_CUDA;
}

lb_status lb_backward_status(lb_backward *B, void *stream)
{
    if (!B) return LB_ERR_INVALID_ARG;
    lb_status a = lb_layer_status(B->Lf, stream), b = lb_layer_status(B->Lt, stream);
    lb_status c = LB_OK;
    // the error slots of the one-launch latent contractions and of the G_U / G_V GEMMs
    for (int *e : {prefill_jobs_err(B->jobs), B->gerr}) {
        if (!e) continue;
        cudaStream_t s = (cudaStream_t)stream;
        int h = 0;
        if (cudaMemcpyAsync(&h, e, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return LB_ERR_CUDA;
        if (h) {
            cudaMemsetAsync(e, 0, sizeof(int), s);
            cudaStreamSynchronize(s);
            c = LB_ERR_TIMEOUT;
        }
    }
    return a != LB_OK ? a : b != LB_OK ? b : c;
}

}  // extern "C"

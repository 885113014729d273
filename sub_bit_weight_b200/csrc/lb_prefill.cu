// Large-batch (prefill) forward of LittleBit layers on 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory).
//
// With many activation rows the two binary contractions of a path
// (LittleBit notes page, "Multi-scale compensation": x (.) g . V_sign (.) l
// . U_sign^T (.) h) are dense skinny GEMMs, so they run as two fp16 x fp16 ->
// fp32 tensor-core GEMMs whose weight operand is generated in shared memory
// from the packed signs:
//
//   latent:  z[m][j'] = sum_k fp16(x[m][k]) * (+-g_p[k])     (+-g exact in fp16)
//            zl = fp16(z * l_p[j])                            (both paths: j' = p*r8 + j)
//   output:  y[m][n]  = sum_j' zl[m][j'] * (+-h_p(j')[n])    (both paths in one GEMM)
//
// Folding g and h into the generated operand keeps every product exact and
// lets one accumulator carry both paths ("Residual compensation" sums them).
//
// Kernel structure (one persistent CTA per SM, 16 warps):
//   warp 0      TMA producer: A tile (128 x 64, 128-byte swizzle) + the 4 KB
//               block of packed signs of the B tile, one mbarrier per stage
//   warp 1      tcgen05.mma issuer (one thread) and tensor-memory owner
//   warps 4-7   epilogue: tcgen05.ld of the fp32 accumulator, scaling, stores
//   warps 8-15  generators: B tile (256 x 64 fp16, 128-byte swizzle) from
//               signs and scales; the latent GEMM also converts the bf16 A
//               tile to fp16 in place.  The output GEMM's sign bits arrive in
//               the first 4 KB of the B stage they are expanded into, so the
//               generator warp that writes those rows waits until every
//               generator has read its bits; the latent GEMM's arrive in its
//               unused epilogue staging area and need no wait
// Two accumulators of 256 columns in tensor memory let the epilogue of one
// tile overlap the main loop of the next.  Every wait is bounded: on timeout
// the kernel records an error code and returns.

#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "lb_prefill.cuh"
#include "lb_tc.cuh"

namespace lb {

// ---------------------------------------------------------------------------
// Weight layouts (built once per layer)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t canon_bit_pf(const uint32_t *P, int wpr, int64_t row, int col)
{
    return (__ldg(P + row * wpr + (col >> 5)) >> (col & 31)) & 1u;
}

// Spread words of the latent-contraction operand: rows j' (path p = j'/r8),
// k = inputs.  Bit = V_sign_p[k][j] < 0.
__global__ void build_b1_kernel(uint32_t *__restrict__ out, int RT1, int KB1, int r, int r8, int K,
                                int npaths, const uint32_t *__restrict__ V0, const uint32_t *__restrict__ V1)
{
    const int wpr = (r + 31) / 32;
    const int64_t total = (int64_t)RT1 * KB1 * 256 * 4;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int q = (int)(idx & 3);
        const int row = (int)((idx >> 2) & 255);
        const int64_t blk = idx >> 10;
        const int kb = (int)(blk % KB1), rt = (int)(blk / KB1);
        const int jr = rt * 256 + row;
        const int p = jr / r8, j = jr - p * r8;
        uint32_t w = 0;
        if (p < npaths && j < r) {
            const uint32_t *V = p ? V1 : V0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int k0 = kb * 64 + 16 * q + 2 * i;
                if (k0 < K) w |= canon_bit_pf(V, wpr, k0, j) << (15 - i);
                if (k0 + 1 < K) w |= canon_bit_pf(V, wpr, k0 + 1, j) << (31 - i);
            }
        }
        out[idx] = w;
    }
}

// Spread words of the output-contraction operand: rows n, k = j' (path p = j'/r8).
// Bit = U_sign_p[n][j] < 0.
__global__ void build_b2_kernel(uint32_t *__restrict__ out, int RT2, int KB2, int r, int r8, int N,
                                int npaths, const uint32_t *__restrict__ U0, const uint32_t *__restrict__ U1)
{
    const int wpr = (r + 31) / 32;
    const int64_t total = (int64_t)RT2 * KB2 * 256 * 4;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int q = (int)(idx & 3);
        const int row = (int)((idx >> 2) & 255);
        const int64_t blk = idx >> 10;
        const int kb = (int)(blk % KB2), rt = (int)(blk / KB2);
        const int n = rt * 256 + row;
        uint32_t w = 0;
        if (n < N) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int jr = kb * 64 + 16 * q + 2 * i + h;
                    const int p = jr / r8, j = jr - p * r8;
                    if (p < npaths && j < r)
                        w |= canon_bit_pf(p ? U1 : U0, wpr, n, j) << (h ? 31 - i : 15 - i);
                }
            }
        }
        out[idx] = w;
    }
}

// g of both paths per 64-wide k-block: dst[kb][p][0..64), zero beyond K and for an absent path.
__global__ void g_blocks_kernel(__half *__restrict__ dst, const uint16_t *__restrict__ g0,
                                const uint16_t *__restrict__ g1, int npaths, int K, int KB1)
{
    const int64_t total = (int64_t)KB1 * 128;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int kb = (int)(idx >> 7), p = (int)((idx >> 6) & 1), i = (int)(idx & 63);
        const int k = kb * 64 + i;
        uint16_t v = 0;
        if (p < npaths && k < K) v = (p ? g1 : g0)[k];
        dst[idx] = __ushort_as_half(v);
    }
}

__global__ void pad_half_kernel(__half *__restrict__ dst, const uint16_t *__restrict__ s0,
                                const uint16_t *__restrict__ s1, int npaths, int n, int npad)
{
    const int64_t total = (int64_t)npaths * npad;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int p = (int)(idx / npad), i = (int)(idx - (int64_t)p * npad);
        dst[idx] = __ushort_as_half((i < n) ? (p ? s1 : s0)[i] : (uint16_t)0);
    }
}

__global__ void lcat_kernel(float *__restrict__ dst, const uint16_t *__restrict__ l0,
                            const uint16_t *__restrict__ l1, int npaths, int r, int r8, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int p = i / r8, j = i - p * r8;
        float v = 0.0f;
        if (p < npaths && j < r) v = __half2float(__ushort_as_half((p ? l1 : l0)[j]));
        dst[i] = v;
    }
}

static void pf_dims(PfWeights &W, const LayerDev &d)
{
    W.r8 = round_up(d.r, 8);
    W.N1 = d.npaths * W.r8;
    W.N1p = round_up(W.N1, 16);
    W.K64 = round_up(d.K, 64);
    W.KB1 = W.K64 / 64;
    W.RT1 = ceil_div(W.N1p, 256);
    W.K2 = round_up(W.N1p, 64);
    W.KB2 = W.K2 / 64;
    W.RT2 = ceil_div(d.N, 256);
    W.N256 = W.RT2 * 256;
}

static size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t prefill_weight_bytes(const LayerDev &d)
{
    PfWeights W;
    pf_dims(W, d);
    return al256((size_t)W.RT1 * W.KB1 * 4096) + al256((size_t)W.KB1 * 128 * 2) +
           al256((size_t)W.N1p * 4) + al256((size_t)W.RT2 * W.KB2 * 4096) + al256((size_t)d.npaths * W.N256 * 2);
}

cudaError_t prefill_build_weights(PfWeights &W, const LayerDev &d, const uint32_t *const *U,
                                  const uint32_t *const *V, const uint16_t *const *h,
                                  const uint16_t *const *g, const uint16_t *const *l, cudaStream_t s)
{
    // memory was carved by the caller: W.b1 points at the start of prefill_weight_bytes(d) bytes
    pf_dims(W, d);
    char *c = (char *)W.b1;
    W.b1 = (uint32_t *)c;      c += al256((size_t)W.RT1 * W.KB1 * 4096);
    W.g64 = (__half *)c;       c += al256((size_t)W.KB1 * 128 * 2);
    W.lcat = (float *)c;       c += al256((size_t)W.N1p * 4);
    W.b2 = (uint32_t *)c;      c += al256((size_t)W.RT2 * W.KB2 * 4096);
    W.h256 = (__half *)c;
    const int P = d.npaths;
    const int T = 256;
    auto grid = [](int64_t n) { return (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 32)); };
    build_b1_kernel<<<grid((int64_t)W.RT1 * W.KB1 * 1024), T, 0, s>>>(W.b1, W.RT1, W.KB1, d.r, W.r8, d.K, P, V[0],
                                                                      P > 1 ? V[1] : V[0]);
    build_b2_kernel<<<grid((int64_t)W.RT2 * W.KB2 * 1024), T, 0, s>>>(W.b2, W.RT2, W.KB2, d.r, W.r8, d.N, P, U[0],
                                                                      P > 1 ? U[1] : U[0]);
    g_blocks_kernel<<<grid((int64_t)W.KB1 * 128), T, 0, s>>>(W.g64, g[0], P > 1 ? g[1] : g[0], P, d.K, W.KB1);
    pad_half_kernel<<<grid((int64_t)P * W.N256), T, 0, s>>>(W.h256, h[0], P > 1 ? h[1] : h[0], P, d.N, W.N256);
    lcat_kernel<<<grid(W.N1p), T, 0, s>>>(W.lcat, l[0], P > 1 ? l[1] : l[0], P, d.r, W.r8, W.N1p);
    return cudaGetLastError();
}


// Instruction descriptor: fp16 A and B (K-major), fp32 accumulator, M = 128.
__device__ __forceinline__ uint32_t idesc_f16(int n)
{
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kPfBM >> 4) << 24);
}

// bf16x2 -> fp16x2 (exact for |x| in the normal fp16 range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v)
{
    const float lo = __uint_as_float(v << 16);
    const float hi = __uint_as_float(v & 0xffff0000u);
    const __half2 hh = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&hh);
}

// ---------------------------------------------------------------------------
// The tensor-core contraction kernel
// ---------------------------------------------------------------------------
static_assert(kPfStages == 4, "the latent GEMM keeps one stage's sign bits in each of the four staging blocks");
struct PfSmem {
    alignas(1024) unsigned char A[kPfStages][kPfBM * kPfBK * 2];
    alignas(1024) unsigned char B[kPfStages][kPfBN * kPfBK * 2];   // the stage's sign bits land in its first 4 KB
    alignas(1024) unsigned char ST[4][32 * 128];  // output GEMM epilogue: 32x32 fp32 block per warp (128B swizzle);
                                                  // latent GEMM: the sign bits of stage s (4 KB) in ST[s]
    alignas(16) __half gst[kPfStages][128];     // latent GEMM: g of both paths for the stage's k-block
    alignas(16) float lsc[kPfBN];               // latent GEMM epilogue: l of the tile's columns
    uint64_t full[kPfStages], ready[kPfStages], empty[kPfStages], bread[kPfStages];
    uint64_t accf[2], acce[2];
    uint32_t tmem_base;
    int abort;
    int tile_start[1];   // flexible: [nlayers + 1]
};

template <int MODE>
__global__ void __launch_bounds__(pf_threads(MODE), 1)
    prefill_kernel(const PfLayer *__restrict__ layers, const int *__restrict__ tile_start, int nlayers, int M,
                   int *err)
{
    extern __shared__ __align__(1024) unsigned char pf_raw[];
    // align inside the shared window by an offset, keeping the pointer a shared-memory pointer
    const uint32_t raw_addr = smem_u32(pf_raw);
    PfSmem &S = *reinterpret_cast<PfSmem *>(pf_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int *abort = &S.abort;

    for (int i = tid; i <= nlayers; i += blockDim.x) S.tile_start[i] = tile_start[i];
    if (tid == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.ready[s], MODE == 0 ? 10 + kPfExtraConv : 8);   // generator warps (+ converter warps)
            mbar_init(&S.bread[s], 8);                    // output GEMM: generator warps have read the stage's bits
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.accf[b], 1);
            mbar_init(&S.acce[b], 4);
        }
        S.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(smem_u32(&S.tmem_base)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const int total = S.tile_start[nlayers];

    // unit t -> layer L, tile (mt, nt) and k-blocks [kb0, kb1); the k-range index is the slowest, so the units of
    // one tile fall in different waves
    const int mtiles = (M + kPfBM - 1) / kPfBM;
    auto locate = [&](int t, int &L, int &mt, int &nt, int &kb0, int &kb1) {
        int lo = 0, hi = nlayers - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (S.tile_start[mid] <= t) lo = mid; else hi = mid - 1;
        }
        L = lo;
        int local = t - S.tile_start[lo];
        const int ntn = layers[lo].ntn, nsp = layers[lo].ksplit, nk = layers[lo].nk;
        const int ks = local / (mtiles * ntn);
        local -= ks * mtiles * ntn;
        mt = local / ntn;
        nt = local - mt * ntn;
        kb0 = ks * nk / nsp;
        kb1 = (ks + 1) * nk / nsp;
    };

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            uint32_t it = 0;
            uint32_t pend = 0, pend_ph = 0;   // stages with a copy issued, and its phase parity
            for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
                int L, mt, nt, kb0, kb1;
                locate(t, L, mt, nt, kb0, kb1);
                const PfLayer ly = layers[L];   // register copy: waits below clobber memory
                const uint32_t *bits = ly.bits + (size_t)nt * ly.nk * 1024;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % kPfStages;
                    const uint32_t ph = (it / kPfStages) & 1;
                    if (!mbar_wait(&S.empty[s], ph ^ 1, abort, err, 1)) break;
                    mbar_expect_tx(&S.full[s], kPfBM * kPfBK * 2 + 4096 + (MODE == 0 ? 256 : 0));
                    tma_load_2d(S.A[s], ly.tmA, kb * kPfBK, mt * kPfBM, &S.full[s]);
                    // latent GEMM: the sign bits go to the (otherwise unused) staging area, so the generators
                    // overwrite nothing they still read; output GEMM: the first 4 KB of the B stage
                    bulk_load(MODE == 0 ? (void *)S.ST[s] : (void *)S.B[s], bits + (size_t)kb * 1024, 4096, &S.full[s]);
                    if (MODE == 0) bulk_load(S.gst[s], ly.base + (size_t)kb * 128, 256, &S.full[s]);
                    pend |= 1u << s;
                    pend_ph = (pend_ph & ~(1u << s)) | (ph << s);
                }
            }
            if (*abort) {
                // let the copies already issued land before the CTA leaves (bounded)
                for (int s = 0; s < kPfStages; ++s) {
                    if (!(pend >> s & 1)) continue;
                    const long long t0 = clock64();
                    while (!mbar_try_wait(&S.full[s], (pend_ph >> s) & 1) && clock64() - t0 < kWaitCycles / 20) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0, tcount = 0;
            for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x, ++tcount) {
                int L, mt, nt, kb0, kb1;
                locate(t, L, mt, nt, kb0, kb1);
                const PfLayer ly = layers[L];   // register copy: waits below clobber memory
                const int nw = min(kPfBN, ly.ncols - nt * kPfBN);
                const int ab = tcount & 1;
                const uint32_t aph = (tcount >> 1) & 1;
                if (!mbar_wait(&S.acce[ab], aph ^ 1, abort, err, 2)) break;
                tc_fence_after();
                const uint32_t idesc = idesc_f16((nw + 15) & ~15);
                const uint32_t dacc = tmem + (uint32_t)(ab * kPfBN);
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % kPfStages;
                    const uint32_t ph = (it / kPfStages) & 1;
                    if (!mbar_wait(&S.full[s], ph, abort, err, 3) || !mbar_wait(&S.ready[s], ph, abort, err, 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(S.A[s]);
                    const uint64_t bd = smem_desc_sw128(S.B[s]);
#pragma unroll
                    for (int kk = 0; kk < kPfBK / 16; ++kk)
                        tc_mma_f16(dacc, ad + 2 * kk, bd + 2 * kk, idesc, (kb > kb0 || kk) ? 1u : 0u);
                    tc_commit(&S.empty[s]);
                }
                if (!ok) break;
                tc_commit(&S.accf[ab]);
            }
        }
    } else if (warp == 2 || warp == 3 || warp >= 16) {
        // ---------------- converters (latent GEMM): bf16 -> fp16 A tile in place
        if (MODE == 0) {
            constexpr int kConv = 32 * (2 + kPfExtraConv);
            const int ct = warp < 16 ? tid - 64 : tid - 512 + 64;   // 0 .. kConv - 1
            uint32_t it = 0;
            for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
                int L, mt, nt, kb0, kb1;
                locate(t, L, mt, nt, kb0, kb1);
                const int a_f16 = layers[L].a_f16;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % kPfStages;
                    const uint32_t ph = (it / kPfStages) & 1;
                    if (!mbar_wait(&S.full[s], ph, abort, err, 7)) {
                        ok = false;
                        break;
                    }
                    const uint32_t A0 = smem_u32(S.A[s]);
                    if (!a_f16) {
#pragma unroll 2
                        for (int i = ct; i < kPfBM * kPfBK * 2 / 16; i += kConv) {
                            uint4 v = lds128(A0 + 16u * i);
                            v.x = bf16x2_to_f16x2(v.x);
                            v.y = bf16x2_to_f16x2(v.y);
                            v.z = bf16x2_to_f16x2(v.z);
                            v.w = bf16x2_to_f16x2(v.w);
                            sts128(A0 + 16u * i, v);
                        }
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.ready[s]);
                }
                if (!ok) break;
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- epilogue
        const int q = warp - 4;
        uint32_t tcount = 0;
        for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x, ++tcount) {
            int L, mt, nt, kb0, kb1;
            locate(t, L, mt, nt, kb0, kb1);
            const PfLayer ly = layers[L];   // register copy: waits below clobber memory
            const int nw = min(kPfBN, ly.ncols - nt * kPfBN);
            const int ab = tcount & 1;
            const uint32_t aph = (tcount >> 1) & 1;
            if (!mbar_wait(&S.accf[ab], aph, abort, err, 5)) break;
            tc_fence_after();
            if (MODE == 0 && !ly.part) {
                // l of this tile's columns into shared memory (the 4 epilogue warps, named barrier 1)
                asm volatile("bar.sync 1, 128;\n" ::: "memory");   // previous tile done with S.lsc
                for (int i = tid - 128; i < kPfBN; i += 128) {
                    const int c = nt * kPfBN + i;
                    S.lsc[i] = (c < ly.ncols) ? __ldg(ly.lcat + c) : 0.0f;
                }
                asm volatile("bar.sync 1, 128;\n" ::: "memory");
            }
            const int m = mt * kPfBM + q * 32 + lane;
            for (int ch = 0; ch < nw; ch += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * kPfBN + ch), v);
                const int c0 = nt * kPfBN + ch;
                if (MODE == 0 && ly.part) {
                    // k-split unit: add the raw partial sums (fp32) to the caller's zeroed buffer
                    if (m < M) {
                        float *o = ly.part + (size_t)m * ly.ld_part + c0;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            if (c0 + 4 * i < ly.ncols)
                                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(o + 4 * i),
                                             "f"(__uint_as_float(v[4 * i])), "f"(__uint_as_float(v[4 * i + 1])),
                                             "f"(__uint_as_float(v[4 * i + 2])), "f"(__uint_as_float(v[4 * i + 3]))
                                             : "memory");
                    }
                } else if (MODE == 0) {
                    if (m < M) {
                        __half *out = reinterpret_cast<__half *>(ly.out) + (size_t)m * ly.ld_out + c0;
                        uint32_t hw[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int c = c0 + 2 * i;
                            const uint32_t la = smem_u32(&S.lsc[ch + 2 * i]);
                            const float a = __uint_as_float(v[2 * i]) * __uint_as_float(lds32(la));
                            const float b = __uint_as_float(v[2 * i + 1]) * __uint_as_float(lds32(la + 4));
                            (void)c;
                            const __half2 hh = __floats2half2_rn(a, b);
                            hw[i] = *reinterpret_cast<const uint32_t *>(&hh);
                        }
                        if (c0 + 32 <= ly.ncols) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                reinterpret_cast<uint4 *>(out)[i] = make_uint4(hw[4 * i], hw[4 * i + 1], hw[4 * i + 2], hw[4 * i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                if (c0 + 2 * i < ly.ncols) reinterpret_cast<uint32_t *>(out)[i] = hw[i];
                        }
                    }
                }
                if (MODE == 1) {
                    if (ly.oscale) {
                        const float f = __ldg(ly.oscale);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
                    }
                    // 32 rows x 32 columns of y through a 128B-swizzled block and one TMA store
                    if (ch > 0 || tcount > 0) {
                        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
                        __syncwarp();
                    }
                    unsigned char *st = S.ST[q];
                    const uint32_t sta = smem_u32(st);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        sts128(sta + sw128(lane, i), make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0 && mt * kPfBM + q * 32 < M) {
                        asm volatile(
                            "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(ly.tmY),
                            "r"(c0), "r"(mt * kPfBM + q * 32), "r"(smem_u32(st))
                            : "memory");
                        asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.acce[ab]);
        }
    } else if (warp >= 8) {
        // ---------------- generators (256 threads)
        const int gt = tid - 256;
        const int gw = warp - 8;
        uint32_t it = 0;
        for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
            int L, mt, nt, kb0, kb1;
            locate(t, L, mt, nt, kb0, kb1);
            const PfLayer ly = layers[L];   // register copy: waits below clobber memory
            const int nw = min(kPfBN, ly.ncols - nt * kPfBN);
            // output contraction: this thread's row n and its two path scales
            uint32_t hh[2] = {0u, 0u};
            if (MODE == 1) {
                const int n = nt * kPfBN + gt;
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    if (p < ly.npaths) {
                        const uint16_t hb = __half_as_ushort(ly.base[(size_t)p * ly.base_ld + n]);
                        hh[p] = (uint32_t)hb | ((uint32_t)hb << 16);
                    }
                }
            }
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % kPfStages;
                const uint32_t ph = (it / kPfStages) & 1;
                if (!mbar_wait(&S.full[s], ph, abort, err, 6)) {
                    ok = false;
                    break;
                }
                const uint32_t Bt = smem_u32(S.B[s]);   // output GEMM: sign bits first: [256 rows][4 words]
                if (MODE == 0) {
                    // thread -> chunk c (8 inputs), rows gt/8 + 32 i; the bits sit apart from B (no barrier)
                    const uint32_t Bits = smem_u32(S.ST[s]);
                    const int c = gt & 7;
                    uint32_t R[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) R[i] = lds32(Bits + 4u * (((gt >> 3) + 32 * i) * 4 + (c >> 1)));
                    uint4 gb[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) gb[p] = lds128(smem_u32(S.gst[s] + p * 64 + 8 * c));
                    const int sh0 = 4 * (c & 1);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int row = (gt >> 3) + 32 * i;
                        if (row < nw) {
                            const int jr = nt * kPfBN + row;
                            const uint4 base = (jr >= ly.r8 && ly.npaths > 1) ? gb[1] : gb[0];
                            uint4 o;
                            o.x = ((R[i] << (sh0 + 0)) & 0x80008000u) ^ base.x;
                            o.y = ((R[i] << (sh0 + 1)) & 0x80008000u) ^ base.y;
                            o.z = ((R[i] << (sh0 + 2)) & 0x80008000u) ^ base.z;
                            o.w = ((R[i] << (sh0 + 3)) & 0x80008000u) ^ base.w;
                            sts128(Bt + sw128(row, c), o);
                        }
                    }
                } else {
                    // thread -> row gt, all 8 chunks.  The bits sit in B rows 0..31: only the warp that writes
                    // those rows waits until every generator has read its bits
                    const int row = gt;
                    const uint4 Rw = lds128(Bt + 16u * row);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.bread[s]);
                    if (gw == 0 && !mbar_wait(&S.bread[s], ph, abort, err, 8)) {
                        ok = false;
                        break;
                    }
                    if (row < nw) {
                        const uint32_t Rs[4] = {Rw.x, Rw.y, Rw.z, Rw.w};
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int jr = kb * kPfBK + 8 * c;
                            const uint32_t base = (jr >= ly.r8 && ly.npaths > 1) ? hh[1] : hh[0];
                            const uint32_t R = Rs[c >> 1];
                            const int sh0 = 4 * (c & 1);
                            uint4 o;
                            o.x = ((R << (sh0 + 0)) & 0x80008000u) ^ base;
                            o.y = ((R << (sh0 + 1)) & 0x80008000u) ^ base;
                            o.z = ((R << (sh0 + 2)) & 0x80008000u) ^ base;
                            o.w = ((R << (sh0 + 3)) & 0x80008000u) ^ base;
                            sts128(Bt + sw128(row, c), o);
                        }
                    }
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.ready[s]);
            }
            if (!ok) break;
            (void)gw;
        }
    }

    if (MODE == 1 && warp >= 4 && warp < 8 && lane == 0) asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem));
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

cudaError_t tmap_encoder_ready()
{
    std::call_once(g_encode_once, [] {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    });
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

bool tmap_encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, long cols, long rows,
                    long pitch_bytes, int box_cols, int box_rows)
{
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static cudaError_t get_encoder() { return tmap_encoder_ready(); }

static bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, int cols, int rows,
                      int esize = 2, int box_cols = kPfBK, int box_rows = kPfBM)
{
    return tmap_encode_2d(map, dt, base, cols, rows, (long)cols * esize, box_cols, box_rows);
}

struct PrefillState {
    int M = 0;                       // rows the scratch was sized for
    int lastM = -1;
    bool lastF16 = false;            // the activations of the last encoded maps are fp16
    const float *lastScale = nullptr;   // the output scale of the last encoded records
    std::vector<const void *> lastX, lastY;
    void *zl = nullptr;              // latent activations of every layer, fp16 [M][K2]
    std::vector<size_t> zl_off;
    CUtensorMap *maps = nullptr;     // device: [2 * n] (x maps, zl maps), 64-byte aligned
    PfLayer *rec = nullptr;          // device: [2 * n] (latent records, output records)
    int *starts = nullptr;           // device: [2 * (n + 1)]
    int *err = nullptr;              // device error code
    int tiles[2] = {0, 0};
};

int *prefill_err_ptr(PrefillState *st) { return st->err; }

void prefill_free(PrefillState *st)
{
    if (!st) return;
    cudaFree(st->zl);
    cudaFree(st->maps);
    cudaFree(st->rec);
    cudaFree(st->starts);
    cudaFree(st->err);
    delete st;
}

static size_t smem_bytes(int nlayers) { return sizeof(PfSmem) + 1024 + sizeof(int) * (size_t)(nlayers + 1); }

static int sm_count()
{
    int sms = 0;
    if (sm_count_of_current(&sms) != cudaSuccess || sms <= 0) sms = 148;
    return sms;
}

// raise the kernels' dynamic shared-memory limit to at least `smem` (grow-only, shared by every launch path)
static cudaError_t ensure_smem(size_t smem)
{
    if (smem > 232448) return cudaErrorInvalidValue;
    cudaError_t e;
    if ((e = ensure_dyn_smem((const void *)prefill_kernel<0>, smem)) != cudaSuccess) return e;
    return ensure_dyn_smem((const void *)prefill_kernel<1>, smem);
}

lb_status prefill_forward(const Plan &Pc, const lb_layer *const *layers, const uint16_t *const *xs,
                          float *const *ys, int M, cudaStream_t s, int *launches, int parts, bool a_f16,
                          bool marks, const float *out_scale)
{
    Plan &P = const_cast<Plan &>(Pc);
    const int n = P.n;
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return LB_ERR_UNSUPPORTED;
    for (int i = 0; i < n; ++i) {
        const LayerDev &d = layers[i]->d;
        if (d.K % 8 || d.N % 4) return LB_ERR_UNSUPPORTED;   // TMA row strides must be multiples of 16 bytes
    }
    if (!P.pf) {
        P.pf = new (std::nothrow) PrefillState();
        if (!P.pf) return LB_ERR_OOM;
        PrefillState &st = *P.pf;
        if ((e = cudaMalloc(&st.maps, sizeof(CUtensorMap) * 3 * n)) != cudaSuccess) return status_from(e);
        if ((e = cudaMalloc(&st.rec, sizeof(PfLayer) * 2 * n)) != cudaSuccess) return status_from(e);
        if ((e = cudaMalloc(&st.starts, sizeof(int) * 2 * (n + 1))) != cudaSuccess) return status_from(e);
        if ((e = cudaMalloc(&st.err, sizeof(int))) != cudaSuccess) return status_from(e);
        if ((e = cudaMemsetAsync(st.err, 0, sizeof(int), s)) != cudaSuccess) return status_from(e);
    }
    PrefillState &st = *P.pf;
    bool dirty = false;
    if (M > st.M) {
        // grow the latent scratch; padding columns stay zero
        if (st.zl) {
            cudaStreamSynchronize(s);
            cudaFree(st.zl);
            st.zl = nullptr;
        }
        size_t tot = 0;
        st.zl_off.resize(n);
        for (int i = 0; i < n; ++i) {
            st.zl_off[i] = tot;
            tot += ((size_t)M * layers[i]->pf.K2 * 2 + 255) & ~(size_t)255;
        }
        if ((e = cudaMalloc(&st.zl, tot)) != cudaSuccess) return status_from(e);
        if ((e = cudaMemsetAsync(st.zl, 0, tot, s)) != cudaSuccess) return status_from(e);
        st.M = M;
        dirty = true;
    }
    if (M != st.lastM || a_f16 != st.lastF16 || out_scale != st.lastScale) dirty = true;
    if ((int)st.lastX.size() != n) {
        st.lastX.assign(n, nullptr);
        st.lastY.assign(n, nullptr);
        dirty = true;
    }
    for (int i = 0; i < n && !dirty; ++i)
        if (st.lastX[i] != xs[i] || st.lastY[i] != ys[i]) dirty = true;
    if (dirty) {
        std::vector<CUtensorMap> maps(3 * n);
        std::vector<PfLayer> rec(2 * n);
        std::vector<int> starts(2 * (n + 1));
        starts[0] = starts[n + 1] = 0;
        for (int i = 0; i < n; ++i) {
            const LayerDev &d = layers[i]->d;
            const PfWeights &W = layers[i]->pf;
            __half *zl = (__half *)((char *)st.zl + st.zl_off[i]);
            if (!encode_2d(&maps[i], a_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xs[i],
                           d.K, M) ||
                !encode_2d(&maps[n + i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, zl, W.K2, M) ||
                !encode_2d(&maps[2 * n + i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ys[i], d.N, M, 4, 32, 32))
                return LB_ERR_UNSUPPORTED;
            const int mtiles = ceil_div(M, kPfBM);
            PfLayer &a = rec[i];
            a.tmA = st.maps + i;
            a.tmY = nullptr;
            a.bits = W.b1;
            a.base = W.g64;
            a.lcat = W.lcat;
            a.out = zl;
            a.nk = W.KB1;
            a.ncols = W.N1p;
            a.ld_out = W.K2;
            a.ntn = ceil_div(W.N1p, kPfBN);
            a.r8 = W.r8;
            a.base_ld = W.K64;
            a.npaths = d.npaths;
            a.a_f16 = a_f16;
            a.ksplit = 1;
            a.part = nullptr;
            a.ld_part = 0;
            a.oscale = nullptr;
            PfLayer &b = rec[n + i];
            b.tmA = st.maps + n + i;
            b.tmY = st.maps + 2 * n + i;
            b.bits = W.b2;
            b.base = W.h256;
            b.lcat = nullptr;
            b.out = ys[i];
            b.nk = W.KB2;
            b.ncols = d.N;
            b.ld_out = d.N;
            b.ntn = ceil_div(d.N, kPfBN);
            b.r8 = W.r8;
            b.base_ld = W.N256;
            b.npaths = d.npaths;
            b.a_f16 = 0;
            b.ksplit = 1;
            b.part = nullptr;
            b.ld_part = 0;
            b.oscale = out_scale;
            starts[i + 1] = starts[i] + mtiles * a.ntn;
            starts[n + 1 + i + 1] = starts[n + 1 + i] + mtiles * b.ntn;
            st.lastX[i] = xs[i];
            st.lastY[i] = ys[i];
        }
        st.tiles[0] = starts[n];
        st.tiles[1] = starts[2 * n + 1];
        st.lastM = M;
        st.lastF16 = a_f16;
        st.lastScale = out_scale;
        // pageable sources: the copies are staged before these calls return
        if ((e = cudaMemcpyAsync(st.maps, maps.data(), sizeof(CUtensorMap) * 3 * n, cudaMemcpyHostToDevice, s)) !=
            cudaSuccess)
            return status_from(e);
        if ((e = cudaMemcpyAsync(st.rec, rec.data(), sizeof(PfLayer) * 2 * n, cudaMemcpyHostToDevice, s)) != cudaSuccess)
            return status_from(e);
        if ((e = cudaMemcpyAsync(st.starts, starts.data(), sizeof(int) * 2 * (n + 1), cudaMemcpyHostToDevice, s)) !=
            cudaSuccess)
            return status_from(e);
        if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return status_from(e);
    }

    const int sms = sm_count();
    const size_t smem = smem_bytes(n);
    if ((e = ensure_smem(smem)) != cudaSuccess) return smem > 232448 ? LB_ERR_UNSUPPORTED : status_from(e);
    const int g0 = std::max(1, std::min(st.tiles[0], sms));
    const int g1 = std::max(1, std::min(st.tiles[1], sms));
    if (marks) profile_mark(0, s);
    if (parts & 1) {
        prefill_kernel<0><<<g0, pf_threads(0), smem, s>>>(st.rec, st.starts, n, M, st.err);
        ++*launches;
        if (marks) profile_mark(*launches, s);
    }
    if (parts & 2) {
        prefill_kernel<1><<<g1, pf_threads(1), smem, s>>>(st.rec + n, st.starts + n + 1, n, M, st.err);
        ++*launches;
        if (marks) profile_mark(*launches, s);
    }
    return status_from(cudaGetLastError());
}

__half *prefill_zl(const Plan &P, int i)
{
    if (!P.pf || !P.pf->zl || i < 0 || i >= (int)P.pf->zl_off.size()) return nullptr;
    return (__half *)((char *)P.pf->zl + P.pf->zl_off[i]);
}

// ---------------------------------------------------------------------------
// Latent contractions of several layers with k-split units (one launch)
// ---------------------------------------------------------------------------
struct PfJobState {
    int n = 0, lastM = -1;
    std::vector<const void *> lastX;
    std::vector<float *> lastPart;
    std::vector<int> lastF16;
    CUtensorMap *maps = nullptr;   // device [n]
    PfLayer *rec = nullptr;        // device [n]
    int *starts = nullptr;         // device [n + 1]
    int *err = nullptr;
    int total = 0;
};

void prefill_jobs_free(PfJobState *st)
{
    if (!st) return;
    cudaFree(st->maps);
    cudaFree(st->rec);
    cudaFree(st->starts);
    cudaFree(st->err);
    delete st;
}

int *prefill_jobs_err(PfJobState *st) { return st ? st->err : nullptr; }

// k-ranges per tile for each job so that the kernel's round-robin assignment of units to `grid` CTAs finishes
// evenly: every target unit length u is tried, job i gets round(nk_i / u) ranges, and the unit costs (k-blocks +
// a fixed per-unit overhead) are dealt out in the kernel's order; the smallest makespan wins.
static std::vector<int> choose_splits(const std::vector<int> &tiles, const std::vector<int> &nk, int sms)
{
    const int n = (int)tiles.size();
    const double overhead = 3.0;      // pipeline fill and epilogue of a unit, in k-blocks
    int maxnk = 1;
    for (int v : nk) maxnk = std::max(maxnk, v);
    std::vector<int> best(n, 1), cur(n);
    double best_t = 1e300;
    std::vector<double> load;
    for (int u = 1; u <= maxnk; ++u) {
        long units = 0;
        for (int i = 0; i < n; ++i) {
            cur[i] = std::max(1, std::min(nk[i], (nk[i] + u / 2) / u));
            units += (long)tiles[i] * cur[i];
        }
        const int grid = (int)std::min<long>(units, sms);
        load.assign(grid, 0.0);
        long t = 0;
        for (int i = 0; i < n; ++i)
            for (int ks = 0; ks < cur[i]; ++ks) {
                const double c = (ks + 1) * nk[i] / cur[i] - ks * nk[i] / cur[i] + overhead;
                for (int k = 0; k < tiles[i]; ++k, ++t) load[t % grid] += c;
            }
        double mk = 0.0;
        for (double v : load) mk = std::max(mk, v);
        if (mk < best_t - 1e-9) {
            best_t = mk;
            best = cur;
        }
    }
    return best;
}

lb_status prefill_latent_jobs(PfJobState **state, const PfLatentJob *jobs, int n, int M, cudaStream_t s,
                              int *launches)
{
    if (!state || !jobs || n < 1 || M < 1) return LB_ERR_INVALID_ARG;
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return LB_ERR_UNSUPPORTED;
    for (int i = 0; i < n; ++i) {
        if (!jobs[i].layer || !jobs[i].x || !jobs[i].part || jobs[i].ld_part < jobs[i].layer->pf.N1p ||
            (jobs[i].ld_part & 3) || ((uintptr_t)jobs[i].part & 15))
            return LB_ERR_INVALID_ARG;
        if (jobs[i].layer->d.K % 8) return LB_ERR_UNSUPPORTED;
    }
    if (!*state) {
        PfJobState *st = new (std::nothrow) PfJobState();
        if (!st) return LB_ERR_OOM;
        st->n = n;
        if (cudaMalloc(&st->maps, sizeof(CUtensorMap) * n) != cudaSuccess ||
            cudaMalloc(&st->rec, sizeof(PfLayer) * n) != cudaSuccess ||
            cudaMalloc(&st->starts, sizeof(int) * (n + 1)) != cudaSuccess ||
            cudaMalloc(&st->err, sizeof(int)) != cudaSuccess || cudaMemsetAsync(st->err, 0, sizeof(int), s) != cudaSuccess) {
            prefill_jobs_free(st);
            return LB_ERR_OOM;
        }
        *state = st;
    }
    PfJobState &st = **state;
    if (st.n != n) return LB_ERR_INVALID_ARG;
    bool dirty = st.lastM != M || (int)st.lastX.size() != n;
    for (int i = 0; i < n && !dirty; ++i)
        dirty = st.lastX[i] != jobs[i].x || st.lastPart[i] != jobs[i].part || st.lastF16[i] != (int)jobs[i].a_f16;
    const int sms = sm_count();
    if (dirty) {
        // longest contraction first: the round-robin deal then starts with the long units
        std::vector<int> ord(n);
        for (int i = 0; i < n; ++i) ord[i] = i;
        std::stable_sort(ord.begin(), ord.end(),
                         [&](int a, int b) { return jobs[a].layer->pf.KB1 > jobs[b].layer->pf.KB1; });
        const int mtiles = ceil_div(M, kPfBM);
        std::vector<int> tiles(n), nk(n);
        for (int q = 0; q < n; ++q) {
            const PfWeights &W = jobs[ord[q]].layer->pf;
            tiles[q] = mtiles * ceil_div(W.N1p, kPfBN);
            nk[q] = W.KB1;
        }
        const std::vector<int> split = choose_splits(tiles, nk, sms);
        std::vector<CUtensorMap> maps(n);
        std::vector<PfLayer> rec(n);
        std::vector<int> starts(n + 1, 0);
        for (int q = 0; q < n; ++q) {
            const PfLatentJob &j = jobs[ord[q]];
            const LayerDev &d = j.layer->d;
            const PfWeights &W = j.layer->pf;
            if (!encode_2d(&maps[q], j.a_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, j.x,
                           d.K, M))
                return LB_ERR_UNSUPPORTED;
            PfLayer &a = rec[q];
            a.tmA = st.maps + q;
            a.tmY = nullptr;
            a.bits = W.b1;
            a.base = W.g64;
            a.lcat = W.lcat;
            a.out = nullptr;
            a.nk = W.KB1;
            a.ncols = W.N1p;
            a.ld_out = W.K2;
            a.ntn = ceil_div(W.N1p, kPfBN);
            a.r8 = W.r8;
            a.base_ld = W.K64;
            a.npaths = d.npaths;
            a.a_f16 = j.a_f16;
            a.ksplit = split[q];
            a.part = j.part;
            a.ld_part = j.ld_part;
            a.oscale = nullptr;
            starts[q + 1] = starts[q] + tiles[q] * split[q];
        }
        if ((e = cudaMemcpyAsync(st.maps, maps.data(), sizeof(CUtensorMap) * n, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
            (e = cudaMemcpyAsync(st.rec, rec.data(), sizeof(PfLayer) * n, cudaMemcpyHostToDevice, s)) != cudaSuccess ||
            (e = cudaMemcpyAsync(st.starts, starts.data(), sizeof(int) * (n + 1), cudaMemcpyHostToDevice, s)) !=
                cudaSuccess ||
            (e = cudaStreamSynchronize(s)) != cudaSuccess)
            return status_from(e);
        st.total = starts[n];
        st.lastM = M;
        st.lastX.assign(n, nullptr);
        st.lastPart.assign(n, nullptr);
        st.lastF16.assign(n, 0);
        for (int i = 0; i < n; ++i) {
            st.lastX[i] = jobs[i].x;
            st.lastPart[i] = jobs[i].part;
            st.lastF16[i] = jobs[i].a_f16;
        }
    }
    const size_t smem = smem_bytes(n);
    if ((e = ensure_smem(smem)) != cudaSuccess) return smem > 232448 ? LB_ERR_UNSUPPORTED : status_from(e);
    const int grid = std::max(1, std::min(st.total, sms));
    prefill_kernel<0><<<grid, pf_threads(0), smem, s>>>(st.rec, st.starts, n, M, st.err);
    ++*launches;
    return status_from(cudaGetLastError());
}

}  // namespace lb


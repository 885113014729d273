// Fused small-batch (decode, M <= 16) forward of LittleBit layers.
//
// The notes page of LittleBit (section "Multi-scale compensation") evaluates
// a path as  x (.) g -> . V_sign -> (.) l -> . U_sign^T -> (.) h  and
// "Residual compensation" sums the primary and residual paths.  Two kernels
// cover every layer of a plan:
//
//   contraction 1 (one work item = one layer x 1024 inputs):
//     t = x (.) g_p for both paths, written as 16-bit fixed point with one
//     power-of-two exponent per (item, path, row) and split into two signed
//     base-256 digits; z-partials = t . V_sign on integer tensor cores, exact
//     in int32.  The last item of a layer to finish (a completion counter,
//     no waiting) sums the partials in a fixed order, applies l, and writes
//     the latent vector as 16-bit fixed-point B fragments for contraction 2.
//   contraction 2 (one work item = one layer x 512 outputs):
//     s_p = zl_p . U_sign,p^T on integer tensor cores, y = sum_p h_p (.) s_p.
//
// A sign s = 1 - 2b (b = stored bit) turns sum_k s_k q_k into
// Qsum - 2 * sum_k b_k q_k, so the tensor cores only ever see {0, 2^i} bytes
// (see the unit layout in lb_internal.cuh).  Rounding happens only when the
// activations enter fixed point (16 significant bits relative to the largest
// magnitude of their block) and in float32 sums; the tolerance budget is in
// the design notes.

#include <cfloat>

#include "lb_internal.cuh"

namespace lb {

__device__ __forceinline__ int exponent_for(float amax, bool nonfinite)
{
    // Largest E with amax * 2^E <= 32639, so that q = rint(t * 2^E) splits into
    // two balanced digits in [-128, 127].
    if (nonfinite) return kNanExp;
    if (!(amax > 0.0f)) return 0;
    int e;
    frexpf(amax, &e);                    // amax = f * 2^e, f in [0.5, 1)
    int E = 15 - e;                      // amax * 2^E in [2^14, 2^15)
    if (ldexpf(amax, E) > 32639.0f) E -= 1;
    return E;
}

__device__ __forceinline__ int quantize(float t, int E)
{
    return (E == kNanExp) ? 0 : __float2int_rn(ldexpf(t, E));
}

// low digit in [-128, 127] and high digit, q = 256 * hi + lo
__device__ __forceinline__ void digits(int q, int &lo, int &hi)
{
    lo = ((q + 128) & 255) - 128;
    hi = (q - lo) >> 8;
}

// Where the two digit words of activation row m, k-group (4 consecutive k
// starting at kk within a 32-wide k-block) live among the 32 lanes' B
// fragments of m16n8k32: column g = 2 * (m % 4) + digit, lane = 4 * g + t,
// word (kk / 16), with t = (kk % 16) / 4.
__device__ __forceinline__ void frag_slot(int m, int kk, int &lane_lo, int &lane_hi, int &word)
{
    const int mm = m & 3;
    const int t = (kk & 15) >> 2;
    word = kk >> 4;
    lane_lo = (2 * mm) * 4 + t;
    lane_hi = (2 * mm + 1) * 4 + t;
}

__device__ __forceinline__ void set_word(uint2 &u, int word, uint32_t v)
{
    if (word) u.y = v; else u.x = v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum(int v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Per-thread contribution (no shuffles: callers may be divergent).
__device__ __forceinline__ int warp_sum_partial(int v, int) { return v; }

__device__ __forceinline__ int warp_or(int v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// Shared helpers of both kernels
// ---------------------------------------------------------------------------
__device__ __forceinline__ void copy_desc(LayerDev &dst, const LayerDev *src)
{
    static_assert(sizeof(LayerDev) % 4 == 0, "descriptor is copied as words");
    for (int i = threadIdx.x; i < (int)(sizeof(LayerDev) / 4); i += blockDim.x)
        reinterpret_cast<int *>(&dst)[i] = reinterpret_cast<const int *>(src)[i];
}

// non-negative floats order like their bit patterns
__device__ __forceinline__ void smem_max(float *a, float v) { atomicMax((int *)a, __float_as_int(v)); }

// ---------------------------------------------------------------------------
// Finish contraction 1 of one layer (run by the last of its items):
// z = sum over chunks (fixed order), zl = z (.) l, zl as B fragments for
// contraction 2.  Also returns the integer partials to zero for the next call.
// ---------------------------------------------------------------------------
__device__ void finish_latent(const LayerDev &d, int M, int NT, int *sE, int *sQs, float *sMax, int *sBad)
{
    const int tid = threadIdx.x, lane = tid & 31;
    const int T = blockDim.x;
    if (tid < 32) {
        sMax[tid] = 0.0f;
        sBad[tid] = 0;
        sQs[tid] = 0;
    }
    __syncthreads();
    const int rows = d.npaths * d.r16;
    for (int e = tid; e < rows * M; e += T) {
        const int jr = e / M, m = e - jr * M;
        const int p = jr / d.r16, j = jr - p * d.r16;
        float z = 0.0f;
        int kc = 0;
        for (; kc + 4 <= d.nkc; kc += 4) {
            int2 mt[4];
            int tv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                mt[u] = __ldcg(&d.pmeta[((kc + u) * 2 + p) * 16 + m]);
                tv[u] = __ldcg(&d.partT[((size_t)(kc + u) * d.R1 + jr) * 16 + m]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                z += (mt[u].x == kNanExp) ? __int_as_float(0x7fc00000)
                                          : ldexpf((float)(mt[u].y - 2 * tv[u]), -mt[u].x);
        }
        for (; kc < d.nkc; ++kc) {
            const int2 mt = __ldcg(&d.pmeta[(kc * 2 + p) * 16 + m]);
            const int tv = __ldcg(&d.partT[((size_t)kc * d.R1 + jr) * 16 + m]);
            z += (mt.x == kNanExp) ? __int_as_float(0x7fc00000) : ldexpf((float)(mt.y - 2 * tv), -mt.x);
        }
        const float zl = (j < d.r) ? z * __half2float(d.l[p * d.r16 + j]) : 0.0f;
        d.zl[(size_t)jr * 16 + m] = zl;
        if (!(fabsf(zl) <= FLT_MAX)) atomicOr(&sBad[p * 16 + m], 1);
        else smem_max(&sMax[p * 16 + m], fabsf(zl));
    }
    __syncthreads();
    // integer partials back to zero (every row, including padding rows)
    for (size_t e = tid; e < (size_t)d.nkc * d.R1 * 16; e += T) d.partT[e] = 0;
    if (tid < d.npaths * M) {
        const int p = tid / M, m = tid - p * M;
        sE[p * 16 + m] = exponent_for(sMax[p * 16 + m], sBad[p * 16 + m] != 0);
    }
    __syncthreads();
    // digits into fragments; rows m in [M, 4*NT) get zero digits
    const int MT = 4 * NT;
    const int ngrp = d.r32 / 4;
    for (int e = tid; e < d.npaths * MT * ngrp; e += T) {
        const int c = e % ngrp;
        const int pm = e / ngrp;
        const int p = pm / MT, m = pm - p * MT;
        uint32_t wlo = 0, whi = 0;
        int qs = 0;
        if (m < M) {
            const int E = sE[p * 16 + m];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = 4 * c + u;
                const float zl = (j < d.r) ? d.zl[(size_t)(p * d.r16 + j) * 16 + m] : 0.0f;
                const int q = (j < d.r) ? quantize(zl, E) : 0;
                int lo, hi;
                digits(q, lo, hi);
                wlo |= (uint32_t)(lo & 255) << (8 * u);
                whi |= (uint32_t)(hi & 255) << (8 * u);
                qs += q;
            }
        }
        const int jj = p * d.r32 + 4 * c;
        int llo, lhi, word;
        frag_slot(m, jj & 31, llo, lhi, word);
        uint2 *fb = d.zfrag + ((size_t)(m >> 2) * d.KB2 + (jj >> 5)) * 32;
        set_word(fb[llo], word, wlo);
        set_word(fb[lhi], word, whi);
        if (m < M) {
            qs = warp_sum_partial(qs, lane);
            if (qs) atomicAdd(&sQs[p * 16 + m], qs);
        }
    }
    __syncthreads();
    if (tid < d.npaths * M) {
        const int p = tid / M, m = tid - p * M;
        d.zmeta[p * 16 + m] = make_int2(sE[p * 16 + m], sQs[p * 16 + m]);
    }
}

// ---------------------------------------------------------------------------
// Contraction 1
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kDecodeThreads)
    contraction1_kernel(const LayerDev *__restrict__ layers, const P1Item *__restrict__ items,
                        int nitems, const __grid_constant__ IoPtrs io, int base, int M)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint2 *sB = (uint2 *)smem_raw;              // [2][kP1ChunkKB][NT][32]
    __shared__ LayerDev sd;
    __shared__ float sMax[32];
    __shared__ int sBad[32], sE[32], sQs[32];
    __shared__ int sLast;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kDecodeThreads / 32;
    const int g = lane >> 2, t4 = lane & 3;

    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
        const P1Item item = items[it];
        __syncthreads();                    // previous item fully done with shared state
        copy_desc(sd, layers + item.layer);
        {
            uint4 *z4 = (uint4 *)sB;
            const int n16 = 2 * kP1ChunkKB * NT * 32 * (int)sizeof(uint2) / 16;
            for (int i = tid; i < n16; i += kDecodeThreads) z4[i] = make_uint4(0, 0, 0, 0);
        }
        if (tid < 32) {
            sMax[tid] = 0.0f;
            sBad[tid] = 0;
            sQs[tid] = 0;
        }
        __syncthreads();
        const LayerDev &d = sd;
        const uint16_t *__restrict__ x = io.x[item.layer - base];
        const int kc = item.kc;
        const int kb0 = kc * kP1ChunkKB;
        const int nkb = min(kP1ChunkKB, d.KB1 - kb0);
        const int k0 = kb0 * kKPerBlock;
        const int klen = nkb * kKPerBlock;

        // ---- t = x (.) g for 8 consecutive inputs per thread: largest magnitude per (path, m)
        const int kk0 = 8 * tid;
        const bool act = kk0 < klen;
        const int kg = k0 + kk0;
        float gv[2][8];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            if (act && p < d.npaths) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(d.g + (size_t)p * d.K32 + kg));
                const __half *hv = reinterpret_cast<const __half *>(&raw);
#pragma unroll
                for (int e = 0; e < 8; ++e) gv[p][e] = __half2float(hv[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gv[p][e] = 0.0f;
            }
        }
        const bool vec = ((d.K & 7) == 0) && (kg + 8 <= d.K);
        auto load_x = [&](int m, float (&xv)[8]) {
            if (!act) {
#pragma unroll
                for (int e = 0; e < 8; ++e) xv[e] = 0.0f;
            } else if (vec) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)m * d.K + kg));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xv[2 * e] = __uint_as_float(w4[e] << 16);
                    xv[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    xv[e] = (kg + e < d.K) ? bf16_bits_to_float(__ldg(x + (size_t)m * d.K + kg + e)) : 0.0f;
            }
        };
        for (int m = 0; m < M; ++m) {
            float xv[8];
            load_x(m, xv);
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float amax = 0.0f;
                int bad = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float tv = fabsf(xv[e] * gv[p][e]);
                    if (!(tv <= FLT_MAX)) bad = 1;
                    else amax = fmaxf(amax, tv);
                }
                amax = warp_max(amax);
                bad = warp_or(bad);
                if (lane == 0 && p < d.npaths) {
                    smem_max(&sMax[p * 16 + m], amax);
                    if (bad) atomicOr(&sBad[p * 16 + m], 1);
                }
            }
        }
        __syncthreads();
        if (tid < d.npaths * M) {
            const int p = tid / M, m = tid - p * M;
            sE[p * 16 + m] = exponent_for(sMax[p * 16 + m], sBad[p * 16 + m] != 0);
        }
        __syncthreads();
        // ---- digits into B fragments, digit sums per (path, m)
        for (int m = 0; m < M; ++m) {
            float xv[8];
            load_x(m, xv);
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                if (p >= d.npaths) continue;
                const int E = sE[p * 16 + m];
                int qs = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t wlo = 0, whi = 0;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q = quantize(xv[4 * h + e] * gv[p][4 * h + e], E);
                        int lo, hi;
                        digits(q, lo, hi);
                        wlo |= (uint32_t)(lo & 255) << (8 * e);
                        whi |= (uint32_t)(hi & 255) << (8 * e);
                        qs += q;
                    }
                    if (act) {
                        const int kk = kk0 + 4 * h;
                        int llo, lhi, word;
                        frag_slot(m, kk & 31, llo, lhi, word);
                        uint2 *fb = sB + (((size_t)p * kP1ChunkKB + (kk >> 5)) * NT + (m >> 2)) * 32;
                        set_word(fb[llo], word, wlo);
                        set_word(fb[lhi], word, whi);
                    }
                }
                qs = warp_sum(qs);
                if (lane == 0 && qs) atomicAdd(&sQs[p * 16 + m], qs);
            }
        }
        __syncthreads();
        if (tid < d.npaths * M) {
            const int p = tid / M, m = tid - p * M;
            d.pmeta[(kc * 2 + p) * 16 + m] = make_int2(sE[p * 16 + m], sQs[p * 16 + m]);
        }

        // ---- main stream: units (row group, k-block) of this chunk, split evenly over the warps
        const int U1 = d.RG1 * nkb;
        const int ub = (int)((long long)U1 * warp / NW), ue = (int)((long long)U1 * (warp + 1) / NW);
        int acc[4][NT][4];
#pragma unroll
        for (int rb = 0; rb < 4; ++rb)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[rb][n][c] = 0;
        int lrg = ub / nkb, lkb = ub - lrg * nkb;     // load cursor
        int prg = lrg, pkb = lkb;                     // process cursor
        int nload = ue - ub, nproc = ue - ub;
        int prb[4];
        auto set_paths = [&](int rg) {
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
                prb[rb] = min((rg * kRowsPerGroup + rb * kRowsPerBlock) / d.r16, d.npaths - 1);
        };
        set_paths(prg);
        auto flush = [&](int rg) {
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int m = 4 * n + t4;
                    if (m < M) {
                        const int Tlo = (acc[rb][n][0] >> rb) + 256 * (acc[rb][n][1] >> rb);
                        const int Thi = (acc[rb][n][2] >> (rb + 4)) + 256 * (acc[rb][n][3] >> (rb + 4));
                        const int row = rg * kRowsPerGroup + rb * kRowsPerBlock + g;
                        if (Tlo) atomicAdd(&d.partT[((size_t)kc * d.R1 + row) * 16 + m], Tlo);
                        if (Thi) atomicAdd(&d.partT[((size_t)kc * d.R1 + row + 8) * 16 + m], Thi);
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[rb][n][c] = 0;
                }
        };
        constexpr int B = 8;
        uint2 bufA[B], bufB[B];
        auto load_batch = [&](uint2 (&buf)[B]) {
#pragma unroll
            for (int i = 0; i < B; ++i) {
                if (nload > 0) {
                    buf[i] = ld_stream_u2(d.vt + ((size_t)lrg * d.KB1 + kb0 + lkb) * 32 + lane);
                    if (++lkb == nkb) { lkb = 0; ++lrg; }
                    --nload;
                }
            }
        };
        auto proc_batch = [&](const uint2 (&buf)[B]) {
#pragma unroll
            for (int i = 0; i < B; ++i) {
                if (nproc > 0) {
                    const uint2 w = buf[i];
                    uint2 bp[2][NT];
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int n = 0; n < NT; ++n)
                            bp[p][n] = sB[(((size_t)p * kP1ChunkKB + pkb) * NT + n) * 32 + lane];
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const uint32_t mlo = 0x01010101u << rb, mhi = 0x01010101u << (rb + 4);
                        const uint32_t a0 = w.x & mlo, a1 = w.x & mhi, a2 = w.y & mlo, a3 = w.y & mhi;
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            const uint2 b = prb[rb] ? bp[1][n] : bp[0][n];
                            mma_u8s8(acc[rb][n], a0, a1, a2, a3, b.x, b.y);
                        }
                    }
                    --nproc;
                    if (++pkb == nkb) {
                        flush(prg);
                        pkb = 0;
                        ++prg;
                        set_paths(prg);
                    }
                }
            }
        };
        load_batch(bufA);
        load_batch(bufB);
        while (nproc > 0) {
            proc_batch(bufA);
            load_batch(bufA);
            proc_batch(bufB);
            load_batch(bufB);
        }
        if (pkb != 0) flush(prg);

        // ---- completion count; the last item of the layer finishes the latent vector
        __threadfence();
        __syncthreads();
        if (tid == 0) sLast = (atomicAdd(d.counter, 1u) == (unsigned)(d.nkc - 1));
        __syncthreads();
        if (sLast) {
            __threadfence();
            finish_latent(d, M, NT, sE, sQs, sMax, sBad);
            __syncthreads();
            if (tid == 0) atomicExch(d.counter, 0u);
        }
    }
}

// ---------------------------------------------------------------------------
// Contraction 2 (+ h, + path sum)
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kDecodeThreads)
    contraction2_kernel(const LayerDev *__restrict__ layers, const P2Item *__restrict__ items,
                        int nitems, const __grid_constant__ IoPtrs io, int base, int M)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint2 *sB = (uint2 *)smem_raw;              // [NT][KB2][32]
    __shared__ LayerDev sd;
    __shared__ int2 sMeta[32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kDecodeThreads / 32;
    const int g = lane >> 2, t4 = lane & 3;

    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
        const P2Item item = items[it];
        __syncthreads();   // previous item's readers of shared state are done
        copy_desc(sd, layers + item.layer);
        __syncthreads();
        const LayerDev &d = sd;
        float *__restrict__ y = io.y[item.layer - base];
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(d.zfrag);
            uint4 *dst = reinterpret_cast<uint4 *>(sB);
            const int n16 = NT * d.KB2 * 32 * (int)sizeof(uint2) / 16;
            for (int i = tid; i < n16; i += kDecodeThreads) dst[i] = __ldcg(src + i);
        }
        if (tid < 32) sMeta[tid] = __ldcg(&d.zmeta[tid]);
        __syncthreads();

        const int kbp = d.r32 / kKPerBlock;   // k-blocks per path
        const int KB2 = d.KB2;
        const int nrg = (item.rg1 - item.rg0 - warp + NW - 1) / NW;   // this warp's row groups
        int nload = max(0, nrg) * KB2, nproc = nload;
        int lrg = item.rg0 + warp, lkb = 0;
        int prg = lrg, pkb = 0;
        int acc[4][NT][4];
        float yv[4][NT][2];
        float hv[2][4][2];
#pragma unroll
        for (int rb = 0; rb < 4; ++rb)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                yv[rb][n][0] = yv[rb][n][1] = 0.0f;
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[rb][n][c] = 0;
            }
        auto load_h = [&](int rg) {
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const int n = rg * kRowsPerGroup + rb * kRowsPerBlock + g;
                    const bool ok = p < d.npaths && rg < item.rg1;
                    hv[p][rb][0] = ok ? __half2float(d.h[p * d.N64 + n]) : 0.0f;
                    hv[p][rb][1] = ok ? __half2float(d.h[p * d.N64 + n + 8]) : 0.0f;
                }
        };
        load_h(prg);
        auto fold = [&](int p) {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int m = 4 * n + t4;
                const int2 meta = (m < M) ? sMeta[p * 16 + m] : make_int2(0, 0);
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const int Tlo = (acc[rb][n][0] >> rb) + 256 * (acc[rb][n][1] >> rb);
                    const int Thi = (acc[rb][n][2] >> (rb + 4)) + 256 * (acc[rb][n][3] >> (rb + 4));
                    float slo, shi;
                    if (meta.x == kNanExp) {
                        slo = shi = __int_as_float(0x7fc00000);
                    } else {
                        slo = ldexpf((float)(meta.y - 2 * Tlo), -meta.x);
                        shi = ldexpf((float)(meta.y - 2 * Thi), -meta.x);
                    }
                    yv[rb][n][0] += (p ? hv[1][rb][0] : hv[0][rb][0]) * slo;
                    yv[rb][n][1] += (p ? hv[1][rb][1] : hv[0][rb][1]) * shi;
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[rb][n][c] = 0;
                }
            }
        };
        auto store = [&](int rg) {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int m = 4 * n + t4;
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const int nlo = rg * kRowsPerGroup + rb * kRowsPerBlock + g;
                    if (m < M) {
                        if (nlo < d.N) y[(size_t)m * d.N + nlo] = yv[rb][n][0];
                        if (nlo + 8 < d.N) y[(size_t)m * d.N + nlo + 8] = yv[rb][n][1];
                    }
                    yv[rb][n][0] = yv[rb][n][1] = 0.0f;
                }
            }
        };
        constexpr int B = 8;
        uint2 bufA[B], bufB[B];
        auto load_batch = [&](uint2 (&buf)[B]) {
#pragma unroll
            for (int i = 0; i < B; ++i) {
                if (nload > 0) {
                    buf[i] = ld_stream_u2(d.ut + ((size_t)lrg * KB2 + lkb) * 32 + lane);
                    if (++lkb == KB2) { lkb = 0; lrg += NW; }
                    --nload;
                }
            }
        };
        auto proc_batch = [&](const uint2 (&buf)[B]) {
#pragma unroll
            for (int i = 0; i < B; ++i) {
                if (nproc > 0) {
                    const uint2 w = buf[i];
                    uint2 b[NT];
#pragma unroll
                    for (int n = 0; n < NT; ++n) b[n] = sB[((size_t)n * KB2 + pkb) * 32 + lane];
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const uint32_t mlo = 0x01010101u << rb, mhi = 0x01010101u << (rb + 4);
                        const uint32_t a0 = w.x & mlo, a1 = w.x & mhi, a2 = w.y & mlo, a3 = w.y & mhi;
#pragma unroll
                        for (int n = 0; n < NT; ++n) mma_u8s8(acc[rb][n], a0, a1, a2, a3, b[n].x, b[n].y);
                    }
                    --nproc;
                    ++pkb;
                    if (pkb % kbp == 0) fold(pkb / kbp - 1);
                    if (pkb == KB2) {
                        store(prg);
                        pkb = 0;
                        prg += NW;
                        load_h(prg);
                    }
                }
            }
        };
        load_batch(bufA);
        load_batch(bufB);
        while (nproc > 0) {
            proc_batch(bufA);
            load_batch(bufA);
            proc_batch(bufB);
            load_batch(bufB);
        }
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct DecodeLaunch {
    void (*k1)(const LayerDev *, const P1Item *, int, const IoPtrs, int, int);
    void (*k2)(const LayerDev *, const P2Item *, int, const IoPtrs, int, int);
    int occ1 = 0, occ2 = 0;
    size_t smem1 = 0, smem2_cap = 0;
    bool ready = false;
};

static DecodeLaunch g_launch[kMaxNT + 1];
static int g_sms = 0;

template <int NT>
static cudaError_t prepare(DecodeLaunch &L)
{
    if (L.ready) return cudaSuccess;
    L.k1 = contraction1_kernel<NT>;
    L.k2 = contraction2_kernel<NT>;
    L.smem1 = (size_t)2 * kP1ChunkKB * NT * 32 * sizeof(uint2);
    // contraction-2 fragments: up to LB_MAX_RANK latent indices per path
    L.smem2_cap = (size_t)(2 * LB_MAX_RANK / kKPerBlock) * NT * 32 * sizeof(uint2);
    cudaError_t e = cudaFuncSetAttribute(L.k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(L.k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem2_cap);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&L.occ1, L.k1, kDecodeThreads, L.smem1);
    if (e != cudaSuccess) return e;
    L.ready = true;
    return cudaSuccess;
}

lb_status decode_forward(const Plan &P, const uint16_t *const *xs, float *const *ys, int M,
                         cudaStream_t s, int *launches)
{
    *launches = 0;
    if (M > kMaxDecodeM) {
        // Rows beyond the decode limit run as consecutive blocks of 16 rows.
        std::vector<const uint16_t *> xc(P.n);
        std::vector<float *> yc(P.n);
        for (int m0 = 0; m0 < M; m0 += kMaxDecodeM) {
            for (int i = 0; i < P.n; ++i) {
                xc[i] = xs[i] + (size_t)m0 * P.host[i].K;
                yc[i] = ys[i] + (size_t)m0 * P.host[i].N;
            }
            int l = 0;
            lb_status st = decode_forward(P, xc.data(), yc.data(), std::min(kMaxDecodeM, M - m0), s, &l);
            *launches += l;
            if (st != LB_OK) return st;
        }
        return LB_OK;
    }
    const int NT = (M + 3) / 4;
    cudaError_t e = cudaSuccess;
    if (!g_sms) {
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return status_from(e);
        if ((e = cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return status_from(e);
    }
    DecodeLaunch &L = g_launch[NT];
    switch (NT) {
    case 1: e = prepare<1>(L); break;
    case 2: e = prepare<2>(L); break;
    case 3: e = prepare<3>(L); break;
    default: e = prepare<4>(L); break;
    }
    if (e != cudaSuccess) return status_from(e);

    int maxKB2 = 0;
    for (const LayerDev &d : P.host) maxKB2 = std::max(maxKB2, d.KB2);
    const size_t smem2 = (size_t)maxKB2 * NT * 32 * sizeof(uint2);
    int occ2 = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ2, L.k2, kDecodeThreads, smem2)) != cudaSuccess)
        return status_from(e);
    occ2 = std::max(1, occ2);
    const int occ1 = std::max(1, L.occ1);

    static thread_local IoPtrs io;
    profile_mark(0, s);
    const int nb = (int)P.p1_start.size() - 1;
    for (int b = 0; b < nb; ++b) {
        const int base = b * kIoBatch;
        const int cnt = std::min(kIoBatch, P.n - base);
        for (int i = 0; i < cnt; ++i) {
            io.x[i] = xs[base + i];
            io.y[i] = ys[base + i];
        }
        const int n1 = P.p1_start[b + 1] - P.p1_start[b];
        const int n2 = P.p2_start[b + 1] - P.p2_start[b];
        const int grid1 = std::max(1, std::min(n1, g_sms * occ1));
        const int grid2 = std::max(1, std::min(n2, g_sms * occ2));
        L.k1<<<grid1, kDecodeThreads, L.smem1, s>>>(P.dev, P.p1 + P.p1_start[b], n1, io, base, M);
        profile_mark(++*launches, s);
        L.k2<<<grid2, kDecodeThreads, smem2, s>>>(P.dev, P.p2 + P.p2_start[b], n2, io, base, M);
        profile_mark(++*launches, s);
    }
    e = cudaGetLastError();
    return status_from(e);
}

}  // namespace lb

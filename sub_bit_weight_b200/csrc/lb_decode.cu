// Fused small-batch (decode, M <= 16) forward of LittleBit layers.
//
// The notes page of LittleBit (section "Multi-scale compensation") evaluates
// a path as  x (.) g -> . V_sign -> (.) l -> . U_sign^T -> (.) h  and
// "Residual compensation" sums the primary and residual paths.  Three kernels
// cover every layer of a plan (a stack), one launch each:
//
//   contraction 1 (work item = one layer x 1024 inputs):
//     t = x (.) g_p for both paths in 16-bit fixed point (one power-of-two
//     exponent E per item, path and activation row; two signed base-256
//     digits), then sum_k b[k][j] * t[k] on integer tensor cores (exact in
//     int32, b = stored sign bit).  Each item adds 2^-E times its integer
//     results into float64 accumulators: sum_k b*t per latent row and sum_k t
//     per path.  Those terms are integers below 2^26 times powers of two, so
//     the float64 sums are exact (hence independent of arrival order) as long
//     as the chunks' exponents lie within ~26 of each other.
//   finish (one CTA per layer, its own launch): z = sum_k t - 2 * sum_k b*t
//     (a sign is s = 1 - 2b), zl = z (.) l, written as 16-bit fixed-point B
//     fragments for contraction 2; the accumulators are cleared for the next
//     call.
//   contraction 2 (work item = one layer x 512 outputs):
//     s = zl . U_sign^T on integer tensor cores, y = sum_p h_p (.) s_p.
//
// Weights stream through a small ring of shared-memory buffers per warp,
// filled by bulk asynchronous copies (cp.async.bulk) that complete on an
// mbarrier; every wait is bounded and reports a timeout instead of hanging.

#include "lb_decode_common.cuh"

namespace lb {

// ---------------------------------------------------------------------------
// Finish of contraction 1 for one layer (run by its last item)
// ---------------------------------------------------------------------------
template <int NT>
__device__ void finish_latent(const LayerDev *dp, int M, float *sMax, int *sBad, int *sE, int *sQs)
{
    const int tid = threadIdx.x;
    const int R1 = dp->R1, r = dp->r, r16 = dp->r16, r32 = dp->r32, npaths = dp->npaths, KB2 = dp->KB2;
    double *acc = dp->acc;
    const __half *lsc = dp->l;
    const double *S = acc + (size_t)R1 * 16;
    const int *badf = reinterpret_cast<const int *>(acc + (size_t)R1 * 16 + 32);
    if (tid < 32) {
        sMax[tid] = 0.0f;
        sBad[tid] = 0;
        sQs[tid] = 0;
    }
    __syncthreads();
    auto zl_at = [&](int p, int j, int m) -> float {
        const double z = __ldcg(S + p * 16 + m) - 2.0 * __ldcg(acc + (size_t)(p * r16 + j) * 16 + m);
        return (float)z * __half2float(lsc[p * r16 + j]);
    };
    for (int e = tid; e < npaths * r * M; e += (int)blockDim.x) {
        const int m = e % M, pj = e / M;
        const int p = pj / r, j = pj - p * r;
        const float zl = zl_at(p, j, m);
        if (!(fabsf(zl) <= FLT_MAX)) atomicOr(&sBad[p * 16 + m], 1);
        else smem_max(&sMax[p * 16 + m], fabsf(zl));
    }
    __syncthreads();
    if (tid < npaths * M) {
        const int p = tid / M, m = tid - p * M;
        sE[p * 16 + m] = exponent_for(sMax[p * 16 + m], sBad[p * 16 + m] != 0 || __ldcg(badf + p * 16 + m) != 0);
    }
    __syncthreads();
    // digits into the fragments of this call's n-tiles (rows m in [M, 4*NT) get zeros)
    const int MT = 4 * NT, ngrp = r32 / 4;
    for (int e = tid; e < npaths * MT * ngrp; e += (int)blockDim.x) {
        const int c = e % ngrp, pm = e / ngrp;
        const int p = pm / MT, m = pm - p * MT;
        uint32_t wlo = 0, whi = 0;
        int qs = 0;
        if (m < M) {
            const int E = sE[p * 16 + m];
            const float sc = (E == kNanExp) ? 0.0f : pow2f(E);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = 4 * c + u;
                const int q = (j < r) ? quantize_s(zl_at(p, j, m), sc) : 0;
                int lo, hi;
                digits(q, lo, hi);
                wlo |= (uint32_t)(lo & 255) << (8 * u);
                whi |= (uint32_t)(hi & 255) << (8 * u);
                qs += q;
            }
            if (qs) atomicAdd(&sQs[p * 16 + m], qs);
        }
        const int jj = p * r32 + 4 * c;
        int llo, lhi, word;
        frag_slot(m, jj & 31, llo, lhi, word);
        uint2 *fb = dp->zfrag + ((size_t)(m >> 2) * KB2 + (jj >> 5)) * 32;
        set_word(fb[llo], word, wlo);
        set_word(fb[lhi], word, whi);
    }
    __syncthreads();
    if (tid < npaths * M) {
        const int p = tid / M, m = tid - p * M;
        dp->zmeta[p * 16 + m] = make_int2(sE[p * 16 + m], sQs[p * 16 + m]);
    }
    // accumulators back to zero for the next call
    for (int i = tid; i < (int)acc_doubles(R1); i += (int)blockDim.x) acc[i] = 0.0;
}

// One CTA per layer of the batch (layer base + blockIdx.x), after contraction 1.
constexpr int kFinishGeneralThreads = 1024;
template <int NT>
__global__ void __launch_bounds__(kFinishGeneralThreads) finish_general_kernel(const LayerDev *__restrict__ layers,
                                                                               int base, int M)
{
    __shared__ float sMax[32];
    __shared__ int sBad[32], sE[32], sQs[32];
    finish_latent<NT>(layers + base + blockIdx.x, M, sMax, sBad, sE, sQs);
}

// ---------------------------------------------------------------------------
// Contraction 1
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kDecodeThreads)
    contraction1_kernel(const LayerDev *__restrict__ layers, const P1Item *__restrict__ items, int nitems,
                        const __grid_constant__ IoPtrs io, int base, int M, int *err)
{
    constexpr int NW = kDecodeThreads / 32;
    constexpr int kHalf = kP1StageKB;                        // k-blocks per ring stage
    constexpr int kStage = kHalf * 256;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *ring = smem_raw;                          // [NW][kP1Stages][kStage]
    uint2 *sB = (uint2 *)(smem_raw + NW * kP1Stages * kStage);   // [2][kP1ChunkKB][NT][32]
    __shared__ uint64_t bars[NW][kP1Stages];
    __shared__ float sMax[32];
    __shared__ int sBad[32], sE[32], sQs[32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    if (lane == 0)
        for (int s = 0; s < kP1Stages; ++s) bar_init(&bars[warp][s]);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncwarp();
    uint32_t issued = 0, consumed = 0;   // this warp's ring sequence numbers
    unsigned char *my_ring = ring + warp * kP1Stages * kStage;

    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
        const P1Item item = items[it];
        const LayerDev *dp = layers + item.layer;
        const int K = dp->K, K32 = dp->K32, KB1 = dp->KB1, KB1e = dp->KB1e, RG1 = dp->RG1, r16 = dp->r16,
                  npaths = dp->npaths;
        const uint2 *__restrict__ vt = dp->vt;
        const __half *__restrict__ gsc = dp->g;
        double *__restrict__ acc = dp->acc;
        const uint16_t *__restrict__ x = io.x[item.layer - base];
        const int kc = item.kc;
        const int kb0 = kc * kP1ChunkKB;
        const int nkb = min(kP1ChunkKB, KB1 - kb0);
        const int k0 = kb0 * kKPerBlock;
        const int klen = nkb * kKPerBlock;
        const int hp = (nkb + kHalf - 1) / kHalf;                // ring stages per row group
        const int nmine = (RG1 - warp + NW - 1) / NW;           // this warp's row groups
        const int nseq = max(0, nmine) * hp;
        auto fill = [&](int q) {   // sequence entry q -> (row group, half)
            const int rg = warp + NW * (q / hp), h = q % hp;
            const int n = min(kHalf, nkb - h * kHalf);
            const int st = issued % kP1Stages;
            // k-blocks come in pairs: an odd last stage also brings the (empty) padding k-block
            ring_fill(my_ring + st * kStage, vt + ((size_t)rg * KB1e + kb0 + h * kHalf) * 32,
                      (unsigned)((n + 1) & ~1) * 256u, &bars[warp][st]);
            ++issued;
        };

        // start streaming this warp's first stages while the activations are prepared
        if (lane == 0)
            for (int q = 0; q < min(kP1Stages, nseq); ++q) fill(q);

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

        // ---- t = x (.) g for 8 consecutive inputs per thread; largest magnitude per (path, m)
        const int kk0 = 8 * tid;
        const bool act = kk0 < klen;
        const int kg = k0 + kk0;
        float gv[2][8];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            if (act && p < npaths) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(gsc + (size_t)p * K32 + kg));
                const __half *hv = reinterpret_cast<const __half *>(&raw);
#pragma unroll
                for (int e = 0; e < 8; ++e) gv[p][e] = __half2float(hv[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gv[p][e] = 0.0f;
            }
        }
        const bool vec = ((K & 7) == 0) && (kg + 8 <= K);
        // the rows' 8 activations each, all loads in flight together (the loops over m below are unrolled)
        uint4 xr[kMaxDecodeM];
#pragma unroll
        for (int m = 0; m < kMaxDecodeM; ++m)
            xr[m] = (m < M && act && vec) ? __ldg(reinterpret_cast<const uint4 *>(x + (size_t)m * K + kg))
                                          : make_uint4(0u, 0u, 0u, 0u);
        auto load_x = [&](int m, float (&xv)[8]) {
            if (!act) {
#pragma unroll
                for (int e = 0; e < 8; ++e) xv[e] = 0.0f;
            } else if (vec) {
                const uint4 raw = xr[m];
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xv[2 * e] = __uint_as_float(w4[e] << 16);
                    xv[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    xv[e] = (kg + e < K) ? bf16_bits_to_float(__ldg(x + (size_t)m * K + kg + e)) : 0.0f;
            }
        };
#pragma unroll
        for (int m = 0; m < kMaxDecodeM; ++m) {
            if (m >= M) break;
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
                if (lane == 0 && p < npaths) {
                    smem_max(&sMax[p * 16 + m], amax);
                    if (bad) atomicOr(&sBad[p * 16 + m], 1);
                }
            }
        }
        __syncthreads();
        if (tid < npaths * M) {
            const int p = tid / M, m = tid - p * M;
            sE[p * 16 + m] = exponent_for(sMax[p * 16 + m], sBad[p * 16 + m] != 0);
        }
        __syncthreads();
        // ---- digits into B fragments, digit sums per (path, m)
#pragma unroll
        for (int m = 0; m < kMaxDecodeM; ++m) {
            if (m >= M) break;
            float xv[8];
            load_x(m, xv);
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                if (p >= npaths) continue;
                const int E = sE[p * 16 + m];
                const float sc = (E == kNanExp) ? 0.0f : pow2f(E);
                int qs = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t wlo = 0, whi = 0;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q = quantize_s(xv[4 * h + e] * gv[p][4 * h + e], sc);
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
        // sum over this chunk of t (per path, row m), and non-finite flags
        if (tid < npaths * M) {
            const int p = tid / M, m = tid - p * M;
            const int E = sE[p * 16 + m];
            if (E == kNanExp) atomicOr(reinterpret_cast<int *>(acc + (size_t)dp->R1 * 16 + 32) + p * 16 + m, 1);
            else if (sQs[p * 16 + m]) atomicAdd(acc + (size_t)dp->R1 * 16 + p * 16 + m, (double)sQs[p * 16 + m] * pow2d(-E));
        }

        // ---- main stream: this warp's row groups of 64 latent rows, half a chunk per stage
        for (int rgi = 0; rgi < nmine; ++rgi) {
            const int rg = warp + NW * rgi;
            int prb[4];
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
                prb[rb] = min((rg * kRowsPerGroup + rb * kRowsPerBlock) / r16, npaths - 1);
            int a4[4][NT][4];
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int c = 0; c < 4; ++c) a4[rb][n][c] = 0;
            for (int h = 0; h < hp; ++h) {
                const int st = consumed % kP1Stages;
                const uint32_t ph = (consumed / kP1Stages) & 1;
                if (!ring_wait(&bars[warp][st], ph, err)) return;
                ++consumed;
                const uint32_t src = sm_addr(my_ring + st * kStage) + lane * 16;   // pairs of k-blocks
                const uint32_t bbase = sm_addr(sB) + lane * 8;
                const int kbA = h * kHalf, n = min(kHalf, nkb - kbA);
#pragma unroll 4
                for (int u = 0; u < n; ++u) {
                    const int kb = kbA + u;
                    const uint2 w = lds64(src + (u >> 1) * 512 + (u & 1) * 8);
                    uint2 bp[2][NT];
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int nn = 0; nn < NT; ++nn)
                            bp[p][nn] = lds64(bbase + (uint32_t)(((p * kP1ChunkKB + kb) * NT + nn) * 256));
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const uint32_t mlo = 0x01010101u << rb, mhi = 0x01010101u << (rb + 4);
                        const uint32_t a0 = w.x & mlo, a1 = w.x & mhi, a2 = w.y & mlo, a3 = w.y & mhi;
#pragma unroll
                        for (int nn = 0; nn < NT; ++nn) {
                            const uint2 b = prb[rb] ? bp[1][nn] : bp[0][nn];
                            mma_u8s8(a4[rb][nn], a0, a1, a2, a3, b.x, b.y);
                        }
                    }
                }
                // stage consumed: refill it with the entry kP1Stages ahead
                __syncwarp();
                if (lane == 0) {
                    const int q = rgi * hp + h + kP1Stages;
                    if (q < nseq) {
                        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                        fill(q);
                    }
                }
            }
            // sum_k b * t for rows g (scale 2^rb) and g + 8 (scale 2^(rb+4)), times 2^-E
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int m = 4 * n + t4;
                    if (m < M) {
                        const int E = sE[prb[rb] * 16 + m];
                        if (E == kNanExp) continue;
                        const double sc = pow2d(-E);
                        const int Tlo = (a4[rb][n][0] >> rb) + 256 * (a4[rb][n][1] >> rb);
                        const int Thi = (a4[rb][n][2] >> (rb + 4)) + 256 * (a4[rb][n][3] >> (rb + 4));
                        const int row = rg * kRowsPerGroup + rb * kRowsPerBlock + g;
                        if (Tlo) atomicAdd(acc + (size_t)row * 16 + m, (double)Tlo * sc);
                        if (Thi) atomicAdd(acc + (size_t)(row + 8) * 16 + m, (double)Thi * sc);
                    }
                }
        }

        __syncthreads();   // shared state is rebuilt by the next item
    }
}

// ---------------------------------------------------------------------------
// Contraction 2 (+ l, + h, + path sum)
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kDecodeThreads)
    contraction2_kernel(const LayerDev *__restrict__ layers, const P2Item *__restrict__ items, int nitems,
                        const __grid_constant__ IoPtrs io, int base, int M, int kb2max, int *err)
{
    constexpr int NW = kDecodeThreads / 32;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int kStage = ((kb2max + 1) & ~1) * 256;                           // a row group's KB2e k-blocks
    unsigned char *ring = smem_raw;                                          // [NW][kP2Stages][kStage]
    uint2 *sB = (uint2 *)(smem_raw + (size_t)NW * kP2Stages * kStage);      // [NT][KB2][32]
    __shared__ uint64_t bars[NW][kP2Stages];
    __shared__ uint64_t fbar;                    // the layer's zl fragments, one bulk copy per item
    __shared__ int sE[32], sQs[32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    if (lane == 0)
        for (int s = 0; s < kP2Stages; ++s) bar_init(&bars[warp][s]);
    if (tid == 0) bar_init(&fbar);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncthreads();
    uint32_t issued = 0, consumed = 0, nitem = 0;
    unsigned char *my_ring = ring + (size_t)warp * kP2Stages * kStage;

    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
        const P2Item item = items[it];
        const LayerDev *dp = layers + item.layer;
        const int N = dp->N, N64 = dp->N64, KB2 = dp->KB2, KB2e = dp->KB2e, r32 = dp->r32;
        const int npaths = dp->npaths;
        const uint2 *__restrict__ ut = dp->ut;
        const __half *__restrict__ hsc = dp->h;
        float *__restrict__ y = io.y[item.layer - base];
        const unsigned stage_bytes = (unsigned)KB2e * 256u;

        if (lane == 0)
            for (int s = 0; s < kP2Stages; ++s) {
                const int rg = item.rg0 + warp + NW * s;
                if (rg < item.rg1) {
                    const int st = issued % kP2Stages;
                    ring_fill(my_ring + (size_t)st * kStage, ut + (size_t)rg * KB2e * 32, stage_bytes, &bars[warp][st]);
                    ++issued;
                }
            }
        // the previous item's reads of sB are done (barrier at its end): one bulk copy brings this layer's fragments
        if (tid == 0) {
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            ring_fill(sB, dp->zfrag, (unsigned)(NT * KB2 * 32 * sizeof(uint2)), &fbar);
        }
        if (tid < 32) {
            const int2 mt = __ldcg(&dp->zmeta[tid]);
            sE[tid] = mt.x;
            sQs[tid] = mt.y;
        }
        if (!ring_wait(&fbar, nitem & 1, err)) return;
        ++nitem;
        __syncthreads();

        // ---- main stream: this warp's row groups of 64 outputs
        const int kbp = r32 / kKPerBlock;
        for (int rg = item.rg0 + warp; rg < item.rg1; rg += NW) {
            const int st = consumed % kP2Stages;
            const uint32_t ph = (consumed / kP2Stages) & 1;
            float hv[2][4][2];
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const int n = rg * kRowsPerGroup + rb * kRowsPerBlock + g;
                    hv[p][rb][0] = (p < npaths) ? __half2float(hsc[p * N64 + n]) : 0.0f;
                    hv[p][rb][1] = (p < npaths) ? __half2float(hsc[p * N64 + n + 8]) : 0.0f;
                }
            if (!ring_wait(&bars[warp][st], ph, err)) return;
            ++consumed;
            const uint32_t src = sm_addr(my_ring + (size_t)st * kStage) + lane * 16;   // pairs of k-blocks
            const uint32_t bbase = sm_addr(sB) + lane * 8;
            float yv[4][NT][2];
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                for (int n = 0; n < NT; ++n) yv[rb][n][0] = yv[rb][n][1] = 0.0f;
            for (int p = 0; p < npaths; ++p) {
                int a4[4][NT][4];
#pragma unroll
                for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int c = 0; c < 4; ++c) a4[rb][n][c] = 0;
#pragma unroll 4
                for (int kb = p * kbp; kb < (p + 1) * kbp; ++kb) {
                    const uint2 w = lds64(src + (kb >> 1) * 512 + (kb & 1) * 8);
                    uint2 b[NT];
#pragma unroll
                    for (int n = 0; n < NT; ++n) b[n] = lds64(bbase + (uint32_t)((n * KB2 + kb) * 256));
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const uint32_t mlo = 0x01010101u << rb, mhi = 0x01010101u << (rb + 4);
                        const uint32_t a0 = w.x & mlo, a1 = w.x & mhi, a2 = w.y & mlo, a3 = w.y & mhi;
#pragma unroll
                        for (int n = 0; n < NT; ++n) mma_u8s8(a4[rb][n], a0, a1, a2, a3, b[n].x, b[n].y);
                    }
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int m = 4 * n + t4;
                    const int E = (m < M) ? sE[p * 16 + m] : 0;
                    const int Q = (m < M) ? sQs[p * 16 + m] : 0;
                    const float sc = (E == kNanExp) ? __int_as_float(0x7fc00000) : pow2f(-E);
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const int Tlo = (a4[rb][n][0] >> rb) + 256 * (a4[rb][n][1] >> rb);
                        const int Thi = (a4[rb][n][2] >> (rb + 4)) + 256 * (a4[rb][n][3] >> (rb + 4));
                        const float slo = (float)(Q - 2 * Tlo) * sc;
                        const float shi = (float)(Q - 2 * Thi) * sc;
                        yv[rb][n][0] += (p ? hv[1][rb][0] : hv[0][rb][0]) * slo;
                        yv[rb][n][1] += (p ? hv[1][rb][1] : hv[0][rb][1]) * shi;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                const int rgn = rg + NW * kP2Stages;
                if (rgn < item.rg1) {
                    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                    const int sn = issued % kP2Stages;
                    ring_fill(my_ring + (size_t)sn * kStage, ut + (size_t)rgn * KB2e * 32, stage_bytes, &bars[warp][sn]);
                    ++issued;
                }
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int m = 4 * n + t4;
                if (m < M) {
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const int nlo = rg * kRowsPerGroup + rb * kRowsPerBlock + g;
                        if (nlo < N) y[(size_t)m * N + nlo] = yv[rb][n][0];
                        if (nlo + 8 < N) y[(size_t)m * N + nlo + 8] = yv[rb][n][1];
                    }
                }
            }
        }
        __syncthreads();   // shared fragments are rebuilt by the next item
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef void (*K1Fn)(const LayerDev *, const P1Item *, int, const IoPtrs, int, int, int *);
typedef void (*KFFn)(const LayerDev *, int, int);
typedef void (*K2Fn)(const LayerDev *, const P2Item *, int, const IoPtrs, int, int, int, int *);

template <int NT>
static void kernels_for(K1Fn &k1, KFFn &kf, K2Fn &k2)
{
    k1 = contraction1_kernel<NT>;
    kf = finish_general_kernel<NT>;
    k2 = contraction2_kernel<NT>;
}

lb_status decode_forward(const Plan &Pc, const uint16_t *const *xs, float *const *ys, int M, cudaStream_t s,
                         int *launches)
{
    Plan &P = const_cast<Plan &>(Pc);
    if (M > kMaxDecodeM) {
        // Rows beyond the decode limit run as consecutive blocks of 16 rows.
        std::vector<const uint16_t *> xc(P.n);
        std::vector<float *> yc(P.n);
        for (int m0 = 0; m0 < M; m0 += kMaxDecodeM) {
            for (int i = 0; i < P.n; ++i) {
                xc[i] = xs[i] + (size_t)m0 * P.host[i].K;
                yc[i] = ys[i] + (size_t)m0 * P.host[i].N;
            }
            lb_status st = decode_forward(P, xc.data(), yc.data(), std::min(kMaxDecodeM, M - m0), s, launches);
            if (st != LB_OK) return st;
        }
        return LB_OK;
    }
    const int NT = (M + 3) / 4;
    cudaError_t e = cudaSuccess;
    int sms = 0;
    if ((e = sm_count_of_current(&sms)) != cudaSuccess) return status_from(e);
    K1Fn k1;
    KFFn kf;
    K2Fn k2;
    switch (NT) {
    case 1: kernels_for<1>(k1, kf, k2); break;
    case 2: kernels_for<2>(k1, kf, k2); break;
    case 3: kernels_for<3>(k1, kf, k2); break;
    default: kernels_for<4>(k1, kf, k2); break;
    }
    int kb2max = 0;
    for (const LayerDev &d : P.host) kb2max = std::max(kb2max, d.KB2);
    const size_t smem1 = (size_t)(kDecodeThreads / 32) * kP1Stages * kP1StageKB * 256 +
                         (size_t)2 * kP1ChunkKB * NT * 32 * sizeof(uint2);
    const size_t smem2 = (size_t)(kDecodeThreads / 32) * kP2Stages * ((kb2max + 1) & ~1) * 256 +
                         (size_t)NT * kb2max * 32 * sizeof(uint2);
    // a stack deeper than the general kernels' shared memory holds runs on the one/two-row streaming kernels
    // (no shared-memory bound on the depth), once per pair of activation rows; the general kernels are set up
    // only where they fit
    const bool general_fits = smem2 <= 227 * 1024;
    const bool by_pairs = M > 2 && !general_fits;
    int occ1 = 1, occ2 = 1;
    if (general_fits) {
        if ((e = ensure_dyn_smem((const void *)k1, smem1)) != cudaSuccess) return status_from(e);
        if ((e = ensure_dyn_smem((const void *)k2, smem2)) != cudaSuccess) return status_from(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ1, k1, kDecodeThreads, smem1)) != cudaSuccess)
            return status_from(e);
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ2, k2, kDecodeThreads, smem2)) != cudaSuccess)
            return status_from(e);
        occ1 = std::max(1, occ1);
        occ2 = std::max(1, occ2);
    }

    static thread_local IoPtrs io;
    profile_mark(0, s);
    const int nb = (int)P.p1_start.size() - 1;
    for (int b = 0; b < nb; ++b) {
        const int base = b * kIoBatch;
        const int cnt = std::min(kIoBatch, P.n - base);
        if (by_pairs) {
            for (int m0 = 0; m0 < M; m0 += 2) {
                for (int i = 0; i < cnt; ++i) {
                    const LayerDev &d = P.host[base + i];
                    io.x[i] = xs[base + i] + (size_t)m0 * d.K;
                    io.y[i] = ys[base + i] + (size_t)m0 * d.N;
                }
                const lb_status st = decode_pair_launch(P.dev, cnt, P.p1 + P.p1_start[b], P.p1_start[b + 1] - P.p1_start[b],
                                                        P, b, io, base, std::min(2, M - m0), kb2max, P.rmax, P.err, s,
                                                        launches, true);
                if (st != LB_OK) return st;
            }
            continue;
        }
        for (int i = 0; i < cnt; ++i) {
            io.x[i] = xs[base + i];
            io.y[i] = ys[base + i];
        }
        const int n1 = P.p1_start[b + 1] - P.p1_start[b];
        const int n2 = P.p2_start[b + 1] - P.p2_start[b];
        if (M <= 2 && kb2max <= kPairMaxKB2) {
            lb_status st = decode_pair_launch(P.dev, cnt, P.p1 + P.p1_start[b], n1, P, b, io, base, M, kb2max, P.rmax,
                                              P.err, s, launches, true);
            if (st == LB_OK) continue;
            if (st != LB_ERR_UNSUPPORTED || !general_fits) return st;
            // a shape the streaming kernels do not take runs on the general kernels
        }
        const int grid1 = std::max(1, std::min(n1, sms * occ1));
        const int grid2 = std::max(1, std::min(n2, sms * occ2));
        k1<<<grid1, kDecodeThreads, smem1, s>>>(P.dev, P.p1 + P.p1_start[b], n1, io, base, M, P.err);
        profile_mark(++*launches, s);
        kf<<<cnt, kFinishGeneralThreads, 0, s>>>(P.dev, base, M);
        profile_mark(++*launches, s);
        k2<<<grid2, kDecodeThreads, smem2, s>>>(P.dev, P.p2 + P.p2_start[b], n2, io, base, M, kb2max, P.err);
        profile_mark(++*launches, s);
    }
    e = cudaGetLastError();
    return status_from(e);
}

// One layer whose descriptor (and scratch) the caller placed in device
// memory: the decode kernels over the work items of the layer's own plan.
// Used by the entry point that must not allocate.
lb_status decode_launch_one(const LayerDev *dev_desc, const LayerDev &host_desc, const Plan &P, const uint16_t *x,
                            float *y, int M, int *err, cudaStream_t s, int *launches)
{
    const P1Item *p1 = P.p1;
    const P2Item *p2 = P.p2;
    const int n1 = P.n_p1, n2 = P.n_p2;
    if (M <= 2 && host_desc.KB2 <= kPairMaxKB2) {
        static thread_local IoPtrs io1;
        io1.x[0] = x;
        io1.y[0] = y;
        lb_status st = decode_pair_launch(dev_desc, 1, p1, n1, P, 0, io1, 0, M, host_desc.KB2, host_desc.r, err, s,
                                          launches, false);
        if (st != LB_ERR_UNSUPPORTED) return st;
        // as in decode_forward: a shape the streaming kernels cannot hold takes the general kernels
    }
    const int NT = (M + 3) / 4;
    cudaError_t e = cudaSuccess;
    int sms = 0;
    if ((e = sm_count_of_current(&sms)) != cudaSuccess) return status_from(e);
    K1Fn k1;
    KFFn kf;
    K2Fn k2;
    switch (NT) {
    case 1: kernels_for<1>(k1, kf, k2); break;
    case 2: kernels_for<2>(k1, kf, k2); break;
    case 3: kernels_for<3>(k1, kf, k2); break;
    default: kernels_for<4>(k1, kf, k2); break;
    }
    const int kb2max = host_desc.KB2;
    const size_t smem1 = (size_t)(kDecodeThreads / 32) * kP1Stages * kP1StageKB * 256 +
                         (size_t)2 * kP1ChunkKB * NT * 32 * sizeof(uint2);
    const size_t smem2 = (size_t)(kDecodeThreads / 32) * kP2Stages * ((kb2max + 1) & ~1) * 256 +
                         (size_t)NT * kb2max * 32 * sizeof(uint2);
    if (smem2 > 227 * 1024) {
        // too deep for the general kernels: the one/two-row streaming kernels, once per pair of rows
        static thread_local IoPtrs iop;
        for (int m0 = 0; m0 < M; m0 += 2) {
            iop.x[0] = x + (size_t)m0 * host_desc.K;
            iop.y[0] = y + (size_t)m0 * host_desc.N;
            const lb_status st = decode_pair_launch(dev_desc, 1, p1, n1, P, 0, iop, 0, std::min(2, M - m0),
                                                    host_desc.KB2, host_desc.r, err, s, launches, false);
            if (st != LB_OK) return st;
        }
        return LB_OK;
    }
    if ((e = ensure_dyn_smem((const void *)k1, smem1)) != cudaSuccess) return status_from(e);
    if ((e = ensure_dyn_smem((const void *)k2, smem2)) != cudaSuccess) return status_from(e);
    int occ1 = 0, occ2 = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ1, k1, kDecodeThreads, smem1)) != cudaSuccess)
        return status_from(e);
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ2, k2, kDecodeThreads, smem2)) != cudaSuccess)
        return status_from(e);
    static thread_local IoPtrs io;
    io.x[0] = x;
    io.y[0] = y;
    const int grid1 = std::max(1, std::min(n1, sms * std::max(1, occ1)));
    const int grid2 = std::max(1, std::min(n2, sms * std::max(1, occ2)));
    k1<<<grid1, kDecodeThreads, smem1, s>>>(dev_desc, p1, n1, io, 0, M, err);
    ++*launches;
    kf<<<1, kFinishGeneralThreads, 0, s>>>(dev_desc, 0, M);
    ++*launches;
    k2<<<grid2, kDecodeThreads, smem2, s>>>(dev_desc, p2, n2, io, 0, M, kb2max, err);
    ++*launches;
    return status_from(cudaGetLastError());
}

}  // namespace lb

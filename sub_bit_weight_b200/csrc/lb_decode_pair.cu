// Decode kernels for one or two activation rows (M <= 2), both paths merged.
//
// Same method as lb_decode.cu (LittleBit notes page, "Multi-scale
// compensation": x (.) g . V_sign (.) l . U_sign^T (.) h; "Residual
// compensation": the two paths summed), specialised for the batch sizes of
// token-by-token decoding.  With M <= 2 the 8 columns of one m16n8k32 B
// fragment hold every activation operand at once:
//
//     column = 4 * m + 2 * path + digit        (m < 2, path < 2, digit < 2)
//
// so one MMA per (row block, k-block) serves both paths.  For M = 1 only the
// first 16 lanes of a B fragment carry data; those fragments are stored
// compactly (16 * M lanes per k-block) and the other lanes read zeros.
//
// Four launches:
//   quantize_pair_kernel      x (.) g_p as 16-bit fixed point per 1024-input
//                             chunk -> contraction-1 B fragments + exponents
//   contraction1_pair_kernel  z = sum_k b * t over V tiles, float64 atomics
//   finish_pair_kernel        zl = z (.) l_p as 16-bit fixed point -> the
//                             contraction-2 B fragments (one CTA per layer)
//   contraction2_pair_kernel  y = sum_p h_p (.) (U_p zl_p) over U tiles
// The float64 row sums of contraction 1 use the first R1 * M doubles of the
// layer's accumulator block as a compact [R1][M] array (the general decode
// kernels use [R1][16]); both leave the block zero for the next call.
// In both contractions every warp streams its own contiguous, equal share of
// the weight bytes (a static partition made at plan build) through a private
// ring of bulk copies; warps never synchronise with each other.

#include <utility>

#include "lb_decode_common.cuh"

namespace lb {

// ---------------------------------------------------------------------------
// Activation quantisation: one warp per 1024-input chunk, lane L takes k-block
// L of the chunk (32 inputs) and writes that k-block's whole B fragment.
// ---------------------------------------------------------------------------
constexpr int kQuantWarps = 4;

// The four bytes of 32-bit values a..d, low byte first.
static __device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d)
{
    return (uint32_t)(a & 255) | ((uint32_t)(b & 255) << 8) | ((uint32_t)(c & 255) << 16) | ((uint32_t)(d & 255) << 24);
}

template <int MM>
__global__ void __launch_bounds__(kQuantWarps * 32, MM == 1 ? 5 : 3)
    quantize_pair_kernel(const LayerDev *__restrict__ layers, const P1Item *__restrict__ items, int nitems,
                         const __grid_constant__ IoPtrs io, int base, int M)
{
    dep_release();
    const int lane = threadIdx.x & 31;
    const int it = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    if (it >= nitems) return;
    const P1Item item = items[it];
    const LayerDev *dp = layers + item.layer;
    const int K = dp->K, K32 = dp->K32, KB1 = dp->KB1, npaths = dp->npaths, R1 = dp->R1;
    const uint16_t *__restrict__ x = io.x[item.layer - base];
    const int kb = item.kc * kP1ChunkKB + lane;
    const bool act = kb < KB1;
    const int k0 = kb * kKPerBlock;

    // raw bf16 activations and binary16 g of this lane's 32 inputs (two per word)
    uint32_t xr[MM][16], gr[2][16];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        if (act && p < npaths) {
            const uint4 *src = reinterpret_cast<const uint4 *>(dp->g + (size_t)p * K32 + k0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = __ldg(src + i);
                gr[p][4 * i] = v.x; gr[p][4 * i + 1] = v.y; gr[p][4 * i + 2] = v.z; gr[p][4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) gr[p][i] = 0u;
        }
    }
    const bool vec = ((K & 7) == 0) && (k0 + kKPerBlock <= K);
#pragma unroll
    for (int m = 0; m < MM; ++m) {
        if (!act || m >= M) {
#pragma unroll
            for (int i = 0; i < 16; ++i) xr[m][i] = 0u;
        } else if (vec) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)m * K + k0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = __ldg(src + i);
                xr[m][4 * i] = v.x; xr[m][4 * i + 1] = v.y; xr[m][4 * i + 2] = v.z; xr[m][4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k = k0 + 2 * i;
                const uint32_t lo = (k < K) ? __ldg(x + (size_t)m * K + k) : 0u;
                const uint32_t hi = (k + 1 < K) ? __ldg(x + (size_t)m * K + k + 1) : 0u;
                xr[m][i] = lo | (hi << 16);
            }
        }
    }
    auto tval = [&](int m, int p, int e) -> float {      // x_e * g_{p,e} (exact in fp32)
        const uint32_t xw = xr[m][e >> 1], gw = gr[p][e >> 1];
        const float xv = __uint_as_float((e & 1) ? (xw & 0xffff0000u) : (xw << 16));
        const float gv = __half2float(__ushort_as_half((unsigned short)((e & 1) ? (gw >> 16) : (gw & 0xffffu))));
        return xv * gv;
    };

    uint4 *dst = reinterpret_cast<uint4 *>(dp->xfrag + (size_t)kb * 16 * MM);
#pragma unroll
    for (int m = 0; m < MM; ++m)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float amax = 0.0f;
            int bad = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float tv = fabsf(tval(m, p, e));
                if (!(tv <= FLT_MAX)) bad = 1;
                else amax = fmaxf(amax, tv);
            }
            amax = warp_max(amax);
            bad = warp_or(bad);
            const bool live = m < M && p < npaths;
            const int E = live ? exponent_for(amax, bad != 0) : kNanExp;
            const float sc = (E == kNanExp) ? 0.0f : pow2f(E);
            // column 4 m + 2 p + d: lanes t = 0..3 hold k 4t..4t+3 (first word) and 16+4t.. (second);
            // one 16-byte store covers lanes 2 tp and 2 tp + 1 of a column
            int qs = 0;
#pragma unroll
            for (int tp = 0; tp < 2; ++tp) {
                uint32_t wlo[4], whi[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 2 * tp + (i >> 1), k = 16 * (i & 1) + 4 * t;
                    int q[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        q[e] = quantize_s(tval(m, p, k + e), sc);
                        qs += q[e];
                    }
                    wlo[i] = pack4(q[0], q[1], q[2], q[3]);
                    whi[i] = pack4((q[0] + 128) >> 8, (q[1] + 128) >> 8, (q[2] + 128) >> 8, (q[3] + 128) >> 8);
                }
                if (act) {
                    const int col = 4 * m + 2 * p;
                    dst[2 * col + tp] = make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
                    dst[2 * (col + 1) + tp] = make_uint4(whi[0], whi[1], whi[2], whi[3]);
                }
            }
            qs = warp_sum(qs);
            if (lane == 0) {
                dp->xmeta[item.kc * 4 + 2 * p + m] = E;
                if (live) {
                    double *acc = dp->acc;
                    if (E == kNanExp) atomicOr(reinterpret_cast<int *>(acc + (size_t)R1 * 16 + 32) + p * 16 + m, 1);
                    else if (qs) atomicAdd(acc + (size_t)R1 * 16 + p * 16 + m, (double)qs * pow2d(-E));
                }
            }
        }
    if (MM == 1 && lane == 0) {
        // m = 1 slots of the chunk's exponents stay absent
        dp->xmeta[item.kc * 4 + 1] = kNanExp;
        dp->xmeta[item.kc * 4 + 3] = kNanExp;
    }
}

// ---------------------------------------------------------------------------
// Finish of contraction 1 (one CTA per layer): zl = (S_p - 2 acc) * l_p as
// 16-bit fixed point per (path, row), written as contraction-2 B fragments
// (16 * M lanes per k-block) plus (exponent, digit sum) in zmeta; clears the
// accumulators for the next call.  zl is staged in shared memory.
// ---------------------------------------------------------------------------
constexpr int kFinishThreads = 256;

template <int MM>
__global__ void __launch_bounds__(kFinishThreads)
    finish_pair_kernel(const LayerDev *__restrict__ layers, int base, int M)
{
    extern __shared__ float szl[];      // [npaths][r][MM]
    __shared__ float sMax[4];
    __shared__ int sBad[4], sE[4], sQs[4];
    const int tid = threadIdx.x;
    dep_release();
    const LayerDev *dp = layers + base + blockIdx.x;
    const int R1 = dp->R1, r = dp->r, r16 = dp->r16, r32 = dp->r32, npaths = dp->npaths, KB2 = dp->KB2;
    double *acc = dp->acc;
    const __half *lsc = dp->l;
    dep_wait();                          // the row sums of contraction 1
    const double *S = acc + (size_t)R1 * 16;
    const int *badf = reinterpret_cast<const int *>(acc + (size_t)R1 * 16 + 32);
    if (tid < 4) {
        sMax[tid] = 0.0f;
        sBad[tid] = 0;
        sQs[tid] = 0;
    }
    __syncthreads();
    for (int e = tid; e < npaths * r * MM; e += kFinishThreads) {
        const int m = e % MM, pj = e / MM;
        const int p = pj / r, j = pj - p * r;
        float zl = 0.0f;
        if (m < M) {
            const double z = __ldcg(S + p * 16 + m) - 2.0 * __ldcg(acc + (size_t)(p * r16 + j) * MM + m);
            zl = (float)z * __half2float(lsc[p * r16 + j]);
            if (!(fabsf(zl) <= FLT_MAX)) atomicOr(&sBad[2 * p + m], 1);
            else smem_max(&sMax[2 * p + m], fabsf(zl));
        }
        szl[e] = zl;
    }
    __syncthreads();
    if (tid < 4) {
        const int p = tid >> 1, m = tid & 1;
        sE[tid] = (p < npaths && m < M) ? exponent_for(sMax[tid], sBad[tid] != 0 || __ldcg(badf + p * 16 + m) != 0)
                                        : kNanExp;
    }
    __syncthreads();
    // fragment word pairs: lane L < 16 * MM of k-block kb holds column L / 4 = 4 m + 2 p + d
    for (int idx = tid; idx < KB2 * 16 * MM; idx += kFinishThreads) {
        const int kb = idx / (16 * MM), lane = idx - kb * 16 * MM;
        const int col = lane >> 2, t = lane & 3;
        const int fm = col >> 2, fp = (col >> 1) & 1, fd = col & 1;
        uint32_t w[2] = {0u, 0u};
        int qs = 0;
        if (fm < M && fp < npaths && kb * kKPerBlock / r32 == fp) {
            const int E = sE[2 * fp + fm];
            const float sc = (E == kNanExp) ? 0.0f : pow2f(E);
            const int j0 = kb * kKPerBlock - fp * r32 + 4 * t;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j0 + 16 * hh + e;
                    const int q = (j < r) ? quantize_s(szl[(fp * r + j) * MM + fm], sc) : 0;
                    int lo, hi;
                    digits(q, lo, hi);
                    w[hh] |= (uint32_t)((fd ? hi : lo) & 255) << (8 * e);
                    qs += q;
                }
            if (fd == 0 && qs) atomicAdd(&sQs[2 * fp + fm], qs);
        }
        dp->zfrag[idx] = make_uint2(w[0], w[1]);
    }
    __syncthreads();
    if (tid < 4) {
        const int p = tid >> 1, m = tid & 1;
        dp->zmeta[p * 16 + m] = make_int2(sE[tid], sQs[tid]);
    }
    // clear for the next call: the rows (compact [R1][MM] here), the k sums and the flags
    for (int i = tid; i < R1 * MM; i += kFinishThreads) acc[i] = 0.0;
    for (int i = tid; i < 48; i += kFinishThreads) acc[(size_t)R1 * 16 + i] = 0.0;
}

// ---------------------------------------------------------------------------
// Per-warp streaming: a ring of kPairStages bulk-copy stages (kPairStageKB
// k-blocks each) and two B slots (fragments + their metadata), one mbarrier
// each.  Unit records are read one unit ahead so no global load sits on the
// path from one unit to the next.
// ---------------------------------------------------------------------------

// N k-blocks of MMAs, fully unrolled: A word pairs 256 bytes apart, B fragments
// 16 * MM * 8 bytes apart (lanes without B data read a zero buffer of the same
// shape), so every shared-memory address is a register plus an immediate.
template <int MM, int N>
static __device__ __forceinline__ void mma_run(int (&a4)[4][4], uint32_t src, uint32_t bsrc)
{
#pragma unroll
    for (int v = 0; v < N; ++v) {
        const uint2 w = lds64(src + v * 256);
        const uint2 b = lds64(bsrc + v * (16 * MM * 8));
#pragma unroll
        for (int rb = 0; rb < 4; ++rb) {
            const uint32_t mlo = 0x01010101u << rb, mhi = 0x01010101u << (rb + 4);
            mma_u8s8(a4[rb], w.x & mlo, w.x & mhi, w.y & mlo, w.y & mhi, b.x, b.y);
        }
    }
}

// n (1..kPairStageKB) k-blocks: a full stage in one unrolled body, otherwise the
// binary decomposition of n (at most four unrolled bodies, no jump table).
template <int MM>
static __device__ __forceinline__ void mma_stage(int (&a4)[4][4], uint32_t src, uint32_t bsrc, int n)
{
    static_assert(kPairStageKB == 16, "stage of 16 k-blocks");
    if (n == 16) {
        mma_run<MM, 16>(a4, src, bsrc);
        return;
    }
    if (n & 8) {
        mma_run<MM, 8>(a4, src, bsrc);
        src += 8 * 256;
        bsrc += 8 * (16 * MM * 8);
    }
    if (n & 4) {
        mma_run<MM, 4>(a4, src, bsrc);
        src += 4 * 256;
        bsrc += 4 * (16 * MM * 8);
    }
    if (n & 2) {
        mma_run<MM, 2>(a4, src, bsrc);
        src += 2 * 256;
        bsrc += 2 * (16 * MM * 8);
    }
    if (n & 1) mma_run<MM, 1>(a4, src, bsrc);
}

// ---------------------------------------------------------------------------
// Contraction 1 (one warp per contiguous run of units).  A ring stage holds up
// to kPairStageKB k-blocks of one unit's V tiles, the B fragments of the same
// k-blocks and the chunk's four exponents (three bulk copies on one mbarrier);
// nothing else is shared between units, so the warp needs no B slots.
// ---------------------------------------------------------------------------
template <int MM>
__global__ void __launch_bounds__(pair_warps_per_cta(MM) * 32, 1)
    contraction1_pair_kernel(const LayerDev *__restrict__ layers, const PairUnit1 *__restrict__ units,
                             const int *__restrict__ wrange, int M, int *err)
{
    constexpr int kBStride = 16 * MM * 8;                   // bytes of B fragments per k-block
    constexpr int kA = kPairStageKB * 256, kB = kPairStageKB * kBStride;
    constexpr int kStageAll = kA + kB + 16;                 // V tiles, B fragments, exponents
    constexpr int kPairWarps = pair_warps_per_cta(MM);
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ uint64_t rbar[kPairWarps][kPairStages];
    __shared__ __align__(16) uint4 zbuf[MM == 1 ? kPairStageKB * 128 / 16 : 1];   // B of the lanes past 16 * MM

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int lane_m = t4 >> 1, lane_p = t4 & 1;       // accumulator columns of this lane
    unsigned char *ring = smem_raw + warp * (kPairStages * kStageAll);
    for (int i = threadIdx.x; i < (int)(sizeof(zbuf) / 16); i += blockDim.x) zbuf[i] = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0)
        for (int s = 0; s < kPairStages; ++s) bar_init(&rbar[warp][s]);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncthreads();    // the only CTA-wide barrier: the zero buffer and the barriers are ready
    dep_release();

    const int gw = warp * gridDim.x + blockIdx.x;     // an SM's warps take ranges spread over the whole batch
    const int u0 = wrange[gw], u1 = wrange[gw + 1];
    if (u0 >= u1) return;
    const uint64_t pol = l2_evict_first();
    // V tiles do not depend on the previous kernel; B fragments and exponents do: stages
    // filled before dep_wait() get theirs afterwards (at most kPairStages of them)
    bool dep_ok = false;
    int npend = 0;
    const uint2 *pend_b[kPairStages];
    const int *pend_e[kPairStages];
    unsigned pend_nb[kPairStages];

    // ---- fill cursor: stages of units [f_u, u1) in consumption order, at most kPairStages ahead
    int f_u = u0, f_h = 0, f_layer = -1, issued = 0, consumed = 0;
    const uint2 *f_xfrag = nullptr;
    const int *f_xmeta = nullptr;
    PairUnit1 f_cur = units[u0], f_nxt = f_cur;
    if (u0 + 1 < u1) f_nxt = units[u0 + 1];
    auto fill = [&]() {
        while (f_u < u1 && issued - consumed < kPairStages) {
            if (f_cur.layer != f_layer) {
                f_layer = f_cur.layer;
                f_xfrag = layers[f_layer].xfrag;
                f_xmeta = layers[f_layer].xmeta;
            }
            const int n = min(kPairStageKB, f_cur.nkb - f_h * kPairStageKB);
            {
                const int st = issued % kPairStages;
                unsigned char *dst = ring + st * kStageAll;
                uint64_t *bar = &rbar[warp][st];
                const int kb0 = f_cur.kc * kP1ChunkKB + f_h * kPairStageKB;
                const uint32_t lead = lane == 0;
                lead_fill_hint(lead, bar, (unsigned)n * (256u + kBStride) + 16u, dst,
                               f_cur.a + (size_t)f_h * kPairStageKB * 32, (unsigned)n * 256u, pol);
                if (dep_ok) {
                    lead_copy(lead, bar, dst + kA, f_xfrag + (size_t)kb0 * 16 * MM, (unsigned)n * kBStride);
                    lead_copy(lead, bar, dst + kA + kB, f_xmeta + f_cur.kc * 4, 16u);
                } else {
#pragma unroll
                    for (int i = 0; i < kPairStages; ++i)
                        if (i == npend) {
                            pend_b[i] = f_xfrag + (size_t)kb0 * 16 * MM;
                            pend_e[i] = f_xmeta + f_cur.kc * 4;
                            pend_nb[i] = (unsigned)n * kBStride;
                        }
                }
            }
            if (!dep_ok) ++npend;
            ++issued;
            if (++f_h * kPairStageKB >= f_cur.nkb) {
                f_h = 0;
                ++f_u;
                f_cur = f_nxt;
                if (f_u + 1 < u1) f_nxt = units[f_u + 1];
            }
        }
    };
    fill();
    dep_wait();
    dep_ok = true;
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < kPairStages; ++i)
            if (i < npend) {
                unsigned char *dst = ring + i * kStageAll;
                bulk_copy(dst + kA, pend_b[i], pend_nb[i], &rbar[warp][i]);
                bulk_copy(dst + kA + kB, pend_e[i], 16u, &rbar[warp][i]);
            }

    // ---- consumer
    int c_layer = -1, c_r16 = 1, c_npaths = 1;
    double *c_acc = nullptr;
    const bool real = lane < 16 * MM;
    const uint32_t zaddr = sm_addr(zbuf) + (lane & 15) * 8;
    PairUnit1 c_nxt = units[u0];
    for (int u = u0; u < u1; ++u) {
        const PairUnit1 cu = c_nxt;
        if (u + 1 < u1) c_nxt = units[u + 1];
        if (cu.layer != c_layer) {
            const LayerDev *dp = layers + cu.layer;
            c_layer = cu.layer;
            c_acc = dp->acc;
            c_r16 = dp->r16;
            c_npaths = dp->npaths;
        }
        int a4[4][4];
#pragma unroll
        for (int rb = 0; rb < 4; ++rb)
#pragma unroll
            for (int c = 0; c < 4; ++c) a4[rb][c] = 0;
        double lane_sc = 0.0;
        bool lane_live = false;
        for (int h = 0; h * kPairStageKB < cu.nkb; ++h) {
            const int st = consumed % kPairStages;
            if (!ring_wait(&rbar[warp][st], (consumed / kPairStages) & 1, err)) return;
            const uint32_t sbase = sm_addr(ring + st * kStageAll);
            if (h == 0) {
                const int E = (lane_m < M && lane_p < c_npaths) ? (int)lds_u32(sbase + kA + kB + 4 * (2 * lane_p + lane_m))
                                                                 : kNanExp;
                lane_live = E != kNanExp;
                lane_sc = lane_live ? pow2d(-E) : 0.0;
            }
            mma_stage<MM>(a4, sbase + lane * 8, real ? sbase + kA + lane * 8 : zaddr,
                          min(kPairStageKB, cu.nkb - h * kPairStageKB));
            __syncwarp();
            proxy_fence();
            ++consumed;
            fill();
        }
        // keep the columns of each row block's own path; partial sums over chunks add up exactly
#pragma unroll
        for (int rb = 0; rb < 4; ++rb) {
            const int row0 = cu.rg * kRowsPerGroup + rb * kRowsPerBlock;
            const int prb = (c_npaths > 1 && row0 >= c_r16) ? 1 : 0;     // path 1 owns rows r16..
            if (prb != lane_p || !lane_live) continue;
            const int Tlo = (a4[rb][0] >> rb) + 256 * (a4[rb][1] >> rb);
            const int Thi = (a4[rb][2] >> (rb + 4)) + 256 * (a4[rb][3] >> (rb + 4));
            if (Tlo) atomicAdd(c_acc + (size_t)(row0 + g) * MM + lane_m, (double)Tlo * lane_sc);
            if (Thi) atomicAdd(c_acc + (size_t)(row0 + g + 8) * MM + lane_m, (double)Thi * lane_sc);
        }
    }
}

// ---------------------------------------------------------------------------
// Contraction 2 (+ h, + path sum): one warp per contiguous run of row groups.
// A layer's U tiles are contiguous over its row groups, so a ring stage takes
// up to kPairStageKB consecutive k-blocks across row-group boundaries (never
// across layers); the consumer folds a row group when its KB2 k-blocks are in.
// ---------------------------------------------------------------------------
template <int MM, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
    contraction2_pair_kernel(const LayerDev *__restrict__ layers, const PairUnit2 *__restrict__ units,
                             const int *__restrict__ wrange, const __grid_constant__ IoPtrs io, int base, int M,
                             int kb2max, int *err)
{
    constexpr int kStage = kPairStageKB * 256;
    constexpr int kBStride = 16 * MM * 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ uint64_t rbar[NW][kPairStages];
    __shared__ uint64_t bbar[NW][2];
    __shared__ int snb[NW][kPairStages];       // k-blocks in each ring stage

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int lane_m = t4 >> 1, lane_p = t4 & 1;
    const int kBFrag = kb2max * kBStride, kBSlot = kBFrag + kPairMeta2;
    unsigned char *ring = smem_raw + (size_t)warp * (kPairStages * kStage + 2 * kBSlot);
    unsigned char *bslot = ring + kPairStages * kStage;
    // after the warps' regions: zeros shaped like a B slot, read by the lanes past 16 * MM
    uint4 *zbuf = reinterpret_cast<uint4 *>(smem_raw + (size_t)NW * (kPairStages * kStage + 2 * kBSlot));
    if (MM == 1)
        for (int i = threadIdx.x; i < kb2max * kBStride / 16; i += blockDim.x) zbuf[i] = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) {
        for (int s = 0; s < kPairStages; ++s) bar_init(&rbar[warp][s]);
        bar_init(&bbar[warp][0]);
        bar_init(&bbar[warp][1]);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    __syncthreads();
    dep_release();

    const int gw = warp * gridDim.x + blockIdx.x;     // an SM's warps take ranges spread over the whole batch
    const int u0 = wrange[gw], u1 = wrange[gw + 1];
    if (u0 >= u1) return;
    const uint64_t pol = l2_evict_first();
    // U tiles and h do not depend on the previous kernel; the zl fragments do: a layer's B
    // slot wanted before dep_wait() is filled afterwards (at most one: the first layer)
    bool dep_ok = false;
    int pend_layer = -1;

    // ---- fill cursor (position: unit f_u, k-block f_kb within it)
    int f_u = u0, f_kb = 0, f_layer = -1, f_cs = -1, issued = 0, consumed = 0, c_cs = -1;
    PairUnit2 f_cur = units[u0], f_nxt = f_cur;
    if (u0 + 1 < u1) f_nxt = units[u0 + 1];
    auto fill = [&]() {
        while (f_u < u1 && issued - consumed < kPairStages) {
            if (f_cur.layer != f_layer) {
                if (f_cs >= c_cs + 1) return;           // both B slots still in use
                ++f_cs;
                f_layer = f_cur.layer;
                if (!dep_ok) pend_layer = f_layer;
                else if (lane == 0) {
                    const LayerDev *fd = layers + f_layer;
                    unsigned char *dst = bslot + (f_cs & 1) * kBSlot;
                    uint64_t *bar = &bbar[warp][f_cs & 1];
                    const unsigned fb = (unsigned)f_cur.kb2 * kBStride;
                    asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(
                                     sm_addr(bar)),
                                 "r"(fb + (unsigned)kPairMeta2)
                                 : "memory");
                    bulk_copy(dst, fd->zfrag, fb, bar);
                    bulk_copy(dst + kBFrag, fd->zmeta, (unsigned)kPairMeta2, bar);
                }
            }
            const uint2 *src = f_cur.a + (size_t)f_kb * 32;
            int n = 0;
            while (true) {
                const int t = min(kPairStageKB - n, f_cur.kb2 - f_kb);
                n += t;
                f_kb += t;
                if (f_kb < f_cur.kb2) break;            // the stage is full inside this row group
                f_kb = 0;
                ++f_u;
                f_cur = f_nxt;
                if (f_u + 1 < u1) f_nxt = units[f_u + 1];
                if (n == kPairStageKB || f_u >= u1 || f_cur.layer != f_layer) break;
            }
            const int st = issued % kPairStages;
            snb[warp][st] = n;
            if (lane == 0) {
                expect_tx(&rbar[warp][st], (unsigned)n * 256u);
                bulk_copy_hint(ring + st * kStage, src, (unsigned)n * 256u, &rbar[warp][st], pol);
            }
            ++issued;
        }
    };
    fill();
    dep_wait();
    dep_ok = true;
    if (pend_layer >= 0 && lane == 0) {
        const LayerDev *fd = layers + pend_layer;
        uint64_t *bar = &bbar[warp][0];
        const unsigned fb = (unsigned)fd->KB2 * kBStride;
        expect_tx(bar, fb + (unsigned)kPairMeta2);
        bulk_copy(bslot, fd->zfrag, fb, bar);
        bulk_copy(bslot + kBFrag, fd->zmeta, (unsigned)kPairMeta2, bar);
    }

    int c_layer = -1, N = 0, npaths = 1;
    float *y = nullptr;
    float my_sc = 0.0f, my_q = 0.0f;
    uint32_t bbase = 0;
    const uint32_t zaddr = sm_addr(zbuf) + (lane & 15) * 8;
    int s_left = 0;             // k-blocks of the current stage not yet used
    uint32_t s_addr = 0;        // this lane's word pair of the stage's next k-block

    // h of this lane's path for rows g and g + 8 of each row block of a unit,
    // read one unit ahead
    int h_layer = -1;
    const __half *h_base = nullptr;      // this lane's path row of h in layer h_layer, or null
    auto load_h = [&](const PairUnit2 &un, __half (&hq)[8]) {
        if (un.layer != h_layer) {
            const LayerDev *dp = layers + un.layer;
            h_layer = un.layer;
            h_base = (lane_p < dp->npaths) ? dp->h + (size_t)lane_p * dp->N64 : nullptr;
        }
        const __half *hp = h_base + un.rg * kRowsPerGroup + g;
#pragma unroll
        for (int i = 0; i < 8; ++i) hq[i] = h_base ? __ldg(hp + (i >> 1) * kRowsPerBlock + 8 * (i & 1)) : __half(0.0f);
    };
    PairUnit2 c_nxt = units[u0];
    __half h_nxt[8];
    load_h(c_nxt, h_nxt);
    for (int u = u0; u < u1; ++u) {
        const PairUnit2 cu = c_nxt;
        float hv[4][2];
#pragma unroll
        for (int i = 0; i < 8; ++i) hv[i >> 1][i & 1] = __half2float(h_nxt[i]);
        if (u + 1 < u1) {
            c_nxt = units[u + 1];
            load_h(c_nxt, h_nxt);
        }
        if (cu.layer != c_layer) {
            const LayerDev *dp = layers + cu.layer;
            c_layer = cu.layer;
            N = dp->N;
            npaths = dp->npaths;
            y = io.y[cu.layer - base];
            ++c_cs;
            fill();
            if (!ring_wait(&bbar[warp][c_cs & 1], (c_cs >> 1) & 1, err)) return;
            const unsigned char *slot = bslot + (c_cs & 1) * kBSlot;
            my_sc = my_q = 0.0f;
            if (lane_m < M && lane_p < npaths) {
                const uint32_t ma = sm_addr(slot + kBFrag + 8 * (lane_p * 16 + lane_m));
                const int ex = (int)lds_u32(ma), qsum = (int)lds_u32(ma + 4);
                if (ex == kNanExp) {
                    my_sc = my_q = __int_as_float(0x7fc00000);
                } else {
                    my_sc = -2.0f * pow2f(-ex);                  // s = Q 2^-E - 2 T 2^-E
                    my_q = (float)qsum * pow2f(-ex);
                }
            }
            const bool real = lane < 16 * MM;
            bbase = real ? sm_addr(slot) + lane * 8 : zaddr;
        }
        const int n0 = cu.rg * kRowsPerGroup + g;

        int a4[4][4];
#pragma unroll
        for (int rb = 0; rb < 4; ++rb)
#pragma unroll
            for (int c = 0; c < 4; ++c) a4[rb][c] = 0;
        for (int kb = 0; kb < cu.kb2;) {
            if (s_left == 0) {
                const int st = consumed % kPairStages;
                if (!ring_wait(&rbar[warp][st], (consumed / kPairStages) & 1, err)) return;
                s_left = snb[warp][st];
                s_addr = sm_addr(ring + st * kStage) + lane * 8;
            }
            const int seg = min(s_left, cu.kb2 - kb);
            mma_stage<MM>(a4, s_addr, bbase + (uint32_t)kb * kBStride, seg);
            kb += seg;
            s_left -= seg;
            s_addr += (uint32_t)seg * 256u;
            if (s_left == 0) {
                __syncwarp();
                if (lane == 0) proxy_fence();
                ++consumed;
                fill();
            }
        }

        // lane (m, path): its path's share of rows g and g + 8, then the pair sum
#pragma unroll
        for (int rb = 0; rb < 4; ++rb) {
            const int Tlo = (a4[rb][0] >> rb) + 256 * (a4[rb][1] >> rb);
            const int Thi = (a4[rb][2] >> (rb + 4)) + 256 * (a4[rb][3] >> (rb + 4));
            float vlo = hv[rb][0] * fmaf((float)Tlo, my_sc, my_q);
            float vhi = hv[rb][1] * fmaf((float)Thi, my_sc, my_q);
            vlo += __shfl_xor_sync(0xffffffffu, vlo, 1);
            vhi += __shfl_xor_sync(0xffffffffu, vhi, 1);
            const int nlo = n0 + rb * kRowsPerBlock;
            if (lane_p == 0 && lane_m < M) {
                if (nlo < N) y[(size_t)lane_m * N + nlo] = vlo;
                if (nlo + 8 < N) y[(size_t)lane_m * N + nlo + 8] = vhi;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int g_pair_smem1[2];          // dynamic shared memory attribute set so far, per MM

// Launch that may overlap the previous kernel of the stream (programmatic stream
// serialisation; the kernel waits with dep_wait() before using its results).
template <typename... P, typename... A>
static cudaError_t launch_dependent(bool pdl, void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t s, A &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}
static int g_pair_smem2[2][5];       // per MM and contraction-2 warp count (16, 12, 8, 6, 4)

template <int MM, int NW>
static cudaError_t launch_c2(bool pdl, int grid, size_t smem, cudaStream_t s, int slot, const LayerDev *dev_layers,
                             const PairUnit2 *u2, const int *wr2, const IoPtrs &io, int base, int M, int kb2max, int *err)
{
    cudaError_t e;
    if ((int)smem > g_pair_smem2[MM - 1][slot]) {
        if ((e = cudaFuncSetAttribute(contraction2_pair_kernel<MM, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        g_pair_smem2[MM - 1][slot] = (int)smem;
    }
    return launch_dependent(pdl, contraction2_pair_kernel<MM, NW>, dim3(grid), dim3(NW * 32), smem, s, dev_layers, u2,
                            wr2, io, base, M, kb2max, err);
}

template <int MM>
static lb_status pair_launch_mm(const LayerDev *dev_layers, int nlayers, const P1Item *p1, int n1,
                                const PairUnit1 *u1, const int *wr1, const PairUnit2 *u2, const int *wr2,
                                int pair_warps, int pair_warps2, const IoPtrs &io, int base, int M, int kb2max, int rmax,
                                int *err, cudaStream_t s, int *launches, bool mark)
{
    cudaError_t e;
    constexpr int kPairWarps = pair_warps_per_cta(MM);
    const int nw2 = pair2_warps_per_cta(MM, kb2max);
    const size_t smem1 = (size_t)kPairWarps * kPairStages * (kPairStageKB * (256 + 16 * MM * 8) + 16);
    const size_t smem2 = pair2_cta_smem(MM, kb2max, nw2);
    if (smem1 > 227 * 1024 || smem2 > 227 * 1024 || kb2max > kPairMaxKB2 || pair_warps2 % nw2 != 0 ||
        (size_t)2 * rmax * MM * sizeof(float) > 48 * 1024)
        return LB_ERR_UNSUPPORTED;
    if ((int)smem1 > g_pair_smem1[MM - 1]) {
        if ((e = cudaFuncSetAttribute(contraction1_pair_kernel<MM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem1)) != cudaSuccess)
            return status_from(e);
        g_pair_smem1[MM - 1] = (int)smem1;
    }
    if (n1 > 0) {
        quantize_pair_kernel<MM><<<(n1 + kQuantWarps - 1) / kQuantWarps, kQuantWarps * 32, 0, s>>>(dev_layers, p1, n1, io,
                                                                                                  base, M);
        ++*launches;
        if (mark) profile_mark(*launches, s);
    }
    // the three kernels after the quantisation may each start while the previous one drains,
    // unless timing events separate the launches
    const bool pdl = !profiling_active();
    if ((e = launch_dependent(pdl, contraction1_pair_kernel<MM>, dim3(pair_warps / kPairWarps), dim3(kPairWarps * 32),
                              smem1, s, dev_layers, u1, wr1, M, err)) != cudaSuccess)
        return status_from(e);
    ++*launches;
    if (mark) profile_mark(*launches, s);
    if ((e = launch_dependent(pdl, finish_pair_kernel<MM>, dim3(nlayers), dim3(kFinishThreads),
                              (size_t)2 * rmax * MM * sizeof(float), s, dev_layers, base, M)) != cudaSuccess)
        return status_from(e);
    ++*launches;
    if (mark) profile_mark(*launches, s);
    const int grid2 = pair_warps2 / nw2;
    switch (nw2) {
    case 16: e = launch_c2<MM, 16>(pdl, grid2, smem2, s, 0, dev_layers, u2, wr2, io, base, M, kb2max, err); break;
    case 12: e = launch_c2<MM, 12>(pdl, grid2, smem2, s, 1, dev_layers, u2, wr2, io, base, M, kb2max, err); break;
    case 8: e = launch_c2<MM, 8>(pdl, grid2, smem2, s, 2, dev_layers, u2, wr2, io, base, M, kb2max, err); break;
    case 6: e = launch_c2<MM, 6>(pdl, grid2, smem2, s, 3, dev_layers, u2, wr2, io, base, M, kb2max, err); break;
    default: e = launch_c2<MM, 4>(pdl, grid2, smem2, s, 4, dev_layers, u2, wr2, io, base, M, kb2max, err); break;
    }
    if (e != cudaSuccess) return status_from(e);
    ++*launches;
    if (mark) profile_mark(*launches, s);
    return status_from(cudaGetLastError());
}

lb_status decode_pair_launch(const LayerDev *dev_layers, int nlayers, const P1Item *p1, int n1, const PairUnit1 *u1,
                             const int *wr1, const PairUnit2 *u2, const int *wr2, int pair_warps, int pair_warps2,
                             const IoPtrs &io, int base, int M, int kb2max, int rmax, int *err, cudaStream_t s,
                             int *launches, bool mark)
{
    if (M == 1)
        return pair_launch_mm<1>(dev_layers, nlayers, p1, n1, u1, wr1, u2, wr2, pair_warps, pair_warps2, io, base, M,
                                 kb2max, rmax, err, s, launches, mark);
    return pair_launch_mm<2>(dev_layers, nlayers, p1, n1, u1, wr1, u2, wr2, pair_warps, pair_warps2, io, base, M,
                             kb2max, rmax, err, s, launches, mark);
}

}  // namespace lb

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
// compactly (16 * M lanes per k-block).
//
// Four launches:
//   quantize_pair_kernel      x (.) g_p as 16-bit fixed point per 1024-input
//                             chunk -> contraction-1 B fragments + exponents
//   contraction1_ldg_kernel   z = sum_k b * t over V tiles, float64 atomics
//   finish_pair_kernel        zl = z (.) l_p as 16-bit fixed point -> the
//                             contraction-2 B fragments (one CTA per layer)
//   contraction2_ldg_kernel   y = sum_p h_p (.) (U_p zl_p) over U tiles
// The float64 row sums of contraction 1 use the first R1 * M doubles of the
// layer's accumulator block as a compact [R1][M] array (the general decode
// kernels use [R1][16]); both leave the block zero for the next call.
// In both contractions every warp streams its own range of units (a
// cost-balanced partition made at plan build) straight into registers;
// warps never synchronise with each other.

#include <algorithm>
#include <utility>

#include "lb_decode_common.cuh"

namespace lb {

// ---------------------------------------------------------------------------
// Activation quantisation: one warp per 1024-input chunk, lane L takes k-block
// L of the chunk (32 inputs) and writes that k-block's whole B fragment.
// ---------------------------------------------------------------------------
constexpr int kQuantWarps = 4;

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

    // k-block kb's fragment: lane L at uint2 (pair * 16 MM + L) * 2 + (kb & 1), pair = kb / 2
    uint2 *dst = dp->xfrag + (size_t)(kb >> 1) * 32 * MM + (kb & 1);
#pragma unroll
    for (int m = 0; m < MM; ++m)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            // every product once: the chunk maximum and the digits both read t[]
            float t[32];
            float amax = 0.0f;
            int bad = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                t[e] = tval(m, p, e);
                const float tv = fabsf(t[e]);
                if (!(tv <= FLT_MAX)) bad = 1;
                else amax = fmaxf(amax, tv);
            }
            amax = warp_max(amax);
            bad = warp_or(bad);
            const bool live = m < M && p < npaths;
            const int E = live ? exponent_for(amax, bad != 0) : kNanExp;
            // q = rint(t 2^E).  t 2^E is exact and |t 2^E| <= 32639 < 2^22, so one FMA that adds 1.5 * 2^23
            // rounds it to the nearest integer (ties to even) in the low mantissa bits, and subtracting the
            // bit pattern of 1.5 * 2^23 leaves q.  An absent or non-finite block gives q = 0.
            const bool none = E == kNanExp;
            const float sc = none ? 0.0f : pow2f(E);
            int qs = 0;
#pragma unroll
            for (int tp = 0; tp < 2; ++tp) {
                uint32_t wlo[4], whi[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tt = 2 * tp + (i >> 1), k = 16 * (i & 1) + 4 * tt;
                    int q[4], hq[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        q[e] = __float_as_int(fmaf(none ? 0.0f : t[k + e], sc, 12582912.0f)) - 0x4B400000;
                        hq[e] = q[e] + 128;         // the high digit (q + 128) >> 8 is byte 1 of q + 128
                        qs += q[e];
                    }
                    wlo[i] = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
                    whi[i] = __byte_perm(__byte_perm(hq[0], hq[1], 0x0051), __byte_perm(hq[2], hq[3], 0x0051), 0x5410);
                }
                if (act) {
                    const int l0 = 4 * (4 * m + 2 * p) + 2 * tp;      // column 4 m + 2 p, lanes 2 tp and 2 tp + 1
                    dst[2 * l0] = make_uint2(wlo[0], wlo[1]);
                    dst[2 * (l0 + 1)] = make_uint2(wlo[2], wlo[3]);
                    dst[2 * (l0 + 4)] = make_uint2(whi[0], whi[1]);
                    dst[2 * (l0 + 5)] = make_uint2(whi[2], whi[3]);
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
    const int R1 = dp->R1, r = dp->r, r16 = dp->r16, r32 = dp->r32, npaths = dp->npaths;
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
    for (int idx = tid; idx < dp->KB2e * 16 * MM; idx += kFinishThreads) {
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
        dp->zfrag[((size_t)(kb >> 1) * 16 * MM + lane) * 2 + (kb & 1)] = make_uint2(w[0], w[1]);
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
// The two contractions, streamed warp by warp into registers.
//
// One CTA of kLdgWarps warps per SM; every warp owns a contiguous range of
// units (64-row groups; the plan splits each batch's units into equal-cost
// ranges, one per warp, cut into segments of one layer).  A warp runs two
// streams at once, the two halves of each unit's k-range (stream 0 the first
// ceil(P/2) pairs of k-blocks, stream 1 the rest), each with its own
// accumulators, and keeps kLdgRing pairs of k-blocks per stream in flight in
// registers: every step consumes the oldest pair of each stream and loads the
// pair kLdgRing steps ahead, across unit and segment boundaries.  The weights
// are read once (no L1 allocation, evict-first in L2); the B fragments of a
// layer or chunk are reused by many units and stay in L1, loaded one step
// ahead.  No shared memory, no barrier, no warp waits for another.
// ---------------------------------------------------------------------------

static __device__ __forceinline__ uint4 ldg_weights(const uint4 *p, uint64_t pol)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// B fragments and exponents come from the previous kernel, which may still be finishing while this one starts
// (programmatic dependent launch): they are read through L2 (.cg), never through the read-only path, whose
// contents are only defined for data that stays unchanged for the kernel's whole lifetime.
static __device__ __forceinline__ uint4 ldg_frag(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// One k-block of MMAs: the lane's sign words (w0, w1) against its B fragment words (b0, b1).
static __device__ __forceinline__ void kblock(int (&a4)[4][4], uint32_t w0, uint32_t w1, uint32_t b0, uint32_t b1)
{
#pragma unroll
    for (int rb = 0; rb < 4; ++rb) {
        const uint32_t mlo = 0x01010101u << rb, mhi = 0x01010101u << (rb + 4);
        mma_u8s8(a4[rb], w0 & mlo, w0 & mhi, w1 & mlo, w1 & mhi, b0, b1);
    }
}

// One step: a pair of k-blocks of each stream (the two halves of the unit's k-range), one accumulator set.
static __device__ __forceinline__ void step_mma(int (&a4)[4][4], const uint4 &w0, const uint4 &w1, const uint4 &b0,
                                                const uint4 &b1)
{
    kblock(a4, w0.x, w0.y, b0.x, b0.y);
    kblock(a4, w1.x, w1.y, b1.x, b1.y);
    kblock(a4, w0.z, w0.w, b0.z, b0.w);
    kblock(a4, w1.z, w1.w, b1.z, b1.w);
}

static __device__ __forceinline__ void zero_acc(int (&a)[4][4])
{
#pragma unroll
    for (int rb = 0; rb < 4; ++rb)
#pragma unroll
        for (int c = 0; c < 4; ++c) a[rb][c] = 0;
}

// The weight stream of a warp: the address of the next pair of k-blocks of stream 0 (stream 1 reads h pairs
// further, when the unit has that pair), walking steps, units and segments; runs kLdgRing steps ahead of the
// MMAs.  Lanes 16..31 of one-row batches read the B data of lanes 0..15: their columns (activation row 1)
// are computed and never used.
template <typename Seg>
struct Prefetch {
    const uint4 *a;         // this lane's 16 bytes of the current unit's first pair
    int t, h, P, rem, stride, s;
    bool live;
    __device__ __forceinline__ void seg(const Seg &sg, int lane, int rstride)
    {
        a = sg_base(sg) + lane;
        P = sg.P;
        h = (P + 1) >> 1;
        rem = sg.n;
        stride = rstride;
        t = 0;
    }
    static __device__ __forceinline__ const uint4 *sg_base(const Seg1 &sg) { return sg.v; }
    static __device__ __forceinline__ const uint4 *sg_base(const Seg2 &sg) { return sg.u; }
};

static __device__ __forceinline__ int seg_stride(const Seg1 &sg) { return sg.rstride; }
static __device__ __forceinline__ int seg_stride(const Seg2 &sg) { return sg.P * 32; }

// 512 bytes of zeros: the pair a stream reads where its unit has none (stream 1 of an odd number of pairs) or
// past the warp's last unit, so that every ring load is unconditional and nothing waits on a load it issued
static __device__ __align__(16) uint4 g_zero_pair[32];

template <typename Seg>
static __device__ __forceinline__ void fetch_step(Prefetch<Seg> &pf, const Seg *segs, int s1, int lane, uint64_t pol,
                                                  uint4 &w0, uint4 &w1)
{
    const uint4 *zero = g_zero_pair + lane;
    const uint4 *a0 = pf.live ? pf.a + pf.t * 32 : zero;
    const uint4 *a1 = (pf.live && pf.h + pf.t < pf.P) ? a0 + pf.h * 32 : zero;
    w0 = ldg_weights(a0, pol);
    w1 = ldg_weights(a1, pol);
    if (!pf.live) return;
    if (++pf.t == pf.h) {
        pf.t = 0;
        if (--pf.rem > 0) {
            pf.a += pf.stride;
        } else if (++pf.s < s1) {
            const Seg sg = segs[pf.s];
            pf.seg(sg, lane, seg_stride(sg));
        } else {
            pf.live = false;
        }
    }
}

// ---------------------------------------------------------------------------
// Contraction 1: z_p = sum_k t_p[k] V_sign,p[k][.] for every latent row.  A
// unit is a row group over one 1024-input chunk (P = ceil(nkb / 2) pairs);
// its exact integer sums per (path, row) times 2^-E of the chunk go to
// float64 accumulators.  A segment lies in one chunk, so its exponents and B
// fragments serve all its units.
// ---------------------------------------------------------------------------
template <int MM>
static __device__ __noinline__ void c1_generic(const LayerDev *__restrict__ layers, const Seg1 *__restrict__ segs,
                                                  int s0, int s1, int M, int lane, uint64_t pol)
{
    const int g = lane >> 2, t4 = lane & 3;
    const int lane_m = t4 >> 1, lane_p = t4 & 1;        // accumulator columns of this lane
    const int blane = lane & (16 * MM - 1);

    Prefetch<Seg1> pf;
    pf.s = s0;
    pf.live = true;
    {
        const Seg1 sg = segs[s0];
        pf.seg(sg, lane, sg.rstride);
    }
    uint4 r0[kLdgRing], r1[kLdgRing];
#pragma unroll
    for (int d = 0; d < kLdgRing; ++d) fetch_step(pf, segs, s1, lane, pol, r0[d], r1[d]);

    dep_wait();     // B fragments, exponents and cleared accumulators come from the previous kernels

    // consumer: segment cs, row group crg, step ct of the unit
    int cs = s0, crg = 0, ct = 0, ch = 1, cP = 1, crem = 0, npaths = 1, r16 = 0;
    const uint4 *xb = nullptr;
    double *acc = nullptr;
    double lsc = 0.0;
    bool elive = false;
    auto seg_in = [&]() {
        const Seg1 sg = segs[cs];
        const LayerDev *dp = layers + sg.layer;
        crg = sg.rg0;
        crem = sg.n;
        cP = sg.P;
        ch = (cP + 1) >> 1;
        xb = reinterpret_cast<const uint4 *>(dp->xfrag) + (size_t)sg.kc * (kP1ChunkKB / 2) * 16 * MM + blane;
        acc = dp->acc;
        npaths = dp->npaths;
        r16 = dp->r16;
        const int E = (lane_m < M && lane_p < npaths) ? __ldcg(dp->xmeta + sg.kc * 4 + 2 * lane_p + lane_m) : kNanExp;
        elive = E != kNanExp;
        lsc = elive ? pow2d(-E) : 0.0;
    };
    seg_in();
    auto bload = [&](int t, uint4 &b0, uint4 &b1) {       // B pairs of step t (stream 1 clamped: its A is zero)
        b0 = ldg_frag(xb + (size_t)t * 16 * MM);
        b1 = ldg_frag(xb + (size_t)min(ch + t, cP - 1) * 16 * MM);
    };
    uint4 bn0, bn1;
    bload(0, bn0, bn1);
    int a4[4][4];
    zero_acc(a4);
    bool live = true;
    while (live) {
#pragma unroll
        for (int d = 0; d < kLdgRing; ++d) {
            if (live) {
                const uint4 w0 = r0[d], w1 = r1[d], b0 = bn0, b1 = bn1;
                fetch_step(pf, segs, s1, lane, pol, r0[d], r1[d]);
                const bool unit_end = ct + 1 == ch;
                bload(unit_end ? 0 : ct + 1, bn0, bn1);     // the next unit of the segment starts at step 0
                step_mma(a4, w0, w1, b0, b1);
                if (unit_end) {
                    // keep the columns of each row block's own path; partial sums over chunks add up exactly
                    if (elive) {
#pragma unroll
                        for (int rb = 0; rb < 4; ++rb) {
                            const int row0 = crg * kRowsPerGroup + rb * kRowsPerBlock;
                            const int prb = (npaths > 1 && row0 >= r16) ? 1 : 0;     // path 1 owns rows r16..
                            if (prb != lane_p) continue;
                            const int Tlo = (a4[rb][0] >> rb) + 256 * (a4[rb][1] >> rb);
                            const int Thi = (a4[rb][2] >> (rb + 4)) + 256 * (a4[rb][3] >> (rb + 4));
                            if (Tlo) atomicAdd(acc + (size_t)(row0 + g) * MM + lane_m, (double)Tlo * lsc);
                            if (Thi) atomicAdd(acc + (size_t)(row0 + g + 8) * MM + lane_m, (double)Thi * lsc);
                        }
                    }
                    zero_acc(a4);
                    ct = 0;
                    if (--crem > 0) {
                        ++crg;
                    } else if (++cs < s1) {
                        seg_in();
                        bload(0, bn0, bn1);
                    } else {
                        live = false;
                    }
                } else {
                    ++ct;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Contraction 2 (+ h, + path sum): y[m][n] = sum_p h_p[n] * sum_j U_sign,p[n][j] zl_p[m][j].
// Its epilogue keeps more state than contraction 1's, so its ring is one step shallower.
constexpr int kRing2 = kLdgRing - 1;
// A unit is a row group (P = KB2e / 2 pairs); the layer's B fragments serve every unit.
// ---------------------------------------------------------------------------
template <int MM>
static __device__ __noinline__ void c2_generic(const LayerDev *__restrict__ layers, const Seg2 *__restrict__ segs,
                                                  int s0, int s1, const IoPtrs &io, int base, int M, int lane,
                                                  uint64_t pol)
{
    const int g = lane >> 2, t4 = lane & 3;
    const int lane_m = t4 >> 1, lane_p = t4 & 1;
    const int blane = lane & (16 * MM - 1);
    const bool store = lane_p == 0 && lane_m < M;

    Prefetch<Seg2> pf;
    pf.s = s0;
    pf.live = true;
    {
        const Seg2 sg = segs[s0];
        pf.seg(sg, lane, sg.P * 32);
    }
    uint4 r0[kRing2], r1[kRing2];
#pragma unroll
    for (int d = 0; d < kRing2; ++d) fetch_step(pf, segs, s1, lane, pol, r0[d], r1[d]);

    // consumer: segment cs, row group crg, step ct of the unit
    int cs = s0, crg = 0, ct = 0, ch = 1, cP = 1, crem = 0, N = 0;
    const uint4 *hq = nullptr, *zb = nullptr;
    float *ym = nullptr;
    float my_sc = 0.0f, my_q = 0.0f;
    auto seg_w = [&]() {        // the weights side of a segment: no dependency on the previous kernel
        const Seg2 sg = segs[cs];
        crg = sg.rg0;
        crem = sg.n;
        cP = sg.P;
        ch = (cP + 1) >> 1;
        hq = sg.hq + lane_p * 8 + g;
        return sg.layer;
    };
    auto seg_b = [&](int layer) {   // the activation side: zl fragments and exponents of the finish kernel
        const LayerDev *dp = layers + layer;
        zb = reinterpret_cast<const uint4 *>(dp->zfrag) + blane;
        N = dp->N;
        ym = io.y[layer - base] + (size_t)lane_m * N;
        my_sc = my_q = 0.0f;
        if (lane_m < M && lane_p < dp->npaths) {
            const int2 mt = __ldcg(dp->zmeta + lane_p * 16 + lane_m);
            if (mt.x == kNanExp) {
                my_sc = my_q = __int_as_float(0x7fc00000);
            } else {
                my_sc = -2.0f * pow2f(-mt.x);                 // s = Q 2^-E - 2 T 2^-E
                my_q = (float)mt.y * pow2f(-mt.x);
            }
        }
    };
    const int layer0 = seg_w();
    uint4 hn = __ldg(hq);                   // the current unit's row scales

    dep_wait();     // the zl fragments and their exponents come from the finish kernel

    seg_b(layer0);
    auto bload = [&](int t, uint4 &b0, uint4 &b1) {       // B pairs of step t (stream 1 clamped: its A is zero)
        b0 = ldg_frag(zb + (size_t)t * 16 * MM);
        b1 = ldg_frag(zb + (size_t)min(ch + t, cP - 1) * 16 * MM);
    };
    uint4 bn0, bn1;
    bload(0, bn0, bn1);
    int a4[4][4];
    zero_acc(a4);
    bool live = true;
    while (live) {
#pragma unroll
        for (int d = 0; d < kRing2; ++d) {
            if (live) {
                const uint4 w0 = r0[d], w1 = r1[d], b0 = bn0, b1 = bn1;
                fetch_step(pf, segs, s1, lane, pol, r0[d], r1[d]);
                const bool unit_end = ct + 1 == ch;
                bload(unit_end ? 0 : ct + 1, bn0, bn1);     // the layer's fragments repeat for every unit
                step_mma(a4, w0, w1, b0, b1);
                if (unit_end) {
                    // lane (m, path): its path's share of rows g and g + 8, then the pair sum
                    const uint32_t hwv[4] = {hn.x, hn.y, hn.z, hn.w};
                    const int n0 = crg * kRowsPerGroup + g;
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const float2 hv = __half22float2(*reinterpret_cast<const __half2 *>(&hwv[rb]));
                        const int Tlo = (a4[rb][0] >> rb) + 256 * (a4[rb][1] >> rb);
                        const int Thi = (a4[rb][2] >> (rb + 4)) + 256 * (a4[rb][3] >> (rb + 4));
                        float vlo = hv.x * fmaf((float)Tlo, my_sc, my_q);
                        float vhi = hv.y * fmaf((float)Thi, my_sc, my_q);
                        vlo += __shfl_xor_sync(0xffffffffu, vlo, 1);
                        vhi += __shfl_xor_sync(0xffffffffu, vhi, 1);
                        const int nlo = n0 + rb * kRowsPerBlock;
                        if (store) {
                            if (nlo < N) ym[nlo] = vlo;
                            if (nlo + 8 < N) ym[nlo + 8] = vhi;
                        }
                    }
                    zero_acc(a4);
                    ct = 0;
                    if (--crem > 0) {
                        ++crg;
                        hq += 16;
                        hn = __ldg(hq);
                    } else if (++cs < s1) {
                        seg_b(seg_w());
                        hn = __ldg(hq);
                        bload(0, bn0, bn1);
                    } else {
                        live = false;
                    }
                } else {
                    ++ct;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Static unit structure.  When every unit of a warp takes the same number H
// of steps, the warp runs blocks of U units (L = U H steps, fully unrolled):
// the ring holds one block, the prefetcher loads the next block at the same
// positions, and every unit boundary, B index and epilogue sits at a
// compile-time position, so the only branches are at block ends.  The last
// block of a segment may hold fewer than U units: the rest read zeros and
// store nothing.  The plan gives each warp units of one step count; counts
// without a static path take the generic loops above.
// ---------------------------------------------------------------------------

// The largest unit of a static path: 2H pairs of k-blocks (contraction 2, H = 13).
constexpr int kStaticMaxPairs = 26;
// Zeros: the weights of a unit past a segment's end or the warp's range (a unit has at most kStaticMaxPairs
// pairs), so that each ring load is one address plus an immediate offset.
static __device__ __align__(16) uint4 g_zero_unit[kStaticMaxPairs * 32];

// A cursor over a warp's segments in blocks of U units, with this lane's address of each unit's first pair.
static __device__ __forceinline__ const uint4 *seg_a(const Seg1 &x) { return x.v; }
static __device__ __forceinline__ const uint4 *seg_a(const Seg2 &x) { return x.u; }

template <typename Seg, int U>
struct BlockCur {
    int s, k, n, stride;    // segment index, first unit of the block, units in the segment, uint4 between units
    bool live;
    const uint4 *base;      // this lane's address of the segment's first unit's first pair
    const uint4 *ub[U];
    __device__ __forceinline__ void seg_load(const Seg *segs, int lane)
    {
        const Seg sg = segs[s];
        base = seg_a(sg) + lane;
        n = sg.n;
        stride = seg_stride(sg);
    }
    __device__ __forceinline__ void bases(int lane)
    {
#pragma unroll
        for (int j = 0; j < U; ++j)
            ub[j] = (live && k + j < n) ? base + (size_t)(k + j) * stride : g_zero_unit + lane;
    }
    __device__ __forceinline__ void start(const Seg *segs, int s0, int lane)
    {
        s = s0;
        k = 0;
        live = true;
        seg_load(segs, lane);
        bases(lane);
    }
    // returns true when the block moved to another segment
    __device__ __forceinline__ bool next(const Seg *segs, int s1, int lane)
    {
        k += U;
        bool moved = false;
        if (k >= n) {
            k = 0;
            moved = true;
            if (++s < s1) seg_load(segs, lane);
            else live = false;
        }
        bases(lane);
        return moved;
    }
};

// Step t of a unit whose first pair this lane reads at ub: pair t (stream 0) and H + t (stream 1).  Where a
// unit has only 2H - 1 pairs, stream 1's last load reads the 512 bytes after the unit (the tile arrays are padded
// by one pair); its B fragment is zero there, so nothing of it counts.
template <int H>
static __device__ __forceinline__ void fetch_unit_step(const uint4 *ub, int t, uint64_t pol, uint4 &w0, uint4 &w1)
{
    w0 = ldg_weights(ub + t * 32, pol);
    w1 = ldg_weights(ub + (H + t) * 32, pol);
}

// The ring load at block position i: step i + D of the stream, in this block (cur) or the next one (nxt).
template <int H, int U, int D, typename Seg>
static __device__ __forceinline__ void fetch_ahead(const BlockCur<Seg, U> &cur, const BlockCur<Seg, U> &nxt, int i,
                                                   uint64_t pol, uint4 &w0, uint4 &w1)
{
    constexpr int L = H * U;
    const int j = i + D;
    if (j < L) fetch_unit_step<H>(cur.ub[j / H], j % H, pol, w0, w1);
    else fetch_unit_step<H>(nxt.ub[(j - L) / H], (j - L) % H, pol, w0, w1);
}

// B fragments of the static paths live in the warp's shared-memory slot: 2H pairs of 16 MM lanes, copied from
// global memory (through L2: the previous kernel wrote them) whenever the warp enters a segment; where the units
// have only 2H - 1 pairs, the last pair of the slot is zero, so stream 1's extra load counts for nothing.
constexpr int kSlotPairs1 = kP1ChunkKB / 2;     // contraction 1: one 1024-input chunk
constexpr int kSlotPairs2 = kStaticMaxPairs;    // contraction 2: the deepest static unit

static __device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

static __device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
// Each warp owns a region of the CTA's shared memory.  Contraction 1: one slot of two-row fragments, or two slots
// of one-row fragments (the next segment's fragments are fetched into the second while the first is read).
// Contraction 2: one slot of kSlotPairs2 pairs.
constexpr uint32_t kSlotBytes1 = kSlotPairs1 * 16 * 16;      // one contraction-1 slot, one activation row
constexpr uint32_t kRegion1 = 2 * kSlotBytes1;
template <int MM>
__host__ __device__ constexpr uint32_t region2() { return kSlotPairs2 * 16 * MM * 16; }
template <int MM>
static __device__ __forceinline__ uint32_t b_slot(int warp, uint32_t region)
{
    extern __shared__ __align__(16) unsigned char sm_raw[];
    return sm_addr(sm_raw) + (uint32_t)warp * region;
}

// 16-byte asynchronous copy global -> shared through L2 (data of the previous launch: never the read-only path)
static __device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
static __device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
static __device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
template <int MM, int H>
static __device__ __forceinline__ void b_fill(uint32_t slot, const uint4 *src, int P, int lane)
{
    __syncwarp();      // every lane is done with the slot's previous contents
#pragma unroll
    for (int i = lane; i < 2 * H * 16 * MM; i += 32) {
        const uint4 v = (i < P * 16 * MM) ? __ldcg(src + i) : make_uint4(0u, 0u, 0u, 0u);
        sts128(slot + (uint32_t)i * 16, v);
    }
    __syncwarp();
}
template <int MM, int H>
static __device__ __forceinline__ void b_read(uint32_t bsl, int t, uint4 &b0, uint4 &b1)
{
    b0 = lds128(bsl + (uint32_t)t * 16 * MM * 16);
    b1 = lds128(bsl + (uint32_t)(H + t) * 16 * MM * 16);
}

// Blocks of U units (L = U H steps, unrolled), a ring of D steps (D divides L): the ring slot of block position
// i is i % D, refilled with step i + D once consumed.
template <int MM, int H, int U, int D>
static __device__ __noinline__ void c1_static(const LayerDev *__restrict__ layers, const Seg1 *__restrict__ segs,
                                              int s0, int s1, int M, int lane, int warp, uint64_t pol)
{
    constexpr int L = H * U;
    static_assert(L % D == 0 && D <= L, "ring");
    const int g = lane >> 2, t4 = lane & 3;
    const int lane_m = t4 >> 1, lane_p = t4 & 1;
    const int blane = lane & (16 * MM - 1);

    BlockCur<Seg1, U> cc, nb;       // the block being computed and the one after it
    cc.start(segs, s0, lane);
    nb = cc;
    nb.next(segs, s1, lane);
    uint4 r0[D], r1[D];
#pragma unroll
    for (int i = 0; i < D; ++i) fetch_unit_step<H>(cc.ub[i / H], i % H, pol, r0[i], r1[i]);

    dep_wait();     // B fragments, exponents and cleared accumulators come from the previous kernels

    static_assert(2 * H <= kSlotPairs1 && kSlotPairs1 * 16 * MM * 16 <= kRegion1, "contraction-1 slot");
    const uint32_t slot = b_slot<MM>(warp, kRegion1);
    uint32_t bsl = slot + blane * 16;
    double *acc = nullptr;
    int npaths = 1, r16 = 0;
    double lsc = 0.0;
    bool elive = false;
    int rg0 = 0;
    // one row: segment s + 1's fragments (cp.async into the other slot), exponent and layer fields are fetched
    // when segment s starts, so that entering a segment waits for nothing but copies issued a segment earlier
    int par = 0;                     // slot of the current segment
    double *n_acc = nullptr;
    int n_npaths = 1, n_r16 = 0, n_rg0 = 0, n_E = kNanExp;
    auto prefetch = [&](int s, uint32_t dst) {
        const Seg1 sg = segs[s];
        const LayerDev *dp = layers + sg.layer;
        const uint4 *src = reinterpret_cast<const uint4 *>(dp->xfrag) + (size_t)sg.kc * (kP1ChunkKB / 2) * 16 * MM;
#pragma unroll
        for (int i = lane; i < 2 * H * 16 * MM; i += 32) {
            if (i < sg.P * 16 * MM) cp_async16(dst + (uint32_t)i * 16, src + i);
            else sts128(dst + (uint32_t)i * 16, make_uint4(0u, 0u, 0u, 0u));
        }
        cp_async_commit();
        n_rg0 = sg.rg0;
        n_acc = dp->acc;
        n_npaths = dp->npaths;
        n_r16 = dp->r16;
        n_E = (lane_m < M && lane_p < n_npaths) ? __ldcg(dp->xmeta + sg.kc * 4 + 2 * lane_p + lane_m) : kNanExp;
    };
    auto seg_in = [&]() {
        if constexpr (MM == 1) {
            cp_async_wait_all();     // this segment's fragments (fetched a segment ago) have landed
            __syncwarp();            // ... for every lane, and every lane is done with the other slot
            bsl = slot + (uint32_t)par * kSlotBytes1 + blane * 16;
            rg0 = n_rg0;
            acc = n_acc;
            npaths = n_npaths;
            r16 = n_r16;
            elive = n_E != kNanExp;
            lsc = elive ? pow2d(-n_E) : 0.0;
            par ^= 1;
            if (cc.s + 1 < s1) prefetch(cc.s + 1, slot + (uint32_t)par * kSlotBytes1);
        } else {
            const Seg1 sg = segs[cc.s];
            const LayerDev *dp = layers + sg.layer;
            b_fill<MM, H>(slot, reinterpret_cast<const uint4 *>(dp->xfrag) + (size_t)sg.kc * (kP1ChunkKB / 2) * 16 * MM,
                          sg.P, lane);
            rg0 = sg.rg0;
            acc = dp->acc;
            npaths = dp->npaths;
            r16 = dp->r16;
            const int E = (lane_m < M && lane_p < npaths) ? __ldcg(dp->xmeta + sg.kc * 4 + 2 * lane_p + lane_m)
                                                         : kNanExp;
            elive = E != kNanExp;
            lsc = elive ? pow2d(-E) : 0.0;
        }
    };
    if constexpr (MM == 1) prefetch(s0, slot);
    seg_in();
    int a4[4][4];
    zero_acc(a4);
    while (cc.live) {
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int k = i / H, t = i % H;
            const uint4 w0 = r0[i % D], w1 = r1[i % D];
            uint4 b0, b1;
            b_read<MM, H>(bsl, t, b0, b1);
            fetch_ahead<H, U, D>(cc, nb, i, pol, r0[i % D], r1[i % D]);
            step_mma(a4, w0, w1, b0, b1);
            if (t == H - 1) {
                // unit k: keep the columns of each row block's own path; partial sums over chunks add up exactly
                if (elive && cc.k + k < cc.n) {
                    const int rowg = (rg0 + cc.k + k) * kRowsPerGroup;
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const int row0 = rowg + rb * kRowsPerBlock;
                        const int prb = (npaths > 1 && row0 >= r16) ? 1 : 0;     // path 1 owns rows r16..
                        if (prb != lane_p) continue;
                        const int Tlo = (a4[rb][0] >> rb) + 256 * (a4[rb][1] >> rb);
                        const int Thi = (a4[rb][2] >> (rb + 4)) + 256 * (a4[rb][3] >> (rb + 4));
                        if (Tlo) atomicAdd(acc + (size_t)(row0 + g) * MM + lane_m, (double)Tlo * lsc);
                        if (Thi) atomicAdd(acc + (size_t)(row0 + g + 8) * MM + lane_m, (double)Thi * lsc);
                    }
                }
                zero_acc(a4);
            }
        }
        const bool moved = cc.next(segs, s1, lane);
        nb.next(segs, s1, lane);
        if (moved && cc.live) seg_in();
    }
}

template <int MM, int H, int U, int D>
static __device__ __noinline__ void c2_static(const LayerDev *__restrict__ layers, const Seg2 *__restrict__ segs,
                                              int s0, int s1, const IoPtrs &io, int base, int M, int lane, int warp,
                                              uint64_t pol)
{
    constexpr int L = H * U;
    static_assert(L % D == 0 && D <= L, "ring");
    const int g = lane >> 2, t4 = lane & 3;
    const int lane_m = t4 >> 1, lane_p = t4 & 1;
    const int blane = lane & (16 * MM - 1);
    const bool store = lane_p == 0 && lane_m < M;

    BlockCur<Seg2, U> cc, nb;
    cc.start(segs, s0, lane);
    nb = cc;
    nb.next(segs, s1, lane);
    uint4 r0[D], r1[D];
#pragma unroll
    for (int i = 0; i < D; ++i) fetch_unit_step<H>(cc.ub[i / H], i % H, pol, r0[i], r1[i]);

    dep_wait();     // the zl fragments and their exponents come from the finish kernel

    static_assert(2 * H <= kSlotPairs2, "contraction-2 slot");
    const uint32_t slot = b_slot<MM>(warp, region2<MM>()), bsl = slot + blane * 16;
    int N = 0;
    float *ym = nullptr;
    float my_sc = 0.0f, my_q = 0.0f;
    int rg0 = 0;
    const uint4 *hq = nullptr;
    auto seg_in = [&]() {
        const Seg2 sg = segs[cc.s];
        const LayerDev *dp = layers + sg.layer;
        b_fill<MM, H>(slot, reinterpret_cast<const uint4 *>(dp->zfrag), sg.P, lane);
        rg0 = sg.rg0;
        hq = sg.hq + lane_p * 8 + g;
        N = dp->N;
        ym = io.y[sg.layer - base] + (size_t)lane_m * N;
        my_sc = my_q = 0.0f;
        if (lane_m < M && lane_p < dp->npaths) {
            const int2 mt = __ldcg(dp->zmeta + lane_p * 16 + lane_m);
            if (mt.x == kNanExp) {
                my_sc = my_q = __int_as_float(0x7fc00000);
            } else {
                my_sc = -2.0f * pow2f(-mt.x);                 // s = Q 2^-E - 2 T 2^-E
                my_q = (float)mt.y * pow2f(-mt.x);
            }
        }
    };
    seg_in();
    uint4 hn = make_uint4(0u, 0u, 0u, 0u);
    int a4[4][4];
    zero_acc(a4);
    while (cc.live) {
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int k = i / H, t = i % H;
            const uint4 w0 = r0[i % D], w1 = r1[i % D];
            uint4 b0, b1;
            b_read<MM, H>(bsl, t, b0, b1);
            fetch_ahead<H, U, D>(cc, nb, i, pol, r0[i % D], r1[i % D]);
            if (t == 0)     // the unit's row scales (a unit past the segment's end reads the block's first unit's)
                hn = __ldg(hq + (size_t)(cc.k + (cc.k + k < cc.n ? k : 0)) * 16);
            step_mma(a4, w0, w1, b0, b1);
            if (t == H - 1) {
                // unit k, lane (m, path): its path's share of rows g and g + 8, then the pair sum
                const bool st = store && cc.k + k < cc.n;
                const uint32_t hwv[4] = {hn.x, hn.y, hn.z, hn.w};
                const int n0 = (rg0 + cc.k + k) * kRowsPerGroup + g;
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const float2 hv = __half22float2(*reinterpret_cast<const __half2 *>(&hwv[rb]));
                    const int Tlo = (a4[rb][0] >> rb) + 256 * (a4[rb][1] >> rb);
                    const int Thi = (a4[rb][2] >> (rb + 4)) + 256 * (a4[rb][3] >> (rb + 4));
                    float vlo = hv.x * fmaf((float)Tlo, my_sc, my_q);
                    float vhi = hv.y * fmaf((float)Thi, my_sc, my_q);
                    vlo += __shfl_xor_sync(0xffffffffu, vlo, 1);
                    vhi += __shfl_xor_sync(0xffffffffu, vhi, 1);
                    const int nlo = n0 + rb * kRowsPerBlock;
                    if (st && nlo < N) ym[nlo] = vlo;
                    if (st && nlo + 8 < N) ym[nlo + 8] = vhi;
                }
                zero_acc(a4);
            }
        }
        const bool moved = cc.next(segs, s1, lane);
        nb.next(segs, s1, lane);
        if (moved && cc.live) seg_in();
    }
}

// Per warp: its units' step count (a static path) or 0 (the generic loop).
template <int MM>
__global__ void __launch_bounds__(kLdgWarps * 32, 1)
    contraction1_ldg_kernel(const LayerDev *__restrict__ layers, const Seg1 *__restrict__ segs,
                            const int *__restrict__ bnd, const int *__restrict__ cls, int M)
{
    dep_release();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kLdgWarps + (threadIdx.x >> 5);
    const int s0 = bnd[gw], s1 = bnd[gw + 1];
    if (s0 >= s1) return;
    const uint64_t pol = l2_evict_first();
    switch (cls[gw]) {
    case 6: c1_static<MM, 6, 2, 4>(layers, segs, s0, s1, M, lane, threadIdx.x >> 5, pol); break;
    case 8: c1_static<MM, 8, 1, 4>(layers, segs, s0, s1, M, lane, threadIdx.x >> 5, pol); break;
    default: c1_generic<MM>(layers, segs, s0, s1, M, lane, pol); break;
    }
}

template <int MM>
__global__ void __launch_bounds__(kLdgWarps * 32, 1)
    contraction2_ldg_kernel(const LayerDev *__restrict__ layers, const Seg2 *__restrict__ segs,
                            const int *__restrict__ bnd, const int *__restrict__ cls, const __grid_constant__ IoPtrs io,
                            int base, int M)
{
    dep_release();
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kLdgWarps + (threadIdx.x >> 5);
    const int s0 = bnd[gw], s1 = bnd[gw + 1];
    if (s0 >= s1) return;
    const uint64_t pol = l2_evict_first();
    switch (cls[gw]) {
    case 1: c2_static<MM, 1, 6, 6>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 2: c2_static<MM, 2, 3, 6>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 3: c2_static<MM, 3, 2, 6>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 4: c2_static<MM, 4, 3, 6>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 5: c2_static<MM, 5, 1, 5>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 6: c2_static<MM, 6, 1, 6>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 9: c2_static<MM, 9, 2, 6>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    case 13: c2_static<MM, 13, 5, 5>(layers, segs, s0, s1, io, base, M, lane, threadIdx.x >> 5, pol); break;
    default: c2_generic<MM>(layers, segs, s0, s1, io, base, M, lane, pol); break;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

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

template <int MM>
static lb_status pair_launch_mm(const LayerDev *dev_layers, int nlayers, const P1Item *p1, int n1, const Plan &P,
                                int batch, const IoPtrs &io, int base, int M, int kb2max, int rmax, cudaStream_t s,
                                int *launches, bool mark)
{
    cudaError_t e;
    const int G = P.stream_grid;
    if (G < 1 || kb2max > kPairMaxKB2 || (size_t)2 * rmax * MM * sizeof(float) > 48 * 1024) return LB_ERR_UNSUPPORTED;
    const int nw = G * kLdgWarps;
    const int *bnd1 = P.bnd1 + (size_t)batch * (nw + 1);
    const int *bnd2 = P.bnd2 + (size_t)batch * (nw + 1);
    const int *cls1 = P.cls1 + (size_t)batch * nw, *cls2 = P.cls2 + (size_t)batch * nw;
    if (n1 > 0) {
        quantize_pair_kernel<MM><<<(n1 + kQuantWarps - 1) / kQuantWarps, kQuantWarps * 32, 0, s>>>(dev_layers, p1, n1, io,
                                                                                                  base, M);
        ++*launches;
        if (mark) profile_mark(*launches, s);
    }
    // the three kernels after the quantisation may each start while the previous one drains,
    // unless timing events separate the launches
    const bool pdl = !profiling_active();
    const size_t slots1 = (size_t)kLdgWarps * kRegion1, slots2 = (size_t)kLdgWarps * region2<MM>();   // B slots
    if ((e = ensure_dyn_smem((const void *)contraction1_ldg_kernel<MM>, slots1)) != cudaSuccess ||
        (e = ensure_dyn_smem((const void *)contraction2_ldg_kernel<MM>, slots2)) != cudaSuccess)
        return status_from(e);
    if ((e = launch_dependent(pdl, contraction1_ldg_kernel<MM>, dim3(G), dim3(kLdgWarps * 32), slots1, s, dev_layers,
                              (const Seg1 *)P.sg1, bnd1, cls1, M)) != cudaSuccess)
        return status_from(e);
    ++*launches;
    if (mark) profile_mark(*launches, s);
    if ((e = launch_dependent(pdl, finish_pair_kernel<MM>, dim3(nlayers), dim3(kFinishThreads),
                              (size_t)2 * rmax * MM * sizeof(float), s, dev_layers, base, M)) != cudaSuccess)
        return status_from(e);
    ++*launches;
    if (mark) profile_mark(*launches, s);
    if ((e = launch_dependent(pdl, contraction2_ldg_kernel<MM>, dim3(G), dim3(kLdgWarps * 32), slots2, s, dev_layers,
                              (const Seg2 *)P.sg2, bnd2, cls2, io, base, M)) != cudaSuccess)
        return status_from(e);
    ++*launches;
    if (mark) profile_mark(*launches, s);
    return status_from(cudaGetLastError());
}

lb_status decode_pair_launch(const LayerDev *dev_layers, int nlayers, const P1Item *p1, int n1, const Plan &P,
                             int batch, const IoPtrs &io, int base, int M, int kb2max, int rmax, int *err,
                             cudaStream_t s, int *launches, bool mark)
{
    (void)err;     // these kernels wait on nothing but their predecessors' completion
    if (M == 1)
        return pair_launch_mm<1>(dev_layers, nlayers, p1, n1, P, batch, io, base, M, kb2max, rmax, s, launches, mark);
    return pair_launch_mm<2>(dev_layers, nlayers, p1, n1, P, batch, io, base, M, kb2max, rmax, s, launches, mark);
}

}  // namespace lb

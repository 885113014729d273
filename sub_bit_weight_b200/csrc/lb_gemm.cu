// D = alpha * A^T B on 5th-generation tensor cores: fp16 operands, fp32
// accumulation in tensor memory, fp32 output.
//
// The factor gradients of the QAT backward pass (LittleBit notes page, "Loss /
// training strategy": SmoothSign, backward through tanh(100 u)) need
//     G_U = dy^T zl   ([N][paths * r], contracted over the batch rows)
//     G_V = x^T  dz   ([K][paths * r])
// whose operands are activations stored row-major [batch row][feature]: the
// contracted index is the slow one in both, so both operands enter the tensor
// core MN-major (feature index contiguous), straight from the TMA copies:
//
//   A tile  128 i x 64 k : two 64-wide slices, each [64 k rows][128 bytes]
//   B tile  256 j x 64 k : four such slices
//   (128-byte swizzle; a slice is one TMA box; slices 8 KB apart)
//
// Kernel structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer (one thread), 4-stage ring, one mbarrier per stage
//   warp 1      tensor-memory owner; one thread issues tcgen05.mma (M = 128,
//               N = 256, K = 16) and commits each stage back to the producer
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (32 rows x 32 columns
//               per warp and step), times alpha, through a 128-byte-swizzled
//               staging block, one TMA store per block (clipped at the edges)
// Two 256-column accumulators let the epilogue of one tile overlap the main
// loop of the next.  One launch may carry two problems (G_U and G_V): their
// tiles form one list dealt round-robin to the CTAs, so the smaller problem
// fills the other's last partial wave.  Every wait is bounded: on timeout the
// kernel records an error code in *err and returns.

#include <algorithm>
#include <cstring>

#include "lb_internal.cuh"
#include "lb_tc.cuh"
#include "littlebit_backward.h"

namespace lb {
namespace {

constexpr int kGBM = 128;      // i per tile (UMMA M)
constexpr int kGBN = 256;      // j per tile (UMMA N, at most)
constexpr int kGBK = 64;       // k rows per stage
constexpr int kGStages = 4;
constexpr int kGThreads = 192;
constexpr uint32_t kSlice = kGBK * 128;   // bytes of one 64-wide slice of a stage

struct GemmSmem {
    alignas(1024) unsigned char A[kGStages][kGBM / 64 * kSlice];
    alignas(1024) unsigned char B[kGStages][kGBN / 64 * kSlice];
    alignas(1024) unsigned char ST[4][32 * 128];   // one 32 x 32 fp32 staging block per epilogue warp
    uint64_t full[kGStages], empty[kGStages];
    uint64_t accf[2], acce[2];
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kGemmSmemBytes = sizeof(GemmSmem) + 1024;

// One problem of a launch: maps of A [Kc][Mr], B [Kc][Nc] (fp16) and D [Mr][Nc] (fp32), its sizes, and the first
// index of its tiles in the launch's tile list.
struct GemmProb {
    CUtensorMap mA, mB, mD;
    const float *alpha;
    int Kc, Mr, Nc, ntj, nkb, tile0;
};
constexpr int kGemmMaxProbs = 2;
struct GemmBatch {
    GemmProb p[kGemmMaxProbs];
    int n, ntiles;
};

// fp16 A and B, both MN-major; fp32 accumulator; M = 128, N = n
__device__ __forceinline__ uint32_t idesc_f16_mn(int n)
{
    return (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kGBM >> 4) << 24);
}

__global__ void __launch_bounds__(kGThreads, 1) gemm_at_b_kernel(const __grid_constant__ GemmBatch G, int *err)
{
    extern __shared__ __align__(1024) unsigned char g_raw[];
    const uint32_t raw_addr = smem_u32(g_raw);
    GemmSmem &S = *reinterpret_cast<GemmSmem *>(g_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&S.full[s], 1);
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
    const int ntiles = G.ntiles;

    // tile t -> problem q, (i tile, j tile) = (local / ntj, local % ntj): the CTAs in flight share a few i tiles of
    // A, and B (the latent side, small) stays in L2
    auto locate = [&](int t, int &q, int &i0, int &j0) {
        q = (G.n > 1 && t >= G.p[1].tile0) ? 1 : 0;
        const int local = t - G.p[q].tile0, ntj = G.p[q].ntj;
        i0 = (local / ntj) * kGBM;
        j0 = (local % ntj) * kGBN;
    };

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            uint32_t it = 0, pend = 0, pend_ph = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
                int q, i0, j0;
                locate(t, q, i0, j0);
                const GemmProb &P = G.p[q];
                const int na = min(kGBM / 64, (P.Mr - i0 + 63) / 64);   // slices with at least one row in range
                const int nb = min(kGBN / 64, (P.Nc - j0 + 63) / 64);
                for (int kb = 0; kb < P.nkb; ++kb, ++it) {
                    const int s = it % kGStages;
                    const uint32_t ph = (it / kGStages) & 1;
                    if (!mbar_wait(&S.empty[s], ph ^ 1, abort, err, 1)) break;
                    mbar_expect_tx(&S.full[s], (uint32_t)(na + nb) * kSlice);
                    for (int b = 0; b < na; ++b) tma_load_2d(S.A[s] + b * kSlice, &P.mA, i0 + 64 * b, kb * kGBK, &S.full[s]);
                    for (int b = 0; b < nb; ++b) tma_load_2d(S.B[s] + b * kSlice, &P.mB, j0 + 64 * b, kb * kGBK, &S.full[s]);
                    pend |= 1u << s;
                    pend_ph = (pend_ph & ~(1u << s)) | (ph << s);
                }
            }
            if (*abort) {
                // let the copies already issued land before the CTA leaves (bounded)
                for (int s = 0; s < kGStages; ++s) {
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
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tcount) {
                int q, i0, j0;
                locate(t, q, i0, j0);
                const int nkb = G.p[q].nkb;
                const int nw = min(kGBN, G.p[q].Nc - j0);
                const int ab = tcount & 1;
                const uint32_t aph = (tcount >> 1) & 1;
                if (!mbar_wait(&S.acce[ab], aph ^ 1, abort, err, 2)) break;
                tc_fence_after();
                const uint32_t idesc = idesc_f16_mn((nw + 15) & ~15);
                const uint32_t dacc = tmem + (uint32_t)(ab * kGBN);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kGStages;
                    const uint32_t ph = (it / kGStages) & 1;
                    if (!mbar_wait(&S.full[s], ph, abort, err, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // 16 k rows = two 8-row swizzle groups = 2048 bytes per MMA step
#pragma unroll
                    for (int kk = 0; kk < kGBK / 16; ++kk)
                        tc_mma_f16(dacc, smem_desc_mn_sw128(S.A[s] + kk * 2048, kSlice),
                                   smem_desc_mn_sw128(S.B[s] + kk * 2048, kSlice), idesc, (kb || kk) ? 1u : 0u);
                    tc_commit(&S.empty[s]);
                }
                if (!ok) break;
                tc_commit(&S.accf[ab]);
            }
        }
    } else {
        // ---------------- epilogue (warps 2-5: tensor-memory lanes 32 (warp % 4) ..)
        const int q4 = warp & 3;
        float f[kGemmMaxProbs];
        for (int q = 0; q < G.n; ++q) f[q] = __ldg(G.p[q].alpha);
        uint32_t tcount = 0;
        bool stored = false;
        for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tcount) {
            int q, i0, j0;
            locate(t, q, i0, j0);
            const GemmProb &P = G.p[q];
            const float fq = q ? f[1] : f[0];
            const int nw = min(kGBN, P.Nc - j0);
            const int ab = tcount & 1;
            const uint32_t aph = (tcount >> 1) & 1;
            if (!mbar_wait(&S.accf[ab], aph, abort, err, 4)) break;
            tc_fence_after();
            const uint32_t sta = smem_u32(S.ST[q4]);
            for (int ch = 0; ch < nw; ch += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(ab * kGBN + ch), v);
                if (stored) {   // the previous store has finished reading the staging block
                    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
                    __syncwarp();
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    sts128(sta + sw128(lane, i),
                           make_uint4(__float_as_uint(__uint_as_float(v[4 * i]) * fq),
                                      __float_as_uint(__uint_as_float(v[4 * i + 1]) * fq),
                                      __float_as_uint(__uint_as_float(v[4 * i + 2]) * fq),
                                      __float_as_uint(__uint_as_float(v[4 * i + 3]) * fq)));
                fence_proxy_async();
                __syncwarp();
                if (lane == 0 && i0 + q4 * 32 < P.Mr) {
                    asm volatile(
                        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(&P.mD),
                        "r"(j0 + ch), "r"(i0 + q4 * 32), "r"(sta)
                        : "memory");
                    asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
                }
                stored = true;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.acce[ab]);
        }
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem));
    }
}

}  // namespace

static lb_status check_desc(const GemmDesc &d)
{
    if (!d.A || !d.B || !d.D || !d.alpha || d.Kc < 0 || d.Mr < 0 || d.Nc < 0) return LB_ERR_INVALID_ARG;
    if (d.Mr == 0 || d.Nc == 0) return LB_OK;
    if (d.lda < d.Mr || d.ldb < d.Nc || d.ldd < d.Nc) return LB_ERR_INVALID_ARG;
    if (((uintptr_t)d.A | (uintptr_t)d.B | (uintptr_t)d.D) & 15) return LB_ERR_INVALID_ARG;
    if (d.lda % 8 || d.ldb % 8 || d.ldd % 4 || d.Nc % 32) return LB_ERR_UNSUPPORTED;
    if (d.Kc == 0) return LB_ERR_UNSUPPORTED;   // an empty contraction: the caller zeroes D itself
    return LB_OK;
}

lb_status gemm_at_b_batch(const GemmDesc *descs, int n, int *err, cudaStream_t s)
{
    if (!descs || !err || n < 1 || n > kGemmMaxProbs) return LB_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const lb_status st = check_desc(descs[i]);
        if (st != LB_OK) return st;
    }
    GemmBatch G;
    memset(&G, 0, sizeof(G));
    bool encoder = false;
    for (int i = 0; i < n; ++i) {
        const GemmDesc &d = descs[i];
        if (d.Mr == 0 || d.Nc == 0) continue;     // nothing to do for this one
        if (!encoder) {
            if (tmap_encoder_ready() != cudaSuccess) return LB_ERR_UNSUPPORTED;
            encoder = true;
        }
        GemmProb &P = G.p[G.n];
        if (!tmap_encode_2d(&P.mA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d.A, d.Mr, d.Kc, (long)d.lda * 2, 64, kGBK) ||
            !tmap_encode_2d(&P.mB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, d.B, d.Nc, d.Kc, (long)d.ldb * 2, 64, kGBK) ||
            !tmap_encode_2d(&P.mD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d.D, d.Nc, d.Mr, (long)d.ldd * 4, 32, 32))
            return LB_ERR_INVALID_ARG;
        P.alpha = d.alpha;
        P.Kc = d.Kc;
        P.Mr = d.Mr;
        P.Nc = d.Nc;
        P.ntj = (d.Nc + kGBN - 1) / kGBN;
        P.nkb = (d.Kc + kGBK - 1) / kGBK;
        P.tile0 = G.ntiles;
        const long tiles = (long)((d.Mr + kGBM - 1) / kGBM) * P.ntj;
        if (G.ntiles + tiles > (1L << 30)) return LB_ERR_UNSUPPORTED;
        G.ntiles += (int)tiles;
        ++G.n;
    }
    if (G.n == 0) return LB_OK;
    cudaError_t e = ensure_dyn_smem((const void *)gemm_at_b_kernel, kGemmSmemBytes);
    if (e != cudaSuccess) return status_from(e);
    int sms = 0;
    if ((e = sm_count_of_current(&sms)) != cudaSuccess) return status_from(e);
    const int grid = std::min(G.ntiles, sms);
    gemm_at_b_kernel<<<grid, kGThreads, kGemmSmemBytes, s>>>(G, err);
    return status_from(cudaGetLastError());
}

lb_status gemm_at_b(const void *A, int lda, const void *B, int ldb, float *D, int ldd, int Kc, int Mr, int Nc,
                    const float *alpha, int *err, cudaStream_t s)
{
    const GemmDesc d{A, lda, B, ldb, D, ldd, Kc, Mr, Nc, alpha};
    if (!err) return LB_ERR_INVALID_ARG;
    return gemm_at_b_batch(&d, 1, err, s);
}

}  // namespace lb

extern "C" lb_status lb_gemm_at_b(const uint16_t *A, int lda, const uint16_t *B, int ldb, float *D, int ldd, int Kc,
                                  int Mr, int Nc, const float *alpha, int *err, void *stream)
{
    lb::set_launch_count(0);
    const lb_status st = lb::gemm_at_b(A, lda, B, ldb, D, ldd, Kc, Mr, Nc, alpha, err, (cudaStream_t)stream);
    if (st == LB_OK && Mr > 0 && Nc > 0) lb::set_launch_count(1);
    return st;
}

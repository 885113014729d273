// Internal declarations of the LittleBit CUDA library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <vector>

#include "littlebit.h"

namespace lb {

// ---------------------------------------------------------------------------
// Decode-path tiling (the fused small-batch kernels).
//
// Both binary contractions run on integer tensor cores (mma.sync m16n8k32,
// A = unsigned 8-bit, B = signed 8-bit, s32 accumulate).  The weight is the A
// operand ("row" = an output of the contraction, "k" = the contracted index),
// the activations are the B operand as two balanced base-256 digits of a
// 16-bit fixed-point value (column = 2*m + digit).
//
// A "unit" is 64 rows x 32 k of one weight matrix, stored as 256 contiguous
// bytes: lane L (g = L >> 2, t = L & 3) owns the uint2 {w0, w1}.  Bit i of
// byte b of word q is the sign bit (1 = -1) of
//     row = 16 * (i & 3) + g + 8 * (i >> 2),   k = 4 * t + b + 16 * q.
// Masking a word with (0x01010101 << i) gives four u8 A elements equal to
// 2^i times the bit, in exactly the register slots mma.sync expects, so a
// row-block's MMA costs four LOP3s and no shifts:
//     row-block rb:  a0 = w0 & m(rb)   a1 = w0 & m(rb + 4)
//                    a2 = w1 & m(rb)   a3 = w1 & m(rb + 4)
// Rows g of row-block rb then carry the factor 2^rb and rows g + 8 the factor
// 2^(rb+4); both are divided out exactly after accumulation.
// ---------------------------------------------------------------------------
constexpr int kRowsPerBlock = 16;
constexpr int kRowsPerGroup = 64;
constexpr int kKPerBlock = 32;
constexpr int kP1ChunkKB = 32;          // k-blocks per contraction-1 work item (1024 inputs)
constexpr int kP2ItemGroups = 16;       // row groups per contraction-2 work item (1024 outputs)
constexpr int kDecodeThreads = 128;     // 4 warps
constexpr int kMaxDecodeM = LB_DECODE_MAX_M;
constexpr int kMaxNT = (kMaxDecodeM + 3) / 4;   // n-tiles of 4 activation rows
constexpr int kIoBatch = 1024;          // layers per launch (pointer tables ride in kernel params)
constexpr int kP1StageKB = 8;           // k-blocks per ring stage, contraction 1 (2 KB)
constexpr int kP1Stages = 3;            // per-warp bulk-copy ring depth, contraction 1
constexpr int kP2Stages = 2;            // per-warp bulk-copy ring depth, contraction 2 (one row group per stage)

// Warp-streaming kernels for one or two activation rows.  Every warp owns an
// equal contiguous share of the bytes a contraction streams (fixed at plan
// build for one CTA per SM), so no work is handed out at run
// time and no warp waits for another.
// contraction-1 warps per CTA (independent of each other), one CTA per SM: 16
// for one row, 12 for two rows (their larger B fragments)
__host__ __device__ constexpr int pair_warps_per_cta(int MM) { return MM == 1 ? 16 : 12; }
constexpr int kPairStages = 2;          // ring stages per warp
constexpr int kPairStageKB = 16;        // k-blocks per ring stage (4 KB)
constexpr int kPairMaxKB2 = 64;         // largest contraction-2 depth (k-blocks) these kernels take (r = 1024, 2 paths)
// Shared memory of the contraction-2 kernel (per warp; per CTA with the zero
// buffer of one-row batches), and its warps per CTA: the most of
// {16, 12, 8, 6, 4} whose CTA fits in 227 KB.
__host__ __device__ constexpr int pair2_smem_per_warp(int MM, int kb2max)
{
    return kPairStages * kPairStageKB * 256 + 2 * (kb2max * 16 * MM * 8 + 144);
}
__host__ __device__ constexpr int pair2_cta_smem(int MM, int kb2max, int nw)
{
    return nw * pair2_smem_per_warp(MM, kb2max) + (MM == 1 ? kb2max * 128 : 0);
}
__host__ __device__ constexpr int pair2_warps_per_cta(int MM, int kb2max)
{
    return (pair2_cta_smem(MM, kb2max, 16) <= 227 * 1024)   ? 16
           : (pair2_cta_smem(MM, kb2max, 12) <= 227 * 1024) ? 12
           : (pair2_cta_smem(MM, kb2max, 8) <= 227 * 1024)  ? 8
           : (pair2_cta_smem(MM, kb2max, 6) <= 227 * 1024)  ? 6
                                                             : 4;
}
constexpr int kPairMeta2 = 144;         // bytes of zmeta copied with a contraction-2 B slot (p * 16 + m, m < 2)

// doubles in the accumulator block of a layer's scratch
__host__ __device__ inline size_t acc_doubles(int R1) { return (size_t)R1 * 16 + 32 + 16; }

static inline int round_up(int a, int b) { return (a + b - 1) / b * b; }
static inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Per-layer descriptor read by the kernels (device copy lives in a plan).
struct LayerDev {
    int N, K, r, npaths;
    int r16, r32;       // rank rounded up to 16 (contraction-1 rows) / 32 (contraction-2 k)
    int R1, RG1;        // contraction-1 rows (both paths, padded to 64) and row groups
    int K32, KB1;       // inputs rounded to 32, contraction-1 k-blocks
    int N64, RG2;       // outputs rounded to 64, contraction-2 row groups
    int KB2;            // contraction-2 k-blocks (npaths * r32 / 32)
    int nkc;            // contraction-1 work items (k chunks)
    const uint2 *vt;    // V tiles  [RG1][KB1][32]
    const uint2 *ut;    // U tiles  [RG2][KB2][32]
    const __half *g;    // [npaths][K32], zero padded
    const __half *h;    // [npaths][N64], zero padded
    const __half *l;    // [npaths][r16], zero padded
    // scratch (owned by the plan that holds this descriptor):
    //   acc:  [R1][16] double  sum over k of b * t (contraction-1 rows x activation rows; the
    //                           one/two-row kernels use the first R1 * M doubles as [R1][M])
    //         [2][16]  double  sum over k of t (per path x activation row)
    //         [2][16]  int     non-finite flags (per path x activation row)
    //   zfrag [kMaxNT][KB2][32] B fragments of contraction 2, zmeta [2][16] (exponent, digit sum)
    //   xfrag [KB1][32] B fragments of contraction 1 (one or two rows: 16 * M lanes per k-block)
    //   xmeta [nkc][2][2] exponent of each (k chunk, path, row)
    double *acc;
    uint2 *zfrag;
    int2 *zmeta;
    uint2 *xfrag;
    int *xmeta;
};

struct P1Item { int layer, kc; };
struct P2Item { int layer, rg0, rg1, pad; };

// Streaming units of the one/two-row kernels.  Contraction 1: row group rg of
// k chunk kc (nkb k-blocks at a); contraction 2: row group rg (KB2 k-blocks at a).
struct PairUnit1 { const uint2 *a; int layer, kc, rg, nkb; };
struct PairUnit2 { const uint2 *a; int layer, rg, kb2, pad; };

struct IoPtrs {
    const uint16_t *x[kIoBatch];
    float *y[kIoBatch];
};

// Sentinel exponent marking a non-finite activation block.
constexpr int kNanExp = -0x40000000;

}  // namespace lb

#include "lb_prefill_types.cuh"

// Host-side record of a layer (what lb_layer points to).
struct lb_layer {
    lb::LayerDev d;            // decode descriptor with pointers into `weights`
    lb::PfWeights pf;          // tensor-core (prefill) layouts, pointers into `weights`
    void *weights = nullptr;   // one allocation: all layouts + scales
    size_t weight_bytes = 0;
    struct lb_stack *self = nullptr;   // single-layer plan (owns scratch)
};

namespace lb {

struct PrefillState;

// A plan: descriptors + work items + scratch for a list of layers.
struct Plan {
    int n = 0;
    std::vector<const lb_layer *> layers;
    PrefillState *pf = nullptr;     // tensor-core path state, created on first use
    std::vector<LayerDev> host;     // descriptors (scratch pointers filled in)
    LayerDev *dev = nullptr;        // device copy of `host`
    P1Item *p1 = nullptr;           // device work items
    P2Item *p2 = nullptr;
    std::vector<int> p1_start, p2_start;   // per IO batch: first item index
    PairUnit1 *u1 = nullptr;        // one/two-row streaming units, all batches
    PairUnit2 *u2 = nullptr;
    // per row count MM (index MM - 1) and batch: pair_warps[MM - 1] + 1 unit boundaries (absolute)
    int *wr1[2] = {nullptr, nullptr}, *wr2[2] = {nullptr, nullptr};
    int pair_warps[2] = {0, 0};     // contraction-1 warps the streaming units are partitioned over, per MM
    int pair_warps2[2] = {0, 0};    // the same for contraction 2
    int kb2max = 0;                 // largest KB2 of the plan
    int rmax = 0;                   // largest rank of the plan
    int *err = nullptr;             // device error code (bounded waits that gave up)
    int n_p1 = 0, n_p2 = 0;
    void *scratch = nullptr;
    size_t scratch_bytes = 0;
};

cudaError_t plan_build(Plan &P, const lb_layer *const *layers, int n, cudaStream_t s);
void plan_free(Plan &P);

lb_status decode_forward(const Plan &P, const uint16_t *const *xs, float *const *ys, int M,
                         cudaStream_t s, int *launches);

lb_status decode_pair_launch(const LayerDev *dev_layers, int nlayers, const P1Item *p1, int n1, const PairUnit1 *u1,
                             const int *wr1, const PairUnit2 *u2, const int *wr2, int pair_warps, int pair_warps2,
                             const IoPtrs &io, int base, int M, int kb2max, int rmax, int *err, cudaStream_t s,
                             int *launches, bool mark);
lb_status decode_launch_one(const LayerDev *dev_desc, const LayerDev &host_desc, const struct Plan &P,
                            const uint16_t *x, float *y, int M, int *err, cudaStream_t s, int *launches);

lb_status status_from(cudaError_t e);
void set_launch_count(int n);
// Timing hook: record the registered event `i` (if any) on stream s.
void profile_mark(int i, cudaStream_t s);
// Whether timing events are registered (launches then stay strictly serialised).
bool profiling_active();

}  // namespace lb

struct lb_stack {
    lb::Plan plan;
    std::vector<const lb_layer *> layers;
};

// ---------------------------------------------------------------------------
// Small device helpers
// ---------------------------------------------------------------------------
namespace lb {

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b)
{
    return __uint_as_float(((uint32_t)b) << 16);
}

}  // namespace lb

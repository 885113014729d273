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
// A "k-block" is 64 rows x 32 k of one weight matrix, 256 bytes: lane L
// (g = L >> 2, t = L & 3) owns the uint2 {w0, w1}.  Bit i of byte b of word q
// is the sign bit (1 = -1) of
//     row = 16 * (i & 3) + g + 8 * (i >> 2),   k = 4 * t + b + 16 * q.
// The k-blocks of a 64-row group are stored in pairs: k-blocks 2j and 2j + 1
// take 512 contiguous bytes in which lane L owns the 16 bytes at 16 L (its
// uint2 of k-block 2j, then its uint2 of k-block 2j + 1), so one 16-byte load
// per lane fetches two k-blocks.  A row group's k-block count is rounded up to
// even (KB1e, KB2e); the padding k-block has no bit set and adds nothing.
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

// Streaming kernels for one or two activation rows (M <= 2): one CTA of
// kLdgWarps warps per SM, every warp streaming its own contiguous range of
// row-group units straight into registers (a ring of kLdgRing pairs of
// k-blocks per stream, two streams per warp: the two halves of each unit's
// k-range).  The ranges are built with the plan, cost-balanced over all warps.
constexpr int kLdgWarps = 16;           // warps per CTA (one CTA per SM)
constexpr int kLdgRing = 6;             // k-block pairs in flight per stream
constexpr int kPairMaxKB2 = 2 * LB_MAX_RANK / 32;   // contraction-2 depth (k-blocks) of the largest layer: every
                                                    // depth (deep units take the generic loop, B from L2)

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
    int KB1e, KB2e;     // KB1, KB2 rounded up to even (k-blocks are stored in pairs)
    const uint2 *vt;    // V tiles  [RG1][KB1e / 2 pairs][32 lanes][2]
    const uint2 *ut;    // U tiles  [RG2][KB2e / 2 pairs][32 lanes][2]
    const __half *g;    // [npaths][K32], zero padded
    const __half *h;    // [npaths][N64], zero padded
    const __half *l;    // [npaths][r16], zero padded
    const uint4 *hq;    // [RG2][2][8][4][2] binary16: h of path p, rows 16 rb + g + 8 hf of each row
                        //   group, ordered so that lane (g, p) of a warp reads its eight with one 16-byte load
    // scratch (owned by the plan that holds this descriptor):
    //   acc:  [R1][16] double  sum over k of b * t (contraction-1 rows x activation rows; the
    //                           one/two-row kernels use the first R1 * M doubles as [R1][M])
    //         [2][16]  double  sum over k of t (per path x activation row)
    //         [2][16]  int     non-finite flags (per path x activation row)
    //   zfrag [kMaxNT][KB2][32] B fragments of contraction 2 (one or two rows: [KB2e / 2][16 * M][2],
    //         pairs of k-blocks as in the tiles), zmeta [2][16] (exponent, digit sum)
    //   xfrag [KB1e / 2][16 * M][2] B fragments of contraction 1 (one or two rows, pairs of k-blocks)
    //   xmeta [nkc][2][2] exponent of each (k chunk, path, row)
    double *acc;
    uint2 *zfrag;
    int2 *zmeta;
    uint2 *xfrag;
    int *xmeta;
};

struct P1Item { int layer, kc; };
struct P2Item { int layer, rg0, rg1, pad; };

// Segments of the one/two-row streaming kernels (32 bytes each): n
// consecutive units of one layer in a warp's range, each P pairs of k-blocks.
// Contraction 1: row groups rg0 .. rg0 + n - 1 of one 1024-input chunk kc
// (v: the tiles of (rg0, kc); consecutive row groups are rstride uint4
// apart); contraction 2: row groups rg0 .. rg0 + n - 1 (u: the tiles of rg0;
// consecutive row groups are contiguous; hq: the row scales of rg0).
struct Seg1 { const uint4 *v; int layer, kc, rg0, n, P, rstride; };
struct Seg2 { const uint4 *u; const uint4 *hq; int layer, rg0, n, P; };

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
    // one/two-row streaming segments, all batches; per batch #SM * kLdgWarps + 1 segment boundaries
    // (absolute indices into the segment arrays), warp w of the launch taking [bnd[w], bnd[w + 1])
    Seg1 *sg1 = nullptr;
    Seg2 *sg2 = nullptr;
    int *bnd1 = nullptr, *bnd2 = nullptr;
    int *cls1 = nullptr, *cls2 = nullptr;   // per batch and warp: the step count of its units (0: mixed counts)
    int stream_grid = 0;            // CTAs of the streaming launches (the SM count)
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

lb_status decode_pair_launch(const LayerDev *dev_layers, int nlayers, const P1Item *p1, int n1, const Plan &P,
                             int batch, const IoPtrs &io, int base, int M, int kb2max, int rmax, int *err,
                             cudaStream_t s, int *launches, bool mark);
lb_status decode_launch_one(const LayerDev *dev_desc, const LayerDev &host_desc, const struct Plan &P,
                            const uint16_t *x, float *y, int M, int *err, cudaStream_t s, int *launches);

lb_status status_from(cudaError_t e);
// D = alpha A^T B on the tensor cores (fp16 in, fp32 out); arguments as lb_gemm_at_b in littlebit_backward.h
lb_status gemm_at_b(const void *A, int lda, const void *B, int ldb, float *D, int ldd, int Kc, int Mr, int Nc,
                    const float *alpha, int *err, cudaStream_t s);
// Several such products (at most two) in one launch, their tiles dealt as one list.
struct GemmDesc {
    const void *A;
    int lda;
    const void *B;
    int ldb;
    float *D;
    int ldd, Kc, Mr, Nc;
    const float *alpha;
};
lb_status gemm_at_b_batch(const GemmDesc *descs, int n, int *err, cudaStream_t s);
// Raise the dynamic shared-memory limit of kernel `fn` on the current device to at least `bytes` (never lowers
// it; per device and kernel, thread-safe).
cudaError_t ensure_dyn_smem(const void *fn, size_t bytes);
// The current device's SM count (cached per device).
cudaError_t sm_count_of_current(int *sms);
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

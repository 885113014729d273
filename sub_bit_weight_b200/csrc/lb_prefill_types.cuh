// Types of the tensor-core (prefill) path that the layer object embeds.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace lb {

// Sign bits of a generated operand, in "spread" order: for one row and one
// 64-wide k-block there are four 32-bit words; word q covers k = 16q .. 16q+15
// with element 16q + 2i at bit (15 - i) and element 16q + 2i + 1 at bit
// (31 - i), so that (word << i) & 0x80008000 puts the signs of elements
// (2i, 2i+1) on the sign bits of an f16x2 register.  Rows are grouped in
// tiles of 256, stored [row tile][k-block][256 rows][4 words] (4 KB blocks).
struct PfWeights {
    // latent contraction: z[m][j'] = sum_k fp16(x[m][k]) * (+-g_p[k]),  j' = p*r8 + j
    uint32_t *b1 = nullptr;   // [RT1][KB1][256][4]
    __half *g64 = nullptr;    // [npaths][K64]
    float *lcat = nullptr;    // [N1p] latent scale per column (0 on padding)
    // output contraction: y[m][n] = sum_j' zl[m][j'] * (+-h_p(j')[n])
    uint32_t *b2 = nullptr;   // [RT2][KB2][256][4]
    __half *h256 = nullptr;   // [npaths][N256]
    int r8 = 0, N1 = 0, N1p = 0, K64 = 0, KB1 = 0, RT1 = 0, K2 = 0, KB2 = 0, RT2 = 0, N256 = 0;
};

// Per-layer launch record of a tensor-core contraction.
struct PfLayer {
    const CUtensorMap *tmA;   // A operand (activations) tensor map
    const CUtensorMap *tmY;   // output GEMM: y tensor map (32 x 32 fp32 boxes)
    const uint32_t *bits;     // generated operand, spread layout
    const __half *base;       // g64 (latent) or h256 (output)
    const float *lcat;        // latent scales per output column (latent contraction only)
    void *out;                // zl (fp16) or y (fp32)
    int nk;                   // k-blocks
    int ncols;                // valid output columns (N1p or N)
    int ld_out;               // row stride of out, elements
    int ntn;                  // column tiles
    int r8;                   // columns per path
    int base_ld;              // row stride of base (K64 or N256)
    int npaths;
    int a_f16;                // latent contraction: A is already fp16 (no bf16 conversion)
    int ksplit;               // k-ranges per output tile (units of work); 1 = whole contraction per tile
    float *part;              // latent contraction with ksplit: fp32 [M][ld_part] that each unit adds its raw
                              // partial sums to (no l; zeroed by the caller); null = the fp16 zl epilogue
    int ld_part;
    const float *oscale;      // output contraction: null, or a device scalar every output is multiplied by
};

}  // namespace lb

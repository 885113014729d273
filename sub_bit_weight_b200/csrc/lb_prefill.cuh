// Prefill (large-M) path: declarations shared by the layer builder and the
// tensor-core kernels.
#pragma once

#include "lb_internal.cuh"

namespace lb {

// Tiles of the two tensor-core contractions.
constexpr int kPfBM = 128;          // activation rows per tile (UMMA M)
constexpr int kPfBN = 256;          // output columns per tile (UMMA N, at most)
constexpr int kPfBK = 64;           // contraction depth per pipeline stage (one 128-byte swizzle atom of fp16)
constexpr int kPfStages = 4;
constexpr int kPfThreads = 512;     // 16 warps: producer, MMA, 2 converters, 4 epilogue, 8 generator warps
constexpr int kPfExtraConv = 4;     // latent GEMM: converter warps 16.. beyond the 16
__host__ __device__ constexpr int pf_threads(int mode) { return kPfThreads + (mode == 0 ? 32 * kPfExtraConv : 0); }

cudaError_t prefill_build_weights(PfWeights &W, const LayerDev &d, const uint32_t *const *U,
                                  const uint32_t *const *V, const uint16_t *const *h,
                                  const uint16_t *const *g, const uint16_t *const *l, cudaStream_t s);
size_t prefill_weight_bytes(const LayerDev &d);

struct PrefillState;   // per plan (owned by Plan)
// parts: 1 = latent contraction only (writes the plan's zl), 2 = output contraction only (reads it), 3 = both,
// 0 = set up the plan's maps and buffers only.  a_f16: the activations xs are fp16 (bit patterns) rather than
// bf16.  marks: record the timing hook's events.  out_scale: null, or a device scalar the output contraction
// multiplies every y by.
lb_status prefill_forward(const Plan &P, const lb_layer *const *layers, const uint16_t *const *xs,
                          float *const *ys, int M, cudaStream_t s, int *launches, int parts = 3, bool a_f16 = false,
                          bool marks = true, const float *out_scale = nullptr);
// latent activations of layer i of the plan, fp16 [M][pf.K2] (null before the first prefill call)
__half *prefill_zl(const Plan &P, int i);
void prefill_free(PrefillState *st);
int *prefill_err_ptr(PrefillState *st);

// Latent contractions of several layers in one launch, each output tile split over k into units whose raw fp32
// partial sums are added (red.global.add) into the job's zeroed `part` [M][ld_part] (no l, no fp16 rounding).  The
// split is chosen so that the units spread evenly over the SMs.  `state` caches tensor maps and records between
// calls (create on first use, free with prefill_jobs_free).
struct PfLatentJob {
    const lb_layer *layer;
    const void *x;        // activations [M][K], bf16 or (a_f16) fp16, 16-byte aligned
    bool a_f16;
    float *part;          // fp32 [M][ld_part], ld_part >= the layer's padded latent width, 16-byte aligned
    int ld_part;
};
struct PfJobState;
lb_status prefill_latent_jobs(PfJobState **state, const PfLatentJob *jobs, int n, int M, cudaStream_t s,
                              int *launches);
void prefill_jobs_free(PfJobState *st);
int *prefill_jobs_err(PfJobState *st);

}  // namespace lb

/*
 * littlebit_backward.h -- C ABI of the LittleBit layer's backward pass for
 * quantisation-aware training (B200, sm_100a).
 *
 * Forward pass of one path (LittleBit paper notes page, "Multi-scale
 * compensation"): t = x (.) g, z = t V_s, zl = z (.) l, s = zl U_s^T,
 * y = sum_paths h (.) s, with U_s = sign(U), V_s = sign(V) of the latent
 * float factors.  QAT trains U, V, h, g, l; the sign's gradient is SmoothSign's
 * (same page, "Loss / training strategy": forward sign, backward tanh(100 u)),
 * d sign(u)/du := 100 (1 - tanh^2(100 u)).  Given dy = dL/dy, per path:
 *
 *   dh = sum_m dy (.) s            dU = (h (.) dy^T zl) (.) 100 (1 - tanh^2(100 U))
 *   dl = sum_m (dy (.) h) U_s (.) z
 *   dg = sum_m dt (.) x            dV = (g (.) x^T dz) (.) 100 (1 - tanh^2(100 V))
 *   dx = sum_paths dt (.) g,  with dz = ((dy (.) h) U_s) (.) l, dt = dz V_s^T.
 *
 * The two binary contractions of the backward are those of the forward pass
 * of the transposed layer (U <-> V, h <-> g) and run on the same tcgen05
 * kernels (z and (dy (.) h) U_s in one launch whose output tiles are split
 * over k, partial sums added in float32); the two dense products dy^T zl
 * (N x 2r) and x^T dz (K x 2r) are fp16 GEMMs with float32 accumulation on
 * the library's own tcgen05 kernel (lb_gemm_at_b below: both operands are
 * read MN-major, as stored), run with the factor gradients on a second stream
 * beside dx.
 *
 * Arithmetic: x enters as bfloat16 (converted to fp16 exactly in fp16's normal
 * range, as in the forward pass); dy is multiplied by one power of two chosen
 * on the device so that dy and (dy (.) h) U_s cannot overflow fp16, and
 * rounded to fp16; zl and dz are rounded to fp16 between the contractions (z
 * and (dy (.) h) U_s are kept in float32); every product accumulates in float32 and the power of two
 * is divided out exactly.  Scales are the layer's binary16 values (the ones
 * its forward pass uses).
 *
 * Conventions are those of littlebit.h: device pointers unless stated, arrays
 * of pointers are HOST arrays of device pointers, row-major dense matrices,
 * `stream` is a cudaStream_t passed as void*.
 */
#ifndef LITTLEBIT_BACKWARD_H
#define LITTLEBIT_BACKWARD_H

#include "littlebit.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lb_backward lb_backward;   /* opaque, library-owned */

/* Backward state of one layer.  Arguments as lb_layer_create (canonical
 * packed signs U [npaths][N rows], V [npaths][K rows]; binary16 h, g, l);
 * N and K must be multiples of 8 (tensor-map row strides in both
 * orientations).  Copies what it needs; the caller keeps its buffers.
 * Errors: LB_ERR_INVALID_ARG (null pointer, bad size), LB_ERR_UNSUPPORTED
 * (npaths, N or K not a multiple of 8), LB_ERR_OOM, LB_ERR_CUDA. */
LB_API lb_status lb_backward_create(lb_backward **out, int N, int K, int r, int npaths,
                                    const uint32_t *const *U, const uint32_t *const *V,
                                    const uint16_t *const *h, const uint16_t *const *g,
                                    const uint16_t *const *l, void *stream);
LB_API void lb_backward_destroy(lb_backward *B);

/* Gradients of one layer for a batch of M rows.
 *   x       bfloat16 [M][K], the forward input      dy   float32 [M][N]
 *   U_lat   [npaths] float32 [N][r]: latent factors whose signs are the packed U (for SmoothSign)
 *   V_lat   [npaths] float32 [K][r]
 *   dx      float32 [M][K]
 *   dh, dg, dl   [npaths] float32 [N], [K], [r]
 *   dU, dV       [npaths] float32 [N][r], [K][r]
 * All outputs are overwritten.  x, dy and dx must be 16-byte aligned.  The
 * work is enqueued on `stream` (no host synchronisation); scratch grows with M
 * and is owned by B, so calls on one B must not overlap.  Errors:
 * LB_ERR_INVALID_ARG, LB_ERR_OOM, LB_ERR_CUDA; a bounded wait that gave up in
 * a contraction kernel surfaces through lb_backward_status.
 *
 * With the timing hook of littlebit.h (lb_profile_events) holding 9 events,
 * events[i] is recorded at the i-th stage boundary: 0 | dy scaling | 1 |
 * z = (x (.) g) V_s and (dy (.) h) U_s, one launch | 2, 3 | dl, dz, zl | 4;
 * after 4 the work forks: dx | 5 on `stream`, and on a second stream of the
 * library (joined back into `stream` before the call returns) dy^T zl and
 * x^T dz, one launch | 6, 7 | dh, dg, dU, dV | 8 (events 2 and 3 mark the same
 * point, and so do 6 and 7). */
LB_API lb_status lb_layer_backward(lb_backward *B, const uint16_t *x, const float *dy, int M,
                                   const float *const *U_lat, const float *const *V_lat, float *dx,
                                   float *const *dh, float *const *dg, float *const *dl,
                                   float *const *dU, float *const *dV, void *stream);

/* Synchronises `stream`, returns and clears the device-side status of B's
 * contraction kernels: LB_OK or LB_ERR_TIMEOUT. */
LB_API lb_status lb_backward_status(lb_backward *B, void *stream);

/* D = alpha * A^T B: the dense products of the backward pass (dy^T zl and
 * x^T dz) as one tcgen05 tensor-core GEMM, fp16 operands, float32
 * accumulation and output.
 *   A      binary16 [Kc][lda], columns 0 .. Mr-1 used   (row-major: A[k][i] at A + k*lda + i)
 *   B      binary16 [Kc][ldb], columns 0 .. Nc-1 used
 *   D      float32  [Mr][ldd], columns 0 .. Nc-1 written, overwritten (padding columns untouched)
 *   alpha  device float32 scalar (read once per launch)
 *   err    device int: left alone on success; a bounded wait in the kernel that gave up (about 2 s)
 *          stores a nonzero code there (1 producer, 2 - 4 MMA / epilogue) and the launch ends early
 * Kc is the contracted extent (the batch rows of the backward pass), Kc >= 1.
 * A, B and D 16-byte aligned; lda and ldb multiples of 8, ldd of 4, Nc of
 * 32, lda >= Mr, ldb >= Nc, ldd >= Nc.  Rows of A and B past Kc, and columns
 * past Mr / Nc, are never read.  Enqueued on `stream`; nothing is allocated.
 * Errors: LB_ERR_INVALID_ARG (null, misaligned or inconsistent sizes),
 * LB_ERR_UNSUPPORTED (lda, ldb, ldd or Nc not a multiple as above, Kc = 0, no
 * tensor-map encoder in the driver), LB_ERR_CUDA.  Mr = 0 or Nc = 0 is a
 * no-op. */
LB_API lb_status lb_gemm_at_b(const uint16_t *A, int lda, const uint16_t *B, int ldb, float *D, int ldd,
                              int Kc, int Mr, int Nc, const float *alpha, int *err, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LITTLEBIT_BACKWARD_H */

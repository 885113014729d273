/*
 * littlebit_init.h -- C ABI of the LittleBit initialisation (B200, sm_100a):
 * Dual-SVID of a dense weight and residual compensation.
 *
 * LittleBit paper notes page, "Dual-SVID initialisation": a truncated SVD of
 * the dense weight W (N x K) to rank r gives U' (N x r) and V' (K x r); the
 * binary factors are their signs; a rank-1 SVD of each magnitude matrix |U'|,
 * |V'| gives the row scale h, the column scale g and the latent scale l, so
 * that diag(h) sign(U') diag(l) sign(V')^T diag(g) approximates U' V'^T.
 * Same page, "Residual compensation": the residual path is initialised by the
 * same procedure applied to W - W_hat_pri.
 *
 * Definitions this library fixes where the notes are silent:
 *   - U' = U_r diag(sqrt(s)), V' = V_r diag(sqrt(s)) (the r singular values
 *     split evenly between the factors);
 *   - the sign of each singular pair makes the largest-magnitude entry of the
 *     U' column positive (first index on ties); the effective weight does not
 *     depend on this choice;
 *   - sign(0) = +1, i.e. the packed bit is set exactly where U' < 0 (the
 *     canonical layout of lb_pack_signs in littlebit.h);
 *   - |U'| ~ s_u a_u b_u^T and |V'| ~ s_v a_v b_v^T with non-negative unit
 *     vectors (a pair is flipped when b sums below zero);
 *     h = a_u, g = a_v, l = s_u s_v (b_u (.) b_v); a zero magnitude matrix
 *     gives zero vectors.
 *
 * All arithmetic is IEEE binary64 on the device.  The truncated SVD is found
 * by randomised subspace iteration (orthonormalised by Cholesky QR after
 * every product with W^T W; a column whose part orthogonal to the others
 * falls below ~3e-7 of its norm is dropped, which only happens when
 * s_1 / s_L exceeds ~1e3 or W has rank below L) followed by a Rayleigh-Ritz
 * step with a Jacobi eigensolver, so
 * its accuracy depends on the number of iterations and on the spectrum: the
 * error of the rank-r subspace shrinks like (s_{L+1} / s_r)^(2 iters), with
 * L = min(min(N, K), max(64, 64 * ceil(2r / 64))) columns in the subspace.
 * When L = min(N, K) the subspace is the whole space and the result is
 * exact up to rounding for any `iters`.
 *
 * Conventions are those of littlebit.h: device pointers unless stated,
 * arrays of pointers are HOST arrays of device pointers, row-major dense
 * matrices, `stream` is a cudaStream_t passed as void*.
 */
#ifndef LITTLEBIT_INIT_H
#define LITTLEBIT_INIT_H

#include "littlebit.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of device workspace lb_dual_svid_init needs for this shape (0 for an
 * invalid shape: N, K or r below 1, or r above min(N, K)). */
LB_API size_t lb_dual_svid_workspace_bytes(int N, int K, int r);

/* Dual-SVID + residual initialisation of one LittleBit layer from a dense weight.
 *
 *   W          device, N x K float32, row-major, 4-byte aligned; not modified.
 *   N, K, r    1 <= r <= min(N, K) and r <= LB_MAX_RANK (littlebit.h).
 *   npaths     1 (primary only) or 2 (primary + residual).
 *   iters      subspace iterations (0 .. 1000); 24 suits spectra that decay
 *              like 1/i; ignored when the subspace is the whole space.
 *   U, V       host arrays of npaths device pointers: packed signs of U' (N
 *              rows) and V' (K rows), lb_packed_words(rows, r) uint32 words
 *              each, canonical layout (bit j % 32 of word [row, j / 32] set
 *              <=> the factor entry is < 0).  Ready for lb_layer_create.
 *   h, g, l    host arrays of npaths device pointers: float32 scales, N, K
 *              and r entries (the binary64 values rounded to nearest).
 *              lb_layer_create takes binary16: the caller rounds.
 *   sigma      NULL, or a device float32 array of npaths * r entries: the
 *              r leading singular values of each path's target matrix
 *              (W, then W - W_hat_pri), in decreasing order.
 *   workspace  device buffer of at least lb_dual_svid_workspace_bytes(N, K, r)
 *              bytes, 256-byte aligned, owned by the caller; its contents on
 *              return are unspecified.
 *
 * Returns LB_ERR_INVALID_ARG for a null pointer, a bad size or a small or
 * misaligned workspace (nothing is enqueued), LB_ERR_UNSUPPORTED for npaths
 * outside {1, 2}.  The work is enqueued on `stream`, and the call then waits
 * for the stream (it is not a hot-path call): LB_ERR_TIMEOUT if a bounded
 * device-side wait of the eigensolver gave up, LB_ERR_CUDA for a CUDA error
 * (including an earlier asynchronous one); the outputs are then undefined.
 *
 * With the timing hook of littlebit.h (lb_profile_events) holding at least 3
 * events, the primary path's first subspace iteration records events[0]
 * before the product Z = A Q, events[1] after it and events[2] after the
 * product A^T Z (A = W if K <= N, else W^T); nothing is recorded when the
 * subspace is the whole space. */
LB_API lb_status lb_dual_svid_init(const float *W, int N, int K, int r, int npaths, int iters,
                                   uint32_t *const *U, uint32_t *const *V,
                                   float *const *h, float *const *g, float *const *l, float *sigma,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * LittleBit-2 initialisation: latent rotation by Joint-ITQ.
 *
 * Wiki page on LittleBit and LittleBit-2, section 1 ("What happened"): the
 * second paper rotates the latent space and runs a joint iterative
 * quantisation (Joint-ITQ) before QAT so that the factors line up with the
 * binary hypercube; only the initialisation changes.  For an orthogonal
 * r x r matrix R, (U' R)(V' R)^T = U' V'^T, so the rotation is free; it only
 * changes the sign patterns.  Definitions this library fixes (the page gives
 * no formulas):
 *   - X = [U' / rho_u ; V' / rho_v] ((N + K) x r), each factor divided by the
 *     root mean square of its entries (a zero factor is left as is);
 *   - ITQ (Gong and Lazebnik's iterative quantisation): from R0, itq_iters
 *     alternations of B = sign(X R) (sign(0) = +1) and R = the orthogonal
 *     Procrustes solution for X^T B (its polar factor; computed here by
 *     Newton-Schulz iteration in binary64, run until an update moves no
 *     entry by more than 1e-9, at most 60 steps);
 *   - then U' <- U' R, V' <- V' R, canonical column signs as above, and the
 *     Dual-SVID steps (signs, rank-1 SVDs of the magnitudes) and the residual
 *     path as in lb_dual_svid_init, each path with its own rotation.
 * The loss ||sign(X R_t) - X R_t||_F^2 / ((N + K) r) never increases.
 * itq_iters = 0 with R0 = NULL is exactly lb_dual_svid_init.
 * ------------------------------------------------------------------------ */

/* Workspace bytes of lb_littlebit2_init (0 for an invalid shape). */
LB_API size_t lb_littlebit2_workspace_bytes(int N, int K, int r);

/* As lb_dual_svid_init, plus:
 *   itq_iters  ITQ alternations per path (0 .. 1000; ITQ's customary 50).
 *   R0         NULL (every path starts from the identity) or a host array of
 *              npaths pointers, each NULL (identity) or a device binary64
 *              r x r row-major orthogonal matrix, 8-byte aligned (ITQ's usual
 *              start is a random rotation).  With itq_iters = 0 it is applied
 *              as given, so it must then be orthogonal.
 *   itq_loss   NULL or device binary64 [npaths][itq_iters + 1]: the loss
 *              after t alternations, t = 0 .. itq_iters.
 *   R_out      NULL or a host array of npaths pointers, each NULL or device
 *              binary64 r x r row-major: the final rotation of the path.
 *   workspace  at least lb_littlebit2_workspace_bytes(N, K, r) bytes.
 * Errors and waiting as lb_dual_svid_init (LB_ERR_INVALID_ARG also for
 * itq_iters out of range or a misaligned R0, R_out or itq_loss). */
LB_API lb_status lb_littlebit2_init(const float *W, int N, int K, int r, int npaths, int iters, int itq_iters,
                                    const double *const *R0, uint32_t *const *U, uint32_t *const *V,
                                    float *const *h, float *const *g, float *const *l, float *sigma,
                                    double *itq_loss, double *const *R_out,
                                    void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LITTLEBIT_INIT_H */

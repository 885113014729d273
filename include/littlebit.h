/*
 * littlebit.h -- C ABI of the LittleBit compressed-linear library (B200, sm_100a).
 *
 * A LittleBit layer replaces a dense N x K weight W by two low-rank binary
 * paths (LittleBit: Ultra Low-Bit Quantization via Latent Factorization,
 * NeurIPS 2025; paper notes page, sections "Multi-scale compensation" and
 * "Residual compensation"):
 *
 *     W_hat = W_pri + W_res,   W_p = diag(h_p) . U_sign,p . diag(l_p) . V_sign,p^T . diag(g_p)
 *
 * with U_sign,p in {+-1}^(N x r), V_sign,p in {+-1}^(K x r), row scales
 * h_p (N), column scales g_p (K) and latent scales l_p (r).  The forward pass
 * y = x . W_hat^T is evaluated factor by factor, as the same section of the
 * notes describes (sequential element-wise products and binary matmuls, the
 * effective weight is never stored):
 *
 *     t = x (.) g_p  ->  z = t . V_sign,p  ->  z (.)= l_p  ->  s = z . U_sign,p^T  ->  y += h_p (.) s
 *
 * Conventions (every entry point):
 *   - All data pointers are DEVICE pointers unless stated otherwise; arrays of
 *     pointers ("const T* const* a") are HOST arrays holding device pointers.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  All device work is enqueued on it; no entry point synchronises
 *     the host with the device unless it says so.
 *   - Scalars h, g, l are IEEE binary16 and x is bfloat16; both are passed as
 *     their 16-bit patterns (uint16_t).  y is float32.  Matrices are
 *     row-major and densely packed.
 *   - No exception crosses the ABI.  Every entry point validates its
 *     arguments and returns an lb_status; on any error nothing is enqueued.
 *     LB_ERR_CUDA reports an error returned by the CUDA runtime on this call
 *     (including an asynchronous error of earlier work on the device).
 *   - The caller keeps ownership of every buffer it passes; the library owns
 *     the objects it creates (lb_layer, lb_stack) and their device memory.
 *   - Use one process per GPU, with one host thread making the calls.  The
 *     library raises each kernel's shared-memory limit once per process and
 *     remembers that it did, in an unlocked cache, while CUDA keeps the limit
 *     per device.  A second GPU in the same process, or two threads whose
 *     first calls overlap, can therefore see a launch fail with LB_ERR_CUDA.
 *     Nothing faults.
 */
#ifndef LITTLEBIT_H
#define LITTLEBIT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LB_API __attribute__((visibility("default")))
#else
#define LB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lb_status {
    LB_OK = 0,
    LB_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, misaligned buffer      */
    LB_ERR_UNSUPPORTED = 2,  /* a valid request this library does not implement         */
    LB_ERR_OOM = 3,          /* a device allocation of the library failed               */
    LB_ERR_CUDA = 4,         /* the CUDA runtime returned an error                      */
    LB_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up (state was reset)    */
} lb_status;

/* Opaque, library-owned objects. */
typedef struct lb_layer lb_layer;
typedef struct lb_stack lb_stack;

/* Largest batch handled by the fused small-batch (decode) kernels; larger M
 * runs on the tensor-core (prefill) kernels. */
#define LB_DECODE_MAX_M 16
/* Most layers one lb_stack_forward call can cover. */
#define LB_STACK_MAX_LAYERS 4096

/* Human-readable name of a status code (static storage, never NULL). */
LB_API const char *lb_status_string(lb_status s);

/* Number of uint32 words of the canonical packed layout of a rows x r factor:
 * rows * ceil(r / 32).  Returns 0 for rows < 0 or r <= 0. */
LB_API size_t lb_packed_words(int64_t rows, int r);

/*
 * Sign binarisation, U_sign = sign(U) (notes page, "Overall framework",
 * step 2), into the canonical packed layout.
 *
 *   F       device, float32 [rows x r], row-major, 4-byte aligned.
 *   packed  device, uint32 [rows x ceil(r/32)], caller-allocated, 4-byte aligned.
 *           Word packed[i*ceil(r/32) + j/32], bit (j % 32), is 1 iff F[i][j] < 0,
 *           so sign(0) = +1, -0.0 -> +1 and NaN -> +1.  Padding bits are 0.
 *           Every word is written.
 * rows = 0 is a valid empty call.  Errors: F or packed NULL (with rows > 0),
 * rows < 0 or r <= 0 -> LB_ERR_INVALID_ARG.
 */
LB_API lb_status lb_pack_signs(const float *F, int64_t rows, int r, uint32_t *packed, void *stream);

/*
 * Build a layer from canonical packed signs and binary16 scales.
 *
 *   out     receives the new layer (host pointer to a handle).
 *   N, K    output / input features (N, K >= 1); r >= 1 latent rank per path.
 *   npaths  1 (primary only) or 2 (primary + residual); path 0 is primary.
 *   U[p]    device, canonical packed U_sign,p, N x ceil(r/32) words.
 *   V[p]    device, canonical packed V_sign,p, K x ceil(r/32) words.
 *   h[p]    device, binary16 [N];  g[p] device, binary16 [K];  l[p] device, binary16 [r].
 *   stream  the copies and re-tiling run on it; the inputs must stay valid
 *           until that work completes (the call returns before it does).
 * The layer copies everything it needs into its own device memory, re-tiled
 * for its kernels; the caller keeps its inputs.  Scales may be any finite
 * binary16 value, including zero and negative values.
 * Errors: LB_ERR_INVALID_ARG (NULL, sizes < 1, r > LB_MAX_RANK),
 * LB_ERR_UNSUPPORTED (npaths not 1 or 2), LB_ERR_OOM, LB_ERR_CUDA.
 */
#define LB_MAX_RANK 2048
LB_API lb_status lb_layer_create(lb_layer **out, int N, int K, int r, int npaths,
                          const uint32_t *const *U, const uint32_t *const *V,
                          const uint16_t *const *h, const uint16_t *const *g,
                          const uint16_t *const *l, void *stream);

/* Free a layer (NULL is a no-op).  Synchronises with the device before freeing. */
LB_API void lb_layer_destroy(lb_layer *L);

/* Shape of a layer; any output pointer may be NULL.  Returns LB_ERR_INVALID_ARG for L == NULL. */
LB_API lb_status lb_layer_shape(const lb_layer *L, int *N, int *K, int *r, int *npaths);

/* Bits per weight by the pages' accounting,
 *   sum_paths [r(N+K) * 1 + 16 (N+K+r)] / (N K),
 * padding excluded (wiki page on LittleBit and LittleBit-2, "How to judge an
 * ultra-low-bit scheme", point 1).  0 for NULL. */
LB_API double lb_layer_bpw(const lb_layer *L);

/* Device bytes the layer owns (weights in all layouts, scales and scratch). */
LB_API size_t lb_layer_device_bytes(const lb_layer *L);

/*
 * Forward pass of one layer:  y[M x N] = x[M x K] . W_hat^T.
 *
 *   x  device, bfloat16 [M x K] row-major, 16-byte aligned.
 *   y  device, float32  [M x N] row-major, 16-byte aligned; fully overwritten.
 * M = 0 is a valid empty call.  M <= LB_DECODE_MAX_M runs the fused decode
 * kernels, larger M the tensor-core kernels.  The layer's scratch memory is
 * reused by every call: calls on one layer must be ordered on the device (one
 * stream, or explicit events); concurrent calls on one layer race.
 * Non-finite values in a row of x give NaN in that row of y.
 * Errors: LB_ERR_INVALID_ARG (NULL, M < 0, misalignment), LB_ERR_OOM
 * (scratch growth for a larger M than before), LB_ERR_CUDA.  Every r <=
 * LB_MAX_RANK runs with one or two paths at every M: one or two rows run on
 * streaming kernels whose depth has no shared-memory bound; 3..16 rows run on
 * kernels that stage a row group's contraction-2 tiles in shared memory,
 * (8 + ceil(min(M,16)/4)) * KB2 * 256 bytes <= 227 KB with KB2 = npaths *
 * ceil(r/32) (two paths: r <= 1184 at every M, r <= 1600 at M <= 4), and a
 * deeper layer (or stack) takes the streaming kernels once per pair of rows
 * instead.  (Decode also serves larger M when K is not a multiple of 8 or N
 * not a multiple of 4, as 16-row blocks.)
 */
LB_API lb_status lb_linear_forward(const uint16_t *x, int M, const lb_layer *L, float *y, void *stream);

/*
 * A stack: many independent layers run by one set of kernel launches (the
 * per-layer work is too small to pay one launch per layer).  The layers stay
 * owned by the caller and must outlive the stack.  Layers may repeat.
 * Errors: LB_ERR_INVALID_ARG (NULL, n < 1, n > LB_STACK_MAX_LAYERS), LB_ERR_OOM, LB_ERR_CUDA.
 */
LB_API lb_status lb_stack_create(lb_stack **out, const lb_layer *const *layers, int n, void *stream);
LB_API void lb_stack_destroy(lb_stack *S);

/*
 * Forward pass of every layer of a stack, layer i reading xs[i] and writing
 * ys[i] (device pointers; xs[i] is bfloat16 [M x K_i], ys[i] float32
 * [M x N_i], 16-byte aligned).  The layers are independent: no output feeds
 * another layer.  Same M for all layers; M = 0 is a valid empty call.  The
 * stack's scratch is reused by every call (order calls on one stack).
 * Errors: as lb_linear_forward.
 */
LB_API lb_status lb_stack_forward(lb_stack *S, const uint16_t *const *xs, float *const *ys, int M, void *stream);

/*
 * Forward pass of one layer, M <= LB_DECODE_MAX_M, that allocates no memory.
 *
 * The paper has no counterpart to this call; it exists for callers that must
 * not allocate device memory while they run: a serving loop whose device
 * memory is planned once at start-up and must not touch the CUDA allocator
 * again (cudaMalloc/cudaFree may synchronise the device, stall every stream
 * and fragment a memory plan), or an embedding runtime that owns all device
 * memory itself.  The layer itself still comes from lb_layer_create (which
 * allocates); this call does not.
 *
 * Same arguments, layouts and result as lb_linear_forward for M <= 16.  The
 * scratch of the decode kernels (float64 accumulators, latent fragments,
 * error code) lives in one fixed array of
 * LB_NOALLOC_SCRATCH_BYTES bytes of static device memory inside this library,
 * which every GPU that loads the library holds until the process exits.  The
 * call issues no cudaMalloc, cudaFree or allocating library routine: it
 * launches one small kernel that writes the layer descriptor into that array
 * and clears the accumulators, then the decode kernels.
 * The first call on each device looks the array's device address up once
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture begins.
 * Every call writes the descriptor and clears the accumulators at its start;
 * the other parts of the array (fragments, exponents) are overwritten before
 * they are read, and otherwise keep the last call's contents.  Calls share the
 * one array, so calls that overlap on the GPU (different streams, or other
 * host threads) race: order them on one stream.
 * A bounded device-side wait that gives up during this call records its code
 * in the layer's own error slot (device memory allocated with the layer, the
 * slot lb_linear_forward reports to as well); lb_layer_status reads and
 * clears it.
 * Errors: LB_ERR_INVALID_ARG (NULL, M < 0, misalignment), LB_ERR_UNSUPPORTED
 * (M > LB_DECODE_MAX_M, the layer needs more than LB_NOALLOC_SCRATCH_BYTES
 * of scratch, or its contraction-2 depth exceeds the decode kernels' shared
 * memory as for lb_linear_forward), LB_ERR_CUDA.  M = 0 is a valid empty call.
 */
#define LB_NOALLOC_SCRATCH_BYTES (1u << 20)
LB_API lb_status lb_linear_forward_noalloc(const uint16_t *x, int M, const lb_layer *L, float *y, void *stream);

/*
 * Device-side failure reporting.  Every wait inside the library's kernels is
 * bounded (about two seconds of clock ticks); a wait that gives up records an
 * error code in the plan's device memory and its kernel returns instead of
 * hanging.  These calls synchronise `stream`, read that code, clear it, and
 * return LB_ERR_TIMEOUT if a wait gave up since the last check (LB_OK if not).
 * A timed-out call leaves its outputs unspecified.
 * Errors: LB_ERR_INVALID_ARG (NULL), LB_ERR_CUDA.
 */
LB_API lb_status lb_stack_status(lb_stack *S, void *stream);
LB_API lb_status lb_layer_status(const lb_layer *L, void *stream);

/*
 * Self-test of the bounded-wait mechanism: launches one thread that waits, with
 * the same helper the kernels use, on an mbarrier that nothing completes,
 * giving up after `cycles` clock ticks.  Synchronises `stream`; returns
 * LB_ERR_TIMEOUT when the wait gave up and reported it (the expected result),
 * LB_OK if it did not.  No GPU fault or hang is involved.
 */
LB_API lb_status lb_selftest_wait_timeout(long long cycles, void *stream);

/*
 * The same self-test aimed at a layer's error slot, the slot the layer's
 * decode kernels report to (lb_linear_forward and lb_linear_forward_noalloc):
 * launches the waiting thread on `stream` and returns without synchronising;
 * a following lb_layer_status(L, stream) returns LB_ERR_TIMEOUT once (and
 * clears the slot).  Errors: L NULL or cycles < 0 -> LB_ERR_INVALID_ARG,
 * LB_ERR_CUDA.
 */
LB_API lb_status lb_layer_selftest_wait_timeout(const lb_layer *L, long long cycles, void *stream);

/* Timing hook.  Registers n CUDA events (cudaEvent_t passed as void*) for the
 * calling thread: the following forward calls record events[0] on their
 * stream before their first kernel launch and events[i] right after their
 * i-th launch (1 <= i < n).  n = 0 (or events == NULL) clears the hook.  The
 * events stay owned by the caller.  Errors: n < 0 -> LB_ERR_INVALID_ARG. */
#define LB_MAX_PROFILE_EVENTS 64
LB_API lb_status lb_profile_events(void *const *events, int n);

/* Number of kernel launches the last forward call (layer or stack) enqueued
 * on this thread; used to count launches in timed regions. */
LB_API int lb_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LITTLEBIT_H */

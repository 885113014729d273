// Sign binarisation into the canonical packed layout, and the ABI's small
// utility entry points.
//
// U_sign = sign(U) (LittleBit notes page, "Overall framework", step 2) with
// sign(0) = +1: a bit is set iff the float compares below zero, so -0.0 and
// NaN give +1.  Word i*ceil(r/32) + j/32, bit j%32 holds element (i, j).

#include "lb_decode_common.cuh"
#include "lb_prefill.cuh"

namespace lb {

static thread_local int g_last_launches = 0;
void set_launch_count(int n) { g_last_launches = n; }

static thread_local cudaEvent_t g_prof_events[LB_MAX_PROFILE_EVENTS];
static thread_local int g_prof_n = 0;

void profile_mark(int i, cudaStream_t s)
{
    if (i >= 0 && i < g_prof_n && g_prof_events[i]) cudaEventRecord(g_prof_events[i], s);
}

bool profiling_active() { return g_prof_n > 0; }

lb_status status_from(cudaError_t e)
{
    if (e == cudaSuccess) return LB_OK;
    if (e == cudaErrorMemoryAllocation) return LB_ERR_OOM;
    return LB_ERR_CUDA;
}

// One warp per output word: lane l tests element 32*w + l of its row (a
// coalesced 128-byte read) and the ballot is the word.
__global__ void __launch_bounds__(256) pack_signs_kernel(const float *__restrict__ F, int64_t rows,
                                                         int r, uint32_t *__restrict__ packed)
{
    const int lane = threadIdx.x & 31;
    const int64_t wpr = (r + 31) / 32;
    const int64_t nwords = rows * wpr;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t w = warp0; w < nwords; w += nwarps) {
        const int64_t i = w / wpr;
        const int j = (int)(w - i * wpr) * 32 + lane;
        bool neg = false;
        if (j < r) neg = __ldcs(F + i * r + j) < 0.0f;
        const uint32_t word = __ballot_sync(0xffffffffu, neg);
        if (lane == 0) packed[w] = word;
    }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// completes, gives up after `cycles` clock ticks and records the error code,
// exactly as the decode kernels do when a bulk copy never lands.
__global__ void wait_selftest_kernel(int *err, long long cycles)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        bar_init(&bar);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        ring_wait(&bar, 0, err, cycles);   // phase 0 never completes
    }
}

static int *g_selftest_err = nullptr;

}  // namespace lb

extern "C" {

const char *lb_status_string(lb_status s)
{
    switch (s) {
    case LB_OK: return "LB_OK";
    case LB_ERR_INVALID_ARG: return "LB_ERR_INVALID_ARG: invalid argument";
    case LB_ERR_UNSUPPORTED: return "LB_ERR_UNSUPPORTED: not supported";
    case LB_ERR_OOM: return "LB_ERR_OOM: device allocation failed";
    case LB_ERR_CUDA: return "LB_ERR_CUDA: CUDA runtime error";
    case LB_ERR_TIMEOUT: return "LB_ERR_TIMEOUT: device-side wait timed out";
    }
    return "unknown lb_status";
}

size_t lb_packed_words(int64_t rows, int r)
{
    if (rows < 0 || r <= 0) return 0;
    return (size_t)rows * (size_t)((r + 31) / 32);
}

int lb_last_launch_count(void) { return lb::g_last_launches; }

static lb_status read_and_clear(int *dev_err, cudaStream_t s)
{
    int h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, dev_err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && h) e = cudaMemsetAsync(dev_err, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return lb::status_from(e);
    return h ? LB_ERR_TIMEOUT : LB_OK;
}

lb_status lb_stack_status(lb_stack *S, void *stream)
{
    if (!S) return LB_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    lb_status st = read_and_clear(S->plan.err, s);
    if (st == LB_OK && S->plan.pf) st = read_and_clear(lb::prefill_err_ptr(S->plan.pf), s);
    return st;
}

lb_status lb_layer_status(const lb_layer *L, void *stream)
{
    if (!L) return LB_ERR_INVALID_ARG;
    return lb_stack_status(L->self, stream);
}

lb_status lb_selftest_wait_timeout(long long cycles, void *stream)
{
    if (cycles < 0) return LB_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (!lb::g_selftest_err) {
        if ((e = cudaMalloc(&lb::g_selftest_err, sizeof(int))) != cudaSuccess) return lb::status_from(e);
    }
    if ((e = cudaMemsetAsync(lb::g_selftest_err, 0, sizeof(int), s)) != cudaSuccess) return lb::status_from(e);
    lb::wait_selftest_kernel<<<1, 32, 0, s>>>(lb::g_selftest_err, cycles);
    if ((e = cudaGetLastError()) != cudaSuccess) return lb::status_from(e);
    return read_and_clear(lb::g_selftest_err, s);
}

lb_status lb_layer_selftest_wait_timeout(const lb_layer *L, long long cycles, void *stream)
{
    if (!L || cycles < 0) return LB_ERR_INVALID_ARG;
    lb::wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(L->self->plan.err, cycles);
    return lb::status_from(cudaGetLastError());
}

lb_status lb_profile_events(void *const *events, int n)
{
    if (n < 0 || n > LB_MAX_PROFILE_EVENTS) return LB_ERR_INVALID_ARG;
    if (!events) n = 0;
    for (int i = 0; i < n; ++i) lb::g_prof_events[i] = (cudaEvent_t)events[i];
    lb::g_prof_n = n;
    return LB_OK;
}

lb_status lb_pack_signs(const float *F, int64_t rows, int r, uint32_t *packed, void *stream)
{
    lb::set_launch_count(0);
    if (rows < 0 || r <= 0) return LB_ERR_INVALID_ARG;
    if (rows == 0) return LB_OK;
    if (!F || !packed) return LB_ERR_INVALID_ARG;
    if (((uintptr_t)F & 3) || ((uintptr_t)packed & 3)) return LB_ERR_INVALID_ARG;
    const int64_t nwords = (int64_t)lb_packed_words(rows, r);
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return lb::status_from(e);
    const int warps_per_block = 256 / 32;
    int64_t blocks = (nwords + warps_per_block - 1) / warps_per_block;
    const int64_t cap = (int64_t)sms * 16;
    if (blocks > cap) blocks = cap;
    lb::pack_signs_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(F, rows, r, packed);
    e = cudaGetLastError();
    if (e == cudaSuccess) lb::set_launch_count(1);
    return lb::status_from(e);
}

}  // extern "C"

// Device helpers shared by the decode (small-batch) kernels.
#pragma once

#include <cfloat>

#include "lb_internal.cuh"

namespace lb {

// ---------------------------------------------------------------------------
// Fixed point
// ---------------------------------------------------------------------------
static __device__ __forceinline__ int exponent_for(float amax, bool nonfinite)
{
    // Largest E with amax * 2^E <= 32639, so that q = rint(t * 2^E) splits into
    // two balanced digits in [-128, 127].
    if (nonfinite) return kNanExp;
    if (!(amax > 0.0f)) return 0;
    int e;
    frexpf(amax, &e);                    // amax = f * 2^e, f in [0.5, 1)
    int E = 15 - e;                      // amax * 2^E in [2^14, 2^15)
    if (ldexpf(amax, E) > 32639.0f) E -= 1;
    return min(E, 126);                  // 2^E and 2^-E stay normal floats (inputs below 2^-111 lose bits)
}

// 2^E as a float (exact: |E| <= 126); quantize(t) = rint(t * 2^E)
static __device__ __forceinline__ float pow2f(int E) { return __int_as_float((127 + E) << 23); }
static __device__ __forceinline__ double pow2d(int E) { return __longlong_as_double((long long)(1023 + E) << 52); }

static __device__ __forceinline__ int quantize_s(float t, float scale) { return __float2int_rn(t * scale); }

// low digit in [-128, 127] and high digit, q = 256 * hi + lo
static __device__ __forceinline__ void digits(int q, int &lo, int &hi)
{
    lo = ((q + 128) & 255) - 128;
    hi = (q - lo) >> 8;
}

// Where the two digit words of activation row m and 4 consecutive k starting
// at kk (within a 32-wide k-block) live among the lanes' m16n8k32 B
// fragments: column g = 2 * (m % 4) + digit, lane = 4 * g + t, word kk / 16,
// with t = (kk % 16) / 4.
static __device__ __forceinline__ void frag_slot(int m, int kk, int &lane_lo, int &lane_hi, int &word)
{
    const int mm = m & 3;
    const int t = (kk & 15) >> 2;
    word = kk >> 4;
    lane_lo = (2 * mm) * 4 + t;
    lane_hi = (2 * mm + 1) * 4 + t;
}

static __device__ __forceinline__ void set_word(uint2 &u, int word, uint32_t v)
{
    if (word) u.y = v; else u.x = v;
}

static __device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

static __device__ __forceinline__ int warp_sum(int v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

static __device__ __forceinline__ int warp_or(int v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Explicit shared-memory loads on 32-bit shared-window addresses (a generic
// pointer into dynamic shared memory may compile to a generic load).
static __device__ __forceinline__ uint2 lds64(uint32_t addr)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

static __device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
    return v;
}

// non-negative floats order like their bit patterns
static __device__ __forceinline__ void smem_max(float *a, float v) { atomicMax((int *)a, __float_as_int(v)); }

// ---------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel of the stream still runs;
// dep_wait() returns once that kernel has completed and its writes are visible
// (immediately when the launch had no such dependency).  dep_release() lets the
// next kernel of the stream start launching.
// ---------------------------------------------------------------------------
static __device__ __forceinline__ void dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
static __device__ __forceinline__ void dep_release() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// mbarrier + bulk copy (one ring of buffers per warp)
// ---------------------------------------------------------------------------
static __device__ __forceinline__ uint32_t sm_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

static __device__ __forceinline__ void bar_init(uint64_t *b)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(sm_addr(b)));
}

static __device__ __forceinline__ void ring_fill(void *dst, const void *src, unsigned bytes, uint64_t *bar)
{
    asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(sm_addr(bar)),
                 "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     sm_addr(dst)),
                 "l"(src), "r"(bytes), "r"(sm_addr(bar))
                 : "memory");
}

// Bulk copy completing on `bar` (the caller has announced the bytes with expect_tx).
static __device__ __forceinline__ void bulk_copy(void *dst, const void *src, unsigned bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     sm_addr(dst)),
                 "l"(src), "r"(bytes), "r"(sm_addr(bar))
                 : "memory");
}

// L2 policy for data read exactly once per call (the weight streams): evict first,
// so that what is re-read (fragments, scales) stays in L2.
static __device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
    return pol;
}

static __device__ __forceinline__ void bulk_copy_hint(void *dst, const void *src, unsigned bytes, uint64_t *bar,
                                                      uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n" ::"r"(
            sm_addr(dst)),
        "l"(src), "r"(bytes), "r"(sm_addr(bar)), "l"(pol)
        : "memory");
}

// One thread's bookkeeping without a divergent branch: `lead` (non-zero in one
// lane) announces `tx` bytes on `bar` and starts a bulk copy of `bytes` into it
// (evict-first L2 policy), all as predicated instructions.
static __device__ __forceinline__ void lead_fill_hint(uint32_t lead, uint64_t *bar, unsigned tx, void *dst,
                                                      const void *src, unsigned bytes, uint64_t pol)
{
    asm volatile("{\n.reg .pred p;\n.reg .b64 st;\nsetp.ne.u32 p, %0, 0;\n"
                 "@p mbarrier.arrive.expect_tx.shared::cta.b64 st, [%1], %2;\n"
                 "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%3], [%4], %5, [%1], %6;\n"
                 "}\n" ::"r"(lead),
                 "r"(sm_addr(bar)), "r"(tx), "r"(sm_addr(dst)), "l"(src), "r"(bytes), "l"(pol)
                 : "memory");
}

// A further bulk copy on `bar` by the leading lane (bytes already announced).
static __device__ __forceinline__ void lead_copy(uint32_t lead, uint64_t *bar, void *dst, const void *src,
                                                 unsigned bytes)
{
    asm volatile("{\n.reg .pred p;\nsetp.ne.u32 p, %0, 0;\n"
                 "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%1], [%2], %3, [%4];\n"
                 "}\n" ::"r"(lead),
                 "r"(sm_addr(dst)), "l"(src), "r"(bytes), "r"(sm_addr(bar))
                 : "memory");
}

// Generic-proxy reads of a ring stage are ordered before the async-proxy copy that refills it.
static __device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

static __device__ __forceinline__ void expect_tx(uint64_t *bar, unsigned bytes)
{
    asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(sm_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

static __device__ __forceinline__ bool bar_try(uint64_t *b, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok)
                 : "r"(sm_addr(b)), "r"(parity)
                 : "memory");
    return ok != 0;
}

constexpr long long kDecWaitCycles = 4000000000LL;   // ~2 s

// Bounded wait for a ring buffer; false (and an error code) on timeout.
static __device__ __forceinline__ bool ring_wait(uint64_t *b, uint32_t parity, int *err,
                                                 long long limit = kDecWaitCycles)
{
    if (bar_try(b, parity)) return true;
    const long long t0 = clock64();
    while (!bar_try(b, parity)) {
        if (clock64() - t0 > limit) {
            atomicCAS(err, 0, 16);
            return false;
        }
    }
    return true;
}

}  // namespace lb

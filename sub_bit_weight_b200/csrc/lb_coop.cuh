// Grid-wide barrier for cooperative launches of the initialisation kernels.
#pragma once

#include <cuda_runtime.h>

namespace lb {

constexpr long long kBarrierCycles = 2000000000LL;   // ~1 s at the boost clock

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// All CTAs of the grid are co-resident (cooperative launch).  bar[0] counts
// arrivals, bar[1] is the generation (both zero before the launch; `gen` is
// thread 0's copy, starting at 0).  The wait is bounded: on timeout, or when
// another CTA already gave up, `err` is set and every CTA returns false.
__device__ __forceinline__ bool grid_barrier(unsigned *bar, unsigned &gen, int *err)
{
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        int good = 1;
        const unsigned want = gen + 1;
        __threadfence();
        if (atomicAdd(&bar[0], 1u) == gridDim.x - 1) {
            atomicExch(&bar[0], 0u);
            __threadfence();
            atomicExch(&bar[1], want);
        } else {
            const long long t0 = clock64();
            while (ld_acquire_u32(&bar[1]) != want) {
                if (*(volatile int *)err != 0 || clock64() - t0 > kBarrierCycles) {
                    atomicCAS(err, 0, 32);
                    good = 0;
                    break;
                }
                __nanosleep(32);
            }
        }
        gen = want;
        __threadfence();
        ok = good;
    }
    __syncthreads();
    return ok != 0;
}

}  // namespace lb

// Bounded waits shared by the kernels that wait at all: a grid-wide barrier
// for cooperative launches and a wait on a shared-memory mbarrier phase.
// Every wait gives up after kWaitLimitNs of %globaltimer and reports it, so a
// missing arrival ends in an error status, never in a hung GPU.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ unsigned long long gtimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p)
{
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(unsigned int *p, unsigned int v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// State of a grid barrier in global memory, zeroed before the launch.
struct GridBarrier {
    unsigned int count;    // blocks arrived at the current barrier
    unsigned int gen;      // barriers completed
    unsigned int abort;    // set by a block that gave up: releases every waiter
};

// Grid-wide barrier of a cooperative launch.  Returns false in every thread
// of the block when its wait ran out (after recording MOE_DERR_TIMEOUT and
// raising abort) or another block had aborted.
__device__ __forceinline__ bool grid_barrier(GridBarrier *b, int32_t *err)
{
    __shared__ int ok_s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        const unsigned int gen = ld_acquire_u32(&b->gen);
        __threadfence();
        if (atomicAdd(&b->count, 1u) + 1 == gridDim.x) {
            atomicExch(&b->count, 0u);
            __threadfence();
            st_release_u32(&b->gen, gen + 1);
        } else {
            const unsigned long long t0 = gtimer_ns();
            while (ld_acquire_u32(&b->gen) == gen) {
                if (ld_acquire_u32(&b->abort)) { ok = 0; break; }
                if (gtimer_ns() - t0 > kWaitLimitNs) {
                    record_error(err, MOE_DERR_TIMEOUT);
                    atomicExch(&b->abort, 1u);
                    ok = 0;
                    break;
                }
                __nanosleep(64);
            }
        }
        __threadfence();
        ok_s = ok;
    }
    __syncthreads();
    return ok_s != 0;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// true once the mbarrier phase with the given parity has completed; false
// when that took longer than kWaitLimitNs.  Each try_wait may suspend the
// thread in hardware until the phase completes, for at most kSuspendHintNs,
// so a waiting warp takes no issue slots from the warps doing the work.
constexpr uint32_t kSuspendHintNs = 1000000;   // 1 ms

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_addr(bar);
    const unsigned long long t0 = gtimer_ns();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity), "r"(kSuspendHintNs)
            : "memory");
        if (done) return true;
        if (gtimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

}  // namespace moe

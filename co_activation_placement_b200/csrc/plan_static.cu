// Dispatch plan for callers that cannot allocate device memory.
//
// moe_plan_dispatch needs a few hundred kilobytes of scratch (per-chunk row
// counts, their prefix sums, the source-rank permutation).  Some callers
// cannot hand it any: code that runs inside another framework's allocator or
// memory-pool hook (where calling cudaMalloc would re-enter the allocator),
// processes that reserve their whole device-memory budget at start-up and
// forbid later allocations, and latency-critical loops where cudaMalloc's
// possible implicit device synchronisation is not acceptable.  For them,
// moe_plan_dispatch_static runs the same kernels on a scratch array that this
// file reserves statically in device memory.  It allocates nothing.
//
// The array lives in every GPU that loads the library, until the process
// exits, and all calls on a device share it: two calls whose kernels overlap
// on the GPU (different streams, no ordering between them) race on it.  The
// part of it that must start at zero is cleared by every call (an async
// memset on the call's stream); the rest is fully written before it is read.
#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) unsigned char g_plan_scratch[MOE_PLAN_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices];   // device address of g_plan_scratch, per device

// The device address of the scratch array on the current device.  The first
// call on a device looks it up (cudaGetSymbolAddress, which also loads this
// module on the device); later calls reuse it.
moe_status scratch_on_current_device(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_plan_dispatch_static(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                               const int32_t *expert_to_rank, const int32_t *src_rank,
                                               const moe_plan *plan, int32_t *err, cudaStream_t stream)
{
    const size_t need = moe_plan_dispatch_workspace(T, k, G, src_rank != nullptr);
    if (need > sizeof(g_plan_scratch)) return MOE_ERR_WORKSPACE;
    void *scratch = nullptr;
    const moe_status st = scratch_on_current_device(&scratch);
    if (st != MOE_OK) return st;
    return moe_plan_dispatch(ids, T, k, E, G, rpn, expert_to_rank, src_rank, plan, err, scratch,
                             sizeof(g_plan_scratch), stream);
}

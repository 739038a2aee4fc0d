// Library-wide entry points: status strings and launch accounting.
#include <atomic>

#include "common.cuh"

namespace moe {

static std::atomic<uint64_t> g_launches{0};

void note_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int sm_count()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace moe

extern "C" const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument";
    case MOE_ERR_DATA: return "invalid data";
    case MOE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    }
    return "unknown status";
}

extern "C" uint64_t moe_launch_count(void) { return moe::g_launches.load(std::memory_order_relaxed); }

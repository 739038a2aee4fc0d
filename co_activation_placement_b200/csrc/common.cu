// Library-wide entry points: status strings, launch accounting and the
// cooperative kernels' grid size.
#include <atomic>

#include "common.cuh"

namespace moe {

static std::atomic<uint64_t> g_launches{0};
static std::atomic<int> g_coop_blocks{0};

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

int coop_grid()
{
    const int n = g_coop_blocks.load(std::memory_order_relaxed), sms = sm_count();
    return n > 0 && n < sms ? n : sms;
}

}  // namespace moe

extern "C" int moe_cooperative_blocks(int blocks)
{
    if (blocks < 0) return -1;
    return moe::g_coop_blocks.exchange(blocks);
}

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

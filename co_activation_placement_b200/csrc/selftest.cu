// Self-test of the bounded waits (no counterpart on the pages): each launch
// makes one kind of wait run out on purpose -- a grid barrier that one block
// never reaches, an mbarrier phase that nothing completes -- and must end,
// after about the 2 s limit, with MOE_DERR_TIMEOUT in the error word and the
// context still usable.  The waits are the ones the balanced shuffle and the
// tensor-core statistics use (waits.cuh).
#include "common.cuh"
#include "waits.cuh"

namespace moe {
namespace {

__global__ void selftest_grid_kernel(GridBarrier *b, int32_t *err)
{
    if (blockIdx.x == 1) return;   // this block never arrives
    grid_barrier(b, err);
}

__global__ void selftest_mbar_kernel(int32_t *err)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // nothing arrives, so phase 0 never completes
    const bool done = mbar_wait(&bar, 0);
    if (!done && threadIdx.x == 0) record_error(err, MOE_DERR_TIMEOUT);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_selftest_workspace(void)
{
    return round_up(sizeof(GridBarrier), 256);
}

extern "C" moe_status moe_selftest_wait_timeout(int kind, int32_t *err, void *ws, size_t ws_bytes,
                                                cudaStream_t stream)
{
    if (!err || (kind != 0 && kind != 1)) return MOE_ERR_ARG;
    if (kind == 1) {
        selftest_mbar_kernel<<<1, 32, 0, stream>>>(err);
    } else {
        if (!ws || !aligned256(ws) || ws_bytes < sizeof(GridBarrier)) return MOE_ERR_WORKSPACE;
        if (cudaMemsetAsync(ws, 0, sizeof(GridBarrier), stream) != cudaSuccess) return MOE_ERR_CUDA;
        GridBarrier *b = static_cast<GridBarrier *>(ws);
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(4);
        cfg.blockDim = dim3(32);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, selftest_grid_kernel, b, err) != cudaSuccess) return MOE_ERR_CUDA;
    }
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

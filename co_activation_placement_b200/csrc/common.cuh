// Shared helpers of the libmoecoact CUDA sources (sm_100a).
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "moe_coact.h"

namespace moe {

// Count of kernels launched by this library (for benchmark accounting).
void note_launches(uint64_t n);

// Record the first device-side data error: the word keeps its first non-zero
// value.  Never traps.
__device__ __forceinline__ void record_error(int32_t *err, int32_t code)
{
    if (err) atomicCAS(err, 0, code);
}

// Opt a kernel into `bytes` of dynamic shared memory on the current device.
// Without the opt-in, static plus dynamic shared memory must stay within
// 48 KB, and several kernels here declare more than 24 KB statically (the
// plan's scatter 30 KB), so the opt-in is made whenever dynamic memory is
// used (cheap to repeat).
template <typename F>
inline cudaError_t allow_smem(F *kernel, size_t bytes)
{
    if (bytes == 0) return cudaSuccess;
    return cudaFuncSetAttribute(reinterpret_cast<const void *>(kernel),
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

inline moe_status launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of SMs of the current device (cached per device ordinal).
int sm_count();

// Blocks of a cooperative launch (moe_cooperative_blocks): one per SM unless
// a smaller count is set.
int coop_grid();

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the previous kernel on its stream is still running: it does the part
// of its work that reads only the call's own inputs, then pdl_wait() -- which
// returns once the previous kernel has completed and its writes are visible --
// before touching anything that kernel writes.  pdl_release() (called after
// the kernel's own pdl_wait, never before) lets the next kernel start early in
// turn, so a kernel can only start once the one two places before it is
// complete.  Both are no-ops for a kernel launched the ordinary way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe

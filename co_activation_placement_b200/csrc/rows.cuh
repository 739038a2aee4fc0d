// Helpers shared by the row kernels (permute, combine, pre-reduction) of
// one device and of several devices: the 16/32-byte streaming vector loads and
// stores, the element view of a vector, the per-token row lists and the grid
// size.
#pragma once

#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kRowThreads = 256;
// Permutes of at least this many tokens keep 8 32-byte vectors per lane in
// flight (2 resident blocks per SM at about 120 registers: measured 0.6%
// faster than 4 on 131072 tokens of 14 KB); smaller ones keep 4 (3 resident
// blocks, fewer waves: 6% faster on 16384 tokens of 8 KB).
constexpr int kDeepPermuteTokens = 32768;
constexpr int kRowBlocksPerSM = 16;   // two waves of resident blocks: measured best for permute and combine

// Warp-uniform per-token row list: dst[j] and a bitmask of the j that are the
// first occurrence of a valid row.  Returns false (after recording the error)
// if any row is out of range.
template <int K>
__device__ __forceinline__ bool token_rows(const int32_t *__restrict__ idx, int t, long long R_max,
                                           int (&dst)[K], unsigned &keep, int32_t *err)
{
    const int lane = threadIdx.x & 31;
    const int mine = lane < K ? __ldg(idx + (size_t)t * K + lane) : 0;
    bool ok = true;
    keep = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        dst[j] = __shfl_sync(0xffffffffu, mine, j);
        const bool valid = dst[j] >= 0 && (long long)dst[j] < R_max;
        ok &= valid;
        bool first = valid;
#pragma unroll
        for (int q = 0; q < j; ++q) first &= dst[q] != dst[j];
        keep |= (unsigned)first << j;
    }
    if (!ok && lane == 0) record_error(err, MOE_DERR_ROW_RANGE);
    return ok;
}

// One vector of VB bytes (16 or 32) as 32-bit words, moved with streaming
// (evict-first) loads and stores; 32-byte vectors use the 256-bit forms.
template <int VB> struct Vw { uint32_t w[VB / 4]; };

template <int VB>
__device__ __forceinline__ Vw<VB> ld_vec(const void *p)
{
    Vw<VB> v;
    if constexpr (VB == 16) {
        const uint4 a = __ldcs(static_cast<const uint4 *>(p));
        v.w[0] = a.x; v.w[1] = a.y; v.w[2] = a.z; v.w[3] = a.w;
    } else {
        asm volatile("ld.global.cs.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]),
                       "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
                     : "l"(p));
    }
    return v;
}

template <int NW>
__device__ __forceinline__ void st_words(void *p, const uint32_t (&w)[NW])
{
    // NW words at p: 8-word (32 B) pieces first, then 4, then 2
    static_assert(NW % 2 == 0, "even word count");
    uint32_t *q = static_cast<uint32_t *>(p);
    int o = 0;
#pragma unroll
    for (; o + 8 <= NW; o += 8)
        asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                     ::"l"(q + o), "r"(w[o]), "r"(w[o + 1]), "r"(w[o + 2]), "r"(w[o + 3]),
                       "r"(w[o + 4]), "r"(w[o + 5]), "r"(w[o + 6]), "r"(w[o + 7])
                     : "memory");
#pragma unroll
    for (; o + 4 <= NW; o += 4) __stcs(reinterpret_cast<uint4 *>(q + o), make_uint4(w[o], w[o + 1], w[o + 2], w[o + 3]));
#pragma unroll
    for (; o + 2 <= NW; o += 2) __stcs(reinterpret_cast<uint2 *>(q + o), make_uint2(w[o], w[o + 1]));
}

// Element e of a vector of Y.
template <typename YT> struct Elem;
template <> struct Elem<float> {
    static constexpr int BYTES = 4;
    template <int NW> __device__ static __forceinline__ float get(const uint32_t (&w)[NW], int e) { return __uint_as_float(w[e]); }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int BYTES = 2;
    template <int NW> __device__ static __forceinline__ float get(const uint32_t (&w)[NW], int e)
    {
        const uint32_t x = w[e >> 1];
        return __uint_as_float((e & 1) ? (x & 0xffff0000u) : (x << 16));
    }
};

// A token's distinct rows, compacted: lane j < K holds pick j's row and
// weight; a pick that repeats an earlier pick's row adds its weight to that
// earlier lane (in j order) and drops out.  Returns the number of distinct
// valid rows U; the q-th of them (in order of first appearance) is
// (shfl(row, src[q]), shfl(W, src[q])).
template <int K, bool UNIT>
__device__ __forceinline__ int token_distinct(const int32_t *__restrict__ idx, const float *__restrict__ w, int t,
                                              long long R_max, int &row, float &W, int (&src)[K], int32_t *err)
{
    const int lane = threadIdx.x & 31;
    row = lane < K ? __ldg(idx + (size_t)t * K + lane) : -1;
    // UNIT: every distinct row counts once with weight 1 (repeats add nothing)
    const float wl = UNIT ? 1.f : (lane < K ? __ldg(w + (size_t)t * K + lane) : 0.f);
    const bool valid = lane < K && row >= 0 && (long long)row < R_max;
    if (__any_sync(0xffffffffu, lane < K && !valid) && lane == 0) record_error(err, MOE_DERR_ROW_RANGE);
    bool first = valid;
    W = wl;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        const int rj = __shfl_sync(0xffffffffu, row, j);
        const float wj = __shfl_sync(0xffffffffu, wl, j);
        if (j < lane && rj == row) first = false;
        if (!UNIT && j > lane && rj == row) W = __fadd_rn(W, wj);
    }
    unsigned m = __ballot_sync(0xffffffffu, first);
    const int U = __popc(m);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        src[q] = m ? __ffs(m) - 1 : 0;
        m &= m - 1;
    }
    return U;
}

int row_grid(long long T)
{
    const long long want = (long long)sm_count() * kRowBlocksPerSM;
    const long long need = (T + (kRowThreads / 32) - 1) / (kRowThreads / 32);
    return (int)std::max<long long>(1, std::min(want, need));
}

size_t dtype_bytes(moe_dtype d) { return d == MOE_F32 ? 4 : (d == MOE_BF16 ? 2 : 0); }

}  // namespace
}  // namespace moe

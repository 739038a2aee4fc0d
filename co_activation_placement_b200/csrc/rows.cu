// Row permute into the rank-major send buffer and the weighted combine.
//
// "Expert Coupling in MoE Pretraining", abstract: tokens are dispatched to
// their experts, each token to each GPU once, "and then combine[d]";
// "Training Communication-Efficient MoE ...", footnote 3: the dispatcher moves
// hidden states (and routed probabilities), the combine is the inverse.
//
// Both kernels are HBM streams with 16-byte vectors; nothing here is a dense
// contraction.  Both are token-major: one warp owns one token at a time.
//  - permute reads the token's row of x once and writes it to each of its
//    distinct send rows (row_of[t][j], duplicates skipped), so HBM traffic is
//    T_active*rowB read + R*rowB written -- the minimum.
//  - combine reads each distinct row a token names once, sums the weights of
//    repeated rows in j order, and accumulates the distinct rows with fp32
//    FMAs in order of first appearance; traffic is U*rowB + T*rowB_out.
// Loads and stores use the streaming (evict-first) cache hint: every byte is
// touched once.  Grids are persistent: a multiple of the SM count.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kRowThreads = 256;
constexpr int kRowBlocksPerSM = 8;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(uint4 *p, const uint4 &v) { __stcs(p, v); }

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

template <int K, int U>
__global__ void __launch_bounds__(kRowThreads)
permute_kernel(const uint4 *__restrict__ x, int nvec, int T, const int32_t *__restrict__ row_of,
               long long R_max, uint4 *__restrict__ send, int32_t *err)
{
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    for (int t = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
        int dst[K];
        unsigned keep;
        token_rows<K>(row_of, t, R_max, dst, keep, err);
        const uint4 *src = x + (size_t)t * nvec;
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            uint4 buf[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < nvec) buf[u] = ld_stream(src + v0 + 32 * u);
#pragma unroll
            for (int j = 0; j < K; ++j) {
                if (!((keep >> j) & 1u)) continue;
                uint4 *o = send + (size_t)dst[j] * nvec;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < nvec) st_stream(o + v0 + 32 * u, buf[u]);
            }
        }
    }
}

// Element access for one 16-byte vector of Y.
template <typename YT> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ static __forceinline__ float get(const uint4 &v, int e)
    {
        const unsigned w = e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
        return __uint_as_float(w);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static __forceinline__ float get(const uint4 &v, int e)
    {
        const unsigned w = (e >> 1) == 0 ? v.x : (e >> 1) == 1 ? v.y : (e >> 1) == 2 ? v.z : v.w;
        return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
    }
};

template <int N, bool OUT_BF16>
__device__ __forceinline__ void store_out(void *out, size_t elem, const float (&a)[N])
{
    if constexpr (!OUT_BF16) {
        float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + elem);
#pragma unroll
        for (int q = 0; q < N / 4; ++q) __stcs(o + q, make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]));
    } else {
        unsigned w[N / 2];
#pragma unroll
        for (int q = 0; q < N / 2; ++q) {
            __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * q], a[2 * q + 1]);
            w[q] = *reinterpret_cast<unsigned *>(&h);
        }
        __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(out) + elem;
        if constexpr (N == 8) __stcs(reinterpret_cast<uint4 *>(ob), make_uint4(w[0], w[1], w[2], w[3]));
        else __stcs(reinterpret_cast<uint2 *>(ob), make_uint2(w[0], w[1]));
    }
}

template <int K, int U, typename YT, bool OUT_BF16>
__global__ void __launch_bounds__(kRowThreads)
combine_kernel(const uint4 *__restrict__ Y, int nvec, long long R_max, const int32_t *__restrict__ idx,
               const float *__restrict__ w, int T, void *__restrict__ out, int32_t *err)
{
    constexpr int N = Vec<YT>::N;
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    for (int t = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
        int row[K];
        unsigned keep;
        token_rows<K>(idx, t, R_max, row, keep, err);
        const float wm = lane < K ? __ldg(w + (size_t)t * K + lane) : 0.f;
        float W[K];
#pragma unroll
        for (int j = 0; j < K; ++j) W[j] = 0.f;
        // fold the weights of repeated rows onto their first occurrence, in j order
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const float wj = __shfl_sync(0xffffffffu, wm, j);
            bool placed = false;
#pragma unroll
            for (int q = 0; q < j; ++q) {
                const bool hit = !placed && ((keep >> q) & 1u) && row[q] == row[j];
                if (hit) W[q] = __fadd_rn(W[q], wj);
                placed |= hit;
            }
            if ((keep >> j) & 1u) W[j] = wj;
        }
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            uint4 y[U][K];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int j = 0; j < K; ++j)
                    if (((keep >> j) & 1u) && v0 + 32 * u < nvec)
                        y[u][j] = ld_stream(Y + (size_t)row[j] * nvec + v0 + 32 * u);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (v0 + 32 * u >= nvec) break;
                float acc[N];
#pragma unroll
                for (int e = 0; e < N; ++e) acc[e] = 0.f;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    if (!((keep >> j) & 1u)) continue;
#pragma unroll
                    for (int e = 0; e < N; ++e) acc[e] = __fmaf_rn(W[j], Vec<YT>::get(y[u][j], e), acc[e]);
                }
                store_out<N, OUT_BF16>(out, ((size_t)t * nvec + v0 + 32 * u) * N, acc);
            }
        }
    }
}

int row_grid(long long T)
{
    const long long want = (long long)sm_count() * kRowBlocksPerSM;
    const long long need = (T + (kRowThreads / 32) - 1) / (kRowThreads / 32);
    return (int)std::max<long long>(1, std::min(want, need));
}

template <int K>
moe_status launch_permute(const void *x, int nvec, int T, const int32_t *row_of, long long R_max, void *send,
                          int32_t *err, cudaStream_t s)
{
    permute_kernel<K, 4><<<row_grid(T), kRowThreads, 0, s>>>(static_cast<const uint4 *>(x), nvec, T, row_of, R_max,
                                                             static_cast<uint4 *>(send), err);
    return launch_status();
}

template <int K, typename YT>
moe_status launch_combine(const void *Y, int nvec, long long R_max, const int32_t *idx, const float *w, int T,
                          void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    constexpr int U = K <= 4 ? 2 : 1;
    const uint4 *y = static_cast<const uint4 *>(Y);
    if (out_bf16)
        combine_kernel<K, U, YT, true><<<row_grid(T), kRowThreads, 0, s>>>(y, nvec, R_max, idx, w, T, out, err);
    else
        combine_kernel<K, U, YT, false><<<row_grid(T), kRowThreads, 0, s>>>(y, nvec, R_max, idx, w, T, out, err);
    return launch_status();
}

template <typename YT>
moe_status dispatch_combine_k(int k, const void *Y, int nvec, long long R_max, const int32_t *idx, const float *w,
                              int T, void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    switch (k) {
    case 1: return launch_combine<1, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 2: return launch_combine<2, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 3: return launch_combine<3, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 4: return launch_combine<4, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 5: return launch_combine<5, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 6: return launch_combine<6, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 7: return launch_combine<7, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    case 8: return launch_combine<8, YT>(Y, nvec, R_max, idx, w, T, out, out_bf16, err, s);
    }
    return MOE_ERR_ARG;
}

size_t dtype_bytes(moe_dtype d) { return d == MOE_F32 ? 4 : (d == MOE_BF16 ? 2 : 0); }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_permute(const void *x, moe_dtype dtype, int T, int d, int k,
                                  const int32_t *row_of, int64_t R_max, void *send,
                                  int32_t *err, cudaStream_t stream)
{
    const size_t eb = dtype_bytes(dtype);
    if (!eb || T < 0 || d < 1 || k < 1 || k > 8 || R_max < 0 || !err) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !row_of || !send || !aligned16(x) || !aligned16(send)) return MOE_ERR_ARG;
    const size_t rowB = eb * (size_t)d;
    if (rowB % 16) return MOE_ERR_UNSUPPORTED;
    const int nvec = (int)(rowB / 16);
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_permute<1>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 2: st = launch_permute<2>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 3: st = launch_permute<3>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 4: st = launch_permute<4>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 5: st = launch_permute<5>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 6: st = launch_permute<6>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 7: st = launch_permute<7>(x, nvec, T, row_of, R_max, send, err, stream); break;
    case 8: st = launch_permute<8>(x, nvec, T, row_of, R_max, send, err, stream); break;
    }
    if (st == MOE_OK) note_launches(1);
    return st;
}

extern "C" moe_status moe_combine(const void *Y, moe_dtype y_dtype, int64_t R_max, int d,
                                  const int32_t *idx, const float *w, int T, int k,
                                  void *out, moe_dtype out_dtype, int32_t *err, cudaStream_t stream)
{
    const size_t eb = dtype_bytes(y_dtype);
    if (!eb || !dtype_bytes(out_dtype) || T < 0 || d < 1 || k < 1 || k > 8 || R_max < 0 || !err) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!Y || !idx || !w || !out || !aligned16(Y) || !aligned16(out)) return MOE_ERR_ARG;
    const size_t rowB = eb * (size_t)d;
    if (rowB % 16) return MOE_ERR_UNSUPPORTED;
    const int nvec = (int)(rowB / 16);
    const bool ob = out_dtype == MOE_BF16;
    moe_status st = y_dtype == MOE_BF16
                        ? dispatch_combine_k<__nv_bfloat16>(k, Y, nvec, R_max, idx, w, T, out, ob, err, stream)
                        : dispatch_combine_k<float>(k, Y, nvec, R_max, idx, w, T, out, ob, err, stream);
    if (st == MOE_OK) note_launches(1);
    return st;
}

// Row permute into the rank-major send buffer and the weighted combine.
//
// "Expert Coupling in MoE Pretraining", abstract: tokens are dispatched to
// their experts, each token to each GPU once, "and then combine[d]";
// "Training Communication-Efficient MoE ...", footnote 3: the dispatcher moves
// hidden states (and routed probabilities), the combine is the inverse.
//
// Both kernels are HBM streams of 32-byte vectors (the 256-bit
// ld/st.global.v8 forms; 16-byte vectors when a row or pointer is not 32-byte
// aligned); nothing here is a dense contraction.  Both are token-major: one
// warp owns one token at a time.
//  - permute reads the token's row of x once (8 or 4 32-byte vectors per lane
//    in flight, by launch size: kDeepPermuteTokens)
//    and writes it to each of its distinct send rows (row_of[t][j], duplicates
//    skipped), so HBM traffic is T_active*rowB read + R*rowB written -- the
//    minimum.  (A variant staging rows in shared memory with bulk async copies
//    measured 2% slower on B200 for 4-14 KB rows and was dropped.)
//  - combine folds the weights of repeated rows in j order (lane-parallel
//    across the token's k picks), compacts the distinct rows, loads them all
//    before accumulating with fp32 FMAs in order of first appearance; traffic
//    is U*rowB + T*rowB_out.
// Loads and stores use the streaming (evict-first) cache hint: every byte is
// touched once.  Grids are persistent: a multiple of the SM count.
#include "rows.cuh"

namespace moe {
namespace {

// Permute with VB-byte vectors: a warp reads a token's row once, U vectors
// per lane in flight, and writes them to each of the token's distinct rows.
template <int K, int U, int VB>
__global__ void __launch_bounds__(kRowThreads)
permute_kernel(const char *__restrict__ x, int nvec, int T, const int32_t *__restrict__ row_of,
               long long R_max, char *__restrict__ send, int32_t *err)
{
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    const size_t rowB = (size_t)nvec * VB;
    for (int t = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
        int dst[K];
        unsigned keep;
        token_rows<K>(row_of, t, R_max, dst, keep, err);
        const char *src = x + (size_t)t * rowB;
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            Vw<VB> buf[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < nvec) buf[u] = ld_vec<VB>(src + (size_t)(v0 + 32 * u) * VB);
#pragma unroll
            for (int j = 0; j < K; ++j) {
                if (!((keep >> j) & 1u)) continue;
                char *o = send + (size_t)dst[j] * rowB;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < nvec) st_words<VB / 4>(o + (size_t)(v0 + 32 * u) * VB, buf[u].w);
            }
        }
    }
}

// Vectors are VB bytes of Y (N elements).  Distinct rows are read in chunks
// of CH rows; U vectors per lane are in flight per row.
template <int K, int CH, int U, typename YT, bool OUT_BF16, int VB, bool UNIT>
__global__ void __launch_bounds__(kRowThreads)
combine_kernel(const char *__restrict__ Y, int nvec, long long R_max, const int32_t *__restrict__ idx,
               const float *__restrict__ w, int T, void *__restrict__ out, int32_t *err)
{
    constexpr int N = VB / Elem<YT>::BYTES;
    constexpr int OW = OUT_BF16 ? N / 2 : N;          // output words per vector
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    const size_t rowB = (size_t)nvec * VB;
    for (int t = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
        int row, src[K];
        float Wl;
        const int Ut = token_distinct<K, UNIT>(idx, w, t, R_max, row, Wl, src, err);
        int rc[K];
        float Wc[K];
#pragma unroll
        for (int q = 0; q < K; ++q) {
            rc[q] = __shfl_sync(0xffffffffu, row, src[q]);
            Wc[q] = __shfl_sync(0xffffffffu, Wl, src[q]);
        }
        char *ob = static_cast<char *>(out) + (size_t)t * nvec * (OW * 4);
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            float acc[U][N];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < N; ++e) acc[u][e] = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < K; c0 += CH) {
                if (c0 >= Ut) break;
                Vw<VB> y[CH][U];
#pragma unroll
                for (int c = 0; c < CH; ++c)
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c0 + c < K && c0 + c < Ut && v0 + 32 * u < nvec)
                            y[c][u] = ld_vec<VB>(Y + (size_t)rc[c0 + c] * rowB + (size_t)(v0 + 32 * u) * VB);
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    if (c0 + c >= K || c0 + c >= Ut) break;
#pragma unroll
                    for (int u = 0; u < U; ++u)
#pragma unroll
                        for (int e = 0; e < N; ++e)
                            acc[u][e] = __fmaf_rn(Wc[c0 + c], Elem<YT>::get(y[c][u].w, e), acc[u][e]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (v0 + 32 * u >= nvec) break;
                uint32_t o[OW];
                if constexpr (OUT_BF16) {
#pragma unroll
                    for (int q = 0; q < OW; ++q) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(acc[u][2 * q], acc[u][2 * q + 1]);
                        o[q] = *reinterpret_cast<uint32_t *>(&h);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < OW; ++q) o[q] = __float_as_uint(acc[u][q]);
                }
                st_words<OW>(ob + (size_t)(v0 + 32 * u) * (OW * 4), o);
            }
        }
    }
}

// Gate dispatch: row i (< R, read from the plan's summary on the device)
// carries (e_tj, w_tj) for the picks j of its token whose expert lives on the
// row's rank, (-1, 0) for the others.
__global__ void __launch_bounds__(kRowThreads)
dispatch_gates_kernel(const int32_t *__restrict__ ids, const float *__restrict__ w, int T, int k,
                      const int32_t *__restrict__ row_token, const uint8_t *__restrict__ row_jmask,
                      const int64_t *__restrict__ summary, long long R_max, int32_t *__restrict__ send_e,
                      float *__restrict__ send_w, int32_t *err)
{
    long long R = *summary;
    if (R > R_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_error(err, MOE_DERR_ROW_RANGE);
        R = R_max;
    }
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < R; i += (long long)gridDim.x * blockDim.x) {
        const int t = __ldg(row_token + i);
        const unsigned jm = __ldg(row_jmask + i);
        const bool ok = (unsigned)t < (unsigned)T;
        if (!ok) record_error(err, MOE_DERR_ROW_RANGE);
        for (int j = 0; j < k; ++j) {
            const bool on = ok && ((jm >> j) & 1u);
            send_e[i * k + j] = on ? __ldg(ids + (size_t)t * k + j) : -1;
            send_w[i * k + j] = on ? __ldg(w + (size_t)t * k + j) : 0.f;
        }
    }
}

// Receiver-side pre-reduction with stand-in experts (expert e maps a row x
// to scale[e] * x): y[i] = sum_j send_w[i][j] * scale[e_ij] * send[i] over the
// row's experts, one warp per row.  g_j = send_w * scale is rounded to fp32
// once, then the row is accumulated with fp32 FMAs in j order.
template <int K, typename YT, bool OUT_BF16, int VB>
__global__ void __launch_bounds__(kRowThreads)
expert_reduce_kernel(const char *__restrict__ send, int nvec, const int64_t *__restrict__ summary, long long R_max,
                     const int32_t *__restrict__ send_e, const float *__restrict__ send_w,
                     const float *__restrict__ scale, int E, void *__restrict__ y, int32_t *err)
{
    constexpr int N = VB / Elem<YT>::BYTES;
    constexpr int OW = OUT_BF16 ? N / 2 : N;
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    long long R = *summary;
    if (R > R_max) R = R_max;
    const size_t rowB = (size_t)nvec * VB;
    for (long long i = (long long)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); i < R; i += nwarps) {
        const int el = lane < K ? __ldg(send_e + i * K + lane) : -1;
        const bool bad = __any_sync(0xffffffffu, el >= E);
        if (bad && lane == 0) record_error(err, MOE_DERR_ID_RANGE);
        const float gl = (el >= 0 && el < E) ? __fmul_rn(__ldg(send_w + i * K + lane), __ldg(scale + el)) : 0.f;
        float g[K];
        bool on[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            g[j] = __shfl_sync(0xffffffffu, gl, j);
            on[j] = __shfl_sync(0xffffffffu, el, j) >= 0 && !bad;
        }
        const char *src = send + (size_t)i * rowB;
        char *dst = static_cast<char *>(y) + (size_t)i * nvec * (OW * 4);
        constexpr int U = 4;   // vectors per lane in flight
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            Vw<VB> x[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < nvec) x[u] = ld_vec<VB>(src + (size_t)(v0 + 32 * u) * VB);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (v0 + 32 * u >= nvec) break;
                float acc[N];
#pragma unroll
                for (int e = 0; e < N; ++e) acc[e] = 0.f;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    if (!on[j]) continue;
#pragma unroll
                    for (int e = 0; e < N; ++e) acc[e] = __fmaf_rn(g[j], Elem<YT>::get(x[u].w, e), acc[e]);
                }
                uint32_t o[OW];
                if constexpr (OUT_BF16) {
#pragma unroll
                    for (int q = 0; q < OW; ++q) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
                        o[q] = *reinterpret_cast<uint32_t *>(&h);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < OW; ++q) o[q] = __float_as_uint(acc[q]);
                }
                st_words<OW>(dst + (size_t)(v0 + 32 * u) * (OW * 4), o);
            }
        }
    }
}

template <int K>
moe_status launch_permute(const void *x, size_t rowB, int T, const int32_t *row_of, long long R_max, void *send,
                          int32_t *err, cudaStream_t s)
{
    const char *xb = static_cast<const char *>(x);
    char *sb = static_cast<char *>(send);
    if (rowB % 32 == 0 && (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && (reinterpret_cast<uintptr_t>(send) & 31u) == 0)
        if (T >= kDeepPermuteTokens)
            permute_kernel<K, 8, 32><<<row_grid(T), kRowThreads, 0, s>>>(xb, (int)(rowB / 32), T, row_of, R_max, sb, err);
        else
            permute_kernel<K, 4, 32><<<row_grid(T), kRowThreads, 0, s>>>(xb, (int)(rowB / 32), T, row_of, R_max, sb, err);
    else
        permute_kernel<K, 4, 16><<<row_grid(T), kRowThreads, 0, s>>>(xb, (int)(rowB / 16), T, row_of, R_max, sb, err);
    return launch_status();
}

// Combine tuning, measured on B200 at d = 7168 bf16, k = 8: one vector per
// lane in flight per distinct row, all distinct rows loaded before the FMAs
// (chunk = k), 32-byte vectors.
constexpr int kCombineU = 1;
constexpr int kCombineChunk = 8;

template <int K, typename YT, int VB, bool UNIT>
moe_status launch_combine_vb(const void *Y, int nvec, long long R_max, const int32_t *idx, const float *w, int T,
                             void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    constexpr int U = kCombineU;
    constexpr int CH = K < kCombineChunk ? K : kCombineChunk;
    const char *y = static_cast<const char *>(Y);
    if (out_bf16)
        combine_kernel<K, CH, U, YT, true, VB, UNIT><<<row_grid(T), kRowThreads, 0, s>>>(y, nvec, R_max, idx, w, T, out, err);
    else
        combine_kernel<K, CH, U, YT, false, VB, UNIT><<<row_grid(T), kRowThreads, 0, s>>>(y, nvec, R_max, idx, w, T, out, err);
    return launch_status();
}

// 32-byte vectors when Y and out are 32-byte aligned and rows split evenly
// into them (out rows are at least as long as Y rows), else 16-byte vectors.
template <int K, typename YT, bool UNIT>
moe_status launch_combine(const void *Y, size_t rowB, long long R_max, const int32_t *idx, const float *w, int T,
                          void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    const bool v32 = rowB % 32 == 0 && (reinterpret_cast<uintptr_t>(Y) & 31u) == 0 &&
                     (reinterpret_cast<uintptr_t>(out) & 31u) == 0 &&
                     (out_bf16 ? (sizeof(YT) == 2 || rowB % 64 == 0) : true);
    if (v32) return launch_combine_vb<K, YT, 32, UNIT>(Y, (int)(rowB / 32), R_max, idx, w, T, out, out_bf16, err, s);
    return launch_combine_vb<K, YT, 16, UNIT>(Y, (int)(rowB / 16), R_max, idx, w, T, out, out_bf16, err, s);
}

template <typename YT, bool UNIT>
moe_status dispatch_combine_k(int k, const void *Y, size_t rowB, long long R_max, const int32_t *idx, const float *w,
                              int T, void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    switch (k) {
    case 1: return launch_combine<1, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 2: return launch_combine<2, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 3: return launch_combine<3, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 4: return launch_combine<4, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 5: return launch_combine<5, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 6: return launch_combine<6, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 7: return launch_combine<7, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 8: return launch_combine<8, YT, UNIT>(Y, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    }
    return MOE_ERR_ARG;
}

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
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_permute<1>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 2: st = launch_permute<2>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 3: st = launch_permute<3>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 4: st = launch_permute<4>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 5: st = launch_permute<5>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 6: st = launch_permute<6>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 7: st = launch_permute<7>(x, rowB, T, row_of, R_max, send, err, stream); break;
    case 8: st = launch_permute<8>(x, rowB, T, row_of, R_max, send, err, stream); break;
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
    const bool ob = out_dtype == MOE_BF16;
    moe_status st = y_dtype == MOE_BF16
                        ? dispatch_combine_k<__nv_bfloat16, false>(k, Y, rowB, R_max, idx, w, T, out, ob, err, stream)
                        : dispatch_combine_k<float, false>(k, Y, rowB, R_max, idx, w, T, out, ob, err, stream);
    if (st == MOE_OK) note_launches(1);
    return st;
}

namespace moe {
namespace {

template <int K, typename YT, bool OB>
moe_status launch_reduce(const void *send, size_t rowB, const int64_t *summary, long long R_max, const int32_t *se,
                         const float *sw, const float *scale, int E, void *y, int32_t *err, cudaStream_t s)
{
    const char *sb = static_cast<const char *>(send);
    const bool v32 = rowB % 32 == 0 && (reinterpret_cast<uintptr_t>(send) & 31u) == 0 &&
                     (reinterpret_cast<uintptr_t>(y) & 31u) == 0 && (!OB || sizeof(YT) == 2 || rowB % 64 == 0);
    if (v32)
        expert_reduce_kernel<K, YT, OB, 32><<<row_grid(R_max), kRowThreads, 0, s>>>(sb, (int)(rowB / 32), summary, R_max,
                                                                                   se, sw, scale, E, y, err);
    else
        expert_reduce_kernel<K, YT, OB, 16><<<row_grid(R_max), kRowThreads, 0, s>>>(sb, (int)(rowB / 16), summary, R_max,
                                                                                   se, sw, scale, E, y, err);
    return launch_status();
}

template <typename YT, bool OB>
moe_status reduce_k(int k, const void *send, size_t rowB, const int64_t *summary, long long R_max, const int32_t *se,
                    const float *sw, const float *scale, int E, void *y, int32_t *err, cudaStream_t s)
{
    switch (k) {
    case 1: return launch_reduce<1, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 2: return launch_reduce<2, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 3: return launch_reduce<3, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 4: return launch_reduce<4, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 5: return launch_reduce<5, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 6: return launch_reduce<6, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 7: return launch_reduce<7, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    case 8: return launch_reduce<8, YT, OB>(send, rowB, summary, R_max, se, sw, scale, E, y, err, s);
    }
    return MOE_ERR_ARG;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_dispatch_gates(const int32_t *ids, const float *w, int T, int k,
                                         const int32_t *row_token, const uint8_t *row_jmask, const int64_t *summary,
                                         int64_t R_max, int32_t *send_e, float *send_w, int32_t *err,
                                         cudaStream_t stream)
{
    if (T < 0 || k < 1 || k > 8 || R_max < 0 || !err) return MOE_ERR_ARG;
    if (R_max == 0) return MOE_OK;
    if (!ids || !w || !row_token || !row_jmask || !summary || !send_e || !send_w) return MOE_ERR_ARG;
    dispatch_gates_kernel<<<row_grid(R_max / 8 + 1), kRowThreads, 0, stream>>>(ids, w, T, k, row_token, row_jmask,
                                                                               summary, R_max, send_e, send_w, err);
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

extern "C" moe_status moe_expert_reduce(const void *send, moe_dtype dtype, int64_t R_max, int d,
                                        const int64_t *summary, const int32_t *send_e, const float *send_w, int k,
                                        const float *scale, int E, void *y, moe_dtype y_dtype, int32_t *err,
                                        cudaStream_t stream)
{
    const size_t eb = dtype_bytes(dtype);
    if (!eb || !dtype_bytes(y_dtype) || R_max < 0 || d < 1 || k < 1 || k > 8 || E < 1 || !err) return MOE_ERR_ARG;
    if (R_max == 0) return MOE_OK;
    if (!send || !summary || !send_e || !send_w || !scale || !y || !aligned16(send) || !aligned16(y)) return MOE_ERR_ARG;
    const size_t rowB = eb * (size_t)d;
    if (rowB % 16) return MOE_ERR_UNSUPPORTED;
    const bool ob = y_dtype == MOE_BF16;
    moe_status st;
    if (dtype == MOE_BF16)
        st = ob ? reduce_k<__nv_bfloat16, true>(k, send, rowB, summary, R_max, send_e, send_w, scale, E, y, err, stream)
                : reduce_k<__nv_bfloat16, false>(k, send, rowB, summary, R_max, send_e, send_w, scale, E, y, err, stream);
    else
        st = ob ? reduce_k<float, true>(k, send, rowB, summary, R_max, send_e, send_w, scale, E, y, err, stream)
                : reduce_k<float, false>(k, send, rowB, summary, R_max, send_e, send_w, scale, E, y, err, stream);
    if (st == MOE_OK) note_launches(1);
    return st;
}

extern "C" moe_status moe_combine_rows(const void *Y, moe_dtype y_dtype, int64_t R_max, int d, const int32_t *row_of,
                                       int T, int k, void *out, moe_dtype out_dtype, int32_t *err, cudaStream_t stream)
{
    const size_t eb = dtype_bytes(y_dtype);
    if (!eb || !dtype_bytes(out_dtype) || T < 0 || d < 1 || k < 1 || k > 8 || R_max < 0 || !err) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!Y || !row_of || !out || !aligned16(Y) || !aligned16(out)) return MOE_ERR_ARG;
    const size_t rowB = eb * (size_t)d;
    if (rowB % 16) return MOE_ERR_UNSUPPORTED;
    const bool ob = out_dtype == MOE_BF16;
    moe_status st = y_dtype == MOE_BF16
                        ? dispatch_combine_k<__nv_bfloat16, true>(k, Y, rowB, R_max, row_of, nullptr, T, out, ob, err, stream)
                        : dispatch_combine_k<float, true>(k, Y, rowB, R_max, row_of, nullptr, T, out, ob, err, stream);
    if (st == MOE_OK) note_launches(1);
    return st;
}

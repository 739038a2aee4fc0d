// Expert parallelism over several devices: the rows of the deduplicated
// dispatch stored straight into the receiving devices' buffers, and the
// combine loading them back from there.
//
// "Expert Coupling in MoE Pretraining", abstract: each token is sent to each
// GPU once and the expert outputs are then combined; "Training
// Communication-Efficient MoE ...", footnote 3: hidden states and routed
// probabilities are dispatched, the combine is the inverse exchange.
//
// The G ranks are spread over W devices, Gl = G/W consecutive ranks per
// device.  Device h's receive buffer holds the rows addressed to its ranks in
// the order a one-device plan over all tokens gives them: destination rank,
// then source rank, then token.  Each device plans its own tokens (source
// ranks in its own range), so its local rows come in segments (r, s) for
// every destination rank r and local source rank s; moe_ep_routes turns the
// gathered per-source counts into, for each segment, the shift from a local
// row index to its row in the receiving device's buffer.  The permute and
// the combine are the one-device kernels with each row's address looked up
// per token: lane j of the token's warp finds pick j's segment by binary
// search over the segment starts (L1-resident, a few hundred bytes per rank).
// Rows cross devices as plain 16/32-byte stores and loads through peer
// pointers (NVLink), never through TMA; every store kernel ends with a
// system-scope fence so that a later cross-device signal orders after it.
#include "rows.cuh"

namespace moe {
namespace {

constexpr int kRouteThreads = 1024;

// Exclusive prefix of counts_all read in (destination, source) order, then
// the per-segment starts and shifts.  One block; G*G <= 4096 entries, at most
// 4 per thread.
__global__ void __launch_bounds__(kRouteThreads)
ep_routes_kernel(const int32_t *__restrict__ counts_all, const int32_t *__restrict__ offsets, int G, int W, int me,
                 int64_t *__restrict__ route, int32_t *err)
{
    __shared__ long long off[64 * 64 + 1];
    __shared__ long long warp_tot[kRouteThreads / 32];
    const int n = G * G;
    const int per = (n + kRouteThreads - 1) / kRouteThreads;
    const int i0 = threadIdx.x * per;
    long long v[4] = {0, 0, 0, 0};
    long long sum = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int i = i0 + q;
        if (q < per && i < n) {
            int c = __ldg(counts_all + (size_t)(i % G) * G + i / G);   // counts_all[s][r] for i = r*G + s
            if (c < 0) {
                record_error(err, MOE_DERR_ROW_RANGE);
                c = 0;
            }
            v[q] = c;
            sum += c;
        }
    }
    // block-wide exclusive scan of the per-thread sums
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        long long t = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_tot[lane] = t;                            // inclusive over warps
    }
    __syncthreads();
    long long run = inc - sum + (warp ? warp_tot[warp - 1] : 0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int i = i0 + q;
        if (q < per && i < n) {
            off[i] = run;
            run += v[q];
        }
    }
    if (threadIdx.x == kRouteThreads - 1) off[n] = warp_tot[kRouteThreads / 32 - 1];
    __syncthreads();
    const int Gl = G / W, P = G * Gl;
    for (int i = threadIdx.x; i < P; i += kRouteThreads) {
        const int r = i / Gl, s = me * Gl + i % Gl;
        const long long start = __ldg(offsets + r * G + s);
        const long long len = (long long)__ldg(offsets + r * G + s + 1) - start;
        if (len != off[r * G + s + 1] - off[r * G + s]) record_error(err, MOE_DERR_ROW_RANGE);
        const long long base_h = off[(size_t)(r / Gl) * Gl * G];   // first row of device r/Gl's buffer
        route[1 + i] = start;
        route[P + 2 + i] = off[r * G + s] - base_h - start;
    }
    if (threadIdx.x == 0) {
        route[1 + P] = __ldg(offsets + n);
        route[0] = off[(size_t)(me + 1) * Gl * G] - off[(size_t)me * Gl * G];
    }
}

// Where local row x lands: its receiving device's buffer and row there, as an
// address; nullptr when x is not a row of the local plan, the row falls
// outside [0, cap) or the buffer is not 32-byte aligned.
struct Routes {
    const int64_t *route;                 // [2P + 2], see moe_ep_routes
    const unsigned long long *base;       // [W] device addresses of the W buffers
    int P, Gl;
    long long cap;                        // rows in every buffer
};

__device__ __forceinline__ char *route_row(const Routes &rt, long long x, size_t rowB)
{
    const int64_t *start = rt.route + 1;
    if (x < __ldg(start) || x >= __ldg(start + rt.P)) return nullptr;
    int lo = 0, hi = rt.P;                // start[lo] <= x < start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(start + mid) <= x) lo = mid;
        else hi = mid;
    }
    const long long q = x + __ldg(rt.route + rt.P + 2 + lo);
    if (q < 0 || q >= rt.cap) return nullptr;
    const unsigned long long b = __ldg(rt.base + lo / rt.Gl / rt.Gl);
    if (b == 0 || (b & 31u)) return nullptr;
    return reinterpret_cast<char *>(b) + (size_t)q * rowB;
}

__device__ __forceinline__ char *shfl_ptr(char *p, int src)
{
    return reinterpret_cast<char *>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(p), src));
}

// Permute to the receiving devices: a warp reads a token's row of x once (U
// vectors per lane in flight) and stores it to each of its distinct rows.
template <int K, int U, int VB>
__global__ void __launch_bounds__(kRowThreads)
ep_permute_kernel(const char *__restrict__ x, int nvec, int T, const int32_t *__restrict__ row_of, long long R_max,
                  Routes rt, int32_t *err)
{
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    const size_t rowB = (size_t)nvec * VB;
    for (int t = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
        int dst[K];
        unsigned keep;
        token_rows<K>(row_of, t, R_max, dst, keep, err);
        // lane j < K: the address of pick j's row (first occurrences only)
        const int mine = lane < K ? __ldg(row_of + (size_t)t * K + lane) : -1;
        char *a = nullptr;
        bool bad = false;
        if (lane < K && ((keep >> lane) & 1u)) {
            a = route_row(rt, mine, rowB);
            bad = a == nullptr;
        }
        if (bad) record_error(err, MOE_DERR_ROW_RANGE);
        char *o[K];
#pragma unroll
        for (int j = 0; j < K; ++j) o[j] = shfl_ptr(a, j);
        const char *src = x + (size_t)t * rowB;
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            Vw<VB> buf[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < nvec) buf[u] = ld_vec<VB>(src + (size_t)(v0 + 32 * u) * VB);
#pragma unroll
            for (int j = 0; j < K; ++j) {
                if (!o[j]) continue;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < nvec) st_words<VB / 4>(o[j] + (size_t)(v0 + 32 * u) * VB, buf[u].w);
            }
        }
    }
    __threadfence_system();
}

// Combine from the receiving devices' buffers: the one-device combine (or,
// with UNIT, the unit-weight sum of a token's distinct rows) with every
// distinct row loaded from its device.
template <int K, int CH, int U, typename YT, bool OUT_BF16, int VB, bool UNIT>
__global__ void __launch_bounds__(kRowThreads)
ep_combine_kernel(Routes rt, int nvec, long long R_max, const int32_t *__restrict__ idx, const float *__restrict__ w,
                  int T, void *__restrict__ out, int32_t *err)
{
    constexpr int N = VB / Elem<YT>::BYTES;
    constexpr int OW = OUT_BF16 ? N / 2 : N;
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kRowThreads / 32);
    const size_t rowB = (size_t)nvec * VB;
    for (int t = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
        int row, src[K];
        float Wl;
        const int Ut = token_distinct<K, UNIT>(idx, w, t, R_max, row, Wl, src, err);
        char *a = nullptr;
        if (lane < K && row >= 0 && (long long)row < R_max) {
            a = route_row(rt, row, rowB);
            if (!a) record_error(err, MOE_DERR_ROW_RANGE);
        }
        const char *yp[K];
        float Wc[K];
#pragma unroll
        for (int q = 0; q < K; ++q) {
            yp[q] = shfl_ptr(a, src[q]);
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
                        if (c0 + c < K && c0 + c < Ut && yp[c0 + c] && v0 + 32 * u < nvec)
                            y[c][u] = ld_vec<VB>(yp[c0 + c] + (size_t)(v0 + 32 * u) * VB);
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    if (c0 + c >= K || c0 + c >= Ut) break;
                    if (!yp[c0 + c]) continue;
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

// Small per-row records (the gates of a row) to the receiving devices: one
// thread per local row x < R (R = route[1 + P]), 4-byte words.
__global__ void __launch_bounds__(kRowThreads)
ep_scatter_rows_kernel(const uint32_t *__restrict__ src, int words, long long R_max, Routes rt, int32_t *err)
{
    long long R = __ldg(rt.route + 1 + rt.P);
    if (R > R_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_error(err, MOE_DERR_ROW_RANGE);
        R = R_max;
    }
    const size_t recB = (size_t)words * 4;
    for (long long x = (long long)blockIdx.x * kRowThreads + threadIdx.x; x < R;
         x += (long long)gridDim.x * kRowThreads) {
        char *a = route_row(rt, x, recB);
        if (!a) {
            record_error(err, MOE_DERR_ROW_RANGE);
            continue;
        }
        uint32_t *d = reinterpret_cast<uint32_t *>(a);
        for (int q = 0; q < words; ++q) d[q] = __ldg(src + (size_t)x * words + q);
    }
    __threadfence_system();
}

template <int K>
moe_status launch_ep_permute(const void *x, size_t rowB, int T, const int32_t *row_of, long long R_max,
                             const Routes &rt, int32_t *err, cudaStream_t s)
{
    const char *xb = static_cast<const char *>(x);
    if (rowB % 32 == 0 && (reinterpret_cast<uintptr_t>(x) & 31u) == 0)
        if (T >= kDeepPermuteTokens)
            ep_permute_kernel<K, 8, 32><<<row_grid(T), kRowThreads, 0, s>>>(xb, (int)(rowB / 32), T, row_of, R_max, rt, err);
        else
            ep_permute_kernel<K, 4, 32><<<row_grid(T), kRowThreads, 0, s>>>(xb, (int)(rowB / 32), T, row_of, R_max, rt, err);
    else
        ep_permute_kernel<K, 4, 16><<<row_grid(T), kRowThreads, 0, s>>>(xb, (int)(rowB / 16), T, row_of, R_max, rt, err);
    return launch_status();
}

template <int K, typename YT, bool UNIT>
moe_status launch_ep_combine(const Routes &rt, size_t rowB, long long R_max, const int32_t *idx, const float *w,
                             int T, void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    constexpr int CH = K;            // every distinct row loaded before the FMAs (as the one-device combine)
    const bool v32 = rowB % 32 == 0 && (reinterpret_cast<uintptr_t>(out) & 31u) == 0 &&
                     (out_bf16 ? (sizeof(YT) == 2 || rowB % 64 == 0) : true);
    if (v32) {
        const int nvec = (int)(rowB / 32);
        if (out_bf16)
            ep_combine_kernel<K, CH, 1, YT, true, 32, UNIT><<<row_grid(T), kRowThreads, 0, s>>>(rt, nvec, R_max, idx, w, T, out, err);
        else
            ep_combine_kernel<K, CH, 1, YT, false, 32, UNIT><<<row_grid(T), kRowThreads, 0, s>>>(rt, nvec, R_max, idx, w, T, out, err);
    } else {
        const int nvec = (int)(rowB / 16);
        if (out_bf16)
            ep_combine_kernel<K, CH, 1, YT, true, 16, UNIT><<<row_grid(T), kRowThreads, 0, s>>>(rt, nvec, R_max, idx, w, T, out, err);
        else
            ep_combine_kernel<K, CH, 1, YT, false, 16, UNIT><<<row_grid(T), kRowThreads, 0, s>>>(rt, nvec, R_max, idx, w, T, out, err);
    }
    return launch_status();
}

template <typename YT, bool UNIT>
moe_status ep_combine_k(int k, const Routes &rt, size_t rowB, long long R_max, const int32_t *idx, const float *w,
                        int T, void *out, bool out_bf16, int32_t *err, cudaStream_t s)
{
    switch (k) {
    case 1: return launch_ep_combine<1, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 2: return launch_ep_combine<2, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 3: return launch_ep_combine<3, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 4: return launch_ep_combine<4, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 5: return launch_ep_combine<5, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 6: return launch_ep_combine<6, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 7: return launch_ep_combine<7, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    case 8: return launch_ep_combine<8, YT, UNIT>(rt, rowB, R_max, idx, w, T, out, out_bf16, err, s);
    }
    return MOE_ERR_ARG;
}

bool ep_shape_ok(int G, int W, int me)
{
    return G >= 1 && G <= 64 && W >= 1 && G % W == 0 && me >= 0 && me < W;
}

Routes make_routes(const int64_t *route, void *const *base, int G, int W, long long cap)
{
    Routes rt;
    rt.route = route;
    rt.base = reinterpret_cast<const unsigned long long *>(base);
    rt.Gl = G / W;
    rt.P = G * rt.Gl;
    rt.cap = cap;
    return rt;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_ep_routes(const int32_t *counts_all, const int32_t *offsets, int G, int W, int me,
                                    int64_t *route, int32_t *err, cudaStream_t stream)
{
    if (!ep_shape_ok(G, W, me) || !counts_all || !offsets || !route || !err) return MOE_ERR_ARG;
    ep_routes_kernel<<<1, kRouteThreads, 0, stream>>>(counts_all, offsets, G, W, me, route, err);
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

extern "C" moe_status moe_ep_permute(const void *x, moe_dtype dtype, int T, int d, int k, const int32_t *row_of,
                                     int64_t R_max, const int64_t *route, int G, int W, void *const *recv_base,
                                     int64_t recv_cap, int32_t *err, cudaStream_t stream)
{
    const size_t eb = dtype_bytes(dtype);
    if (!eb || T < 0 || d < 1 || k < 1 || k > 8 || R_max < 0 || recv_cap < 0 || !err) return MOE_ERR_ARG;
    if (!ep_shape_ok(G, W, 0)) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !row_of || !route || !recv_base || !aligned16(x)) return MOE_ERR_ARG;
    const size_t rowB = eb * (size_t)d;
    if (rowB % 16) return MOE_ERR_UNSUPPORTED;
    const Routes rt = make_routes(route, recv_base, G, W, recv_cap);
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_ep_permute<1>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 2: st = launch_ep_permute<2>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 3: st = launch_ep_permute<3>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 4: st = launch_ep_permute<4>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 5: st = launch_ep_permute<5>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 6: st = launch_ep_permute<6>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 7: st = launch_ep_permute<7>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    case 8: st = launch_ep_permute<8>(x, rowB, T, row_of, R_max, rt, err, stream); break;
    }
    if (st == MOE_OK) note_launches(1);
    return st;
}

extern "C" moe_status moe_ep_combine(void *const *y_base, moe_dtype y_dtype, int64_t y_cap, int d,
                                     const int64_t *route, int G, int W, int64_t R_max, const int32_t *idx,
                                     const float *w, int T, int k, void *out, moe_dtype out_dtype, int32_t *err,
                                     cudaStream_t stream)
{
    const size_t eb = dtype_bytes(y_dtype);
    if (!eb || !dtype_bytes(out_dtype) || T < 0 || d < 1 || k < 1 || k > 8 || R_max < 0 || y_cap < 0 || !err)
        return MOE_ERR_ARG;
    if (!ep_shape_ok(G, W, 0)) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!y_base || !route || !idx || !out || !aligned16(out)) return MOE_ERR_ARG;
    const size_t rowB = eb * (size_t)d;
    if (rowB % 16) return MOE_ERR_UNSUPPORTED;
    const Routes rt = make_routes(route, y_base, G, W, y_cap);
    const bool ob = out_dtype == MOE_BF16;
    moe_status st;
    if (w)
        st = y_dtype == MOE_BF16 ? ep_combine_k<__nv_bfloat16, false>(k, rt, rowB, R_max, idx, w, T, out, ob, err, stream)
                                 : ep_combine_k<float, false>(k, rt, rowB, R_max, idx, w, T, out, ob, err, stream);
    else
        st = y_dtype == MOE_BF16 ? ep_combine_k<__nv_bfloat16, true>(k, rt, rowB, R_max, idx, nullptr, T, out, ob, err, stream)
                                 : ep_combine_k<float, true>(k, rt, rowB, R_max, idx, nullptr, T, out, ob, err, stream);
    if (st == MOE_OK) note_launches(1);
    return st;
}

extern "C" moe_status moe_ep_scatter_rows(const void *src, int64_t row_bytes, int64_t R_max, const int64_t *route,
                                          int G, int W, void *const *dst_base, int64_t dst_cap, int32_t *err,
                                          cudaStream_t stream)
{
    if (row_bytes < 4 || row_bytes % 4 || row_bytes > 1024 || R_max < 0 || dst_cap < 0 || !err) return MOE_ERR_ARG;
    if (!ep_shape_ok(G, W, 0)) return MOE_ERR_ARG;
    if (R_max == 0) return MOE_OK;
    if (!src || !route || !dst_base || (reinterpret_cast<uintptr_t>(src) & 3u)) return MOE_ERR_ARG;
    const Routes rt = make_routes(route, dst_base, G, W, dst_cap);
    const long long want = (long long)sm_count() * 8;
    const long long need = (R_max + kRowThreads - 1) / kRowThreads;
    const int grid = (int)std::max<long long>(1, std::min(want, need));
    ep_scatter_rows_kernel<<<grid, kRowThreads, 0, stream>>>(static_cast<const uint32_t *>(src), (int)(row_bytes / 4),
                                                             R_max, rt, err);
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

// Rows that cross devices in the exchange: sent[h] = rows from device h's
// source ranks to other devices' ranks, received[h] = rows to device h's
// ranks from other devices' sources; each such row crosses once in the
// dispatch and once back in the combine.
extern "C" moe_status moe_ep_exchange_rows(const int32_t *counts_all, int G, int W, long long *sent,
                                           long long *received)
{
    if (!counts_all || !sent || !received || G < 1 || G > 64 || W < 1 || G % W) return MOE_ERR_ARG;
    const int Gl = G / W;
    for (int h = 0; h < W; ++h) sent[h] = received[h] = 0;
    for (int s = 0; s < G; ++s)
        for (int r = 0; r < G; ++r) {
            const int32_t c = counts_all[(size_t)s * G + r];
            if (c < 0) return MOE_ERR_ARG;
            if (s / Gl != r / Gl) {
                sent[s / Gl] += c;
                received[r / Gl] += c;
            }
        }
    return MOE_OK;
}

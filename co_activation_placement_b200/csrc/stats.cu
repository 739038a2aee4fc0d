// Co-activation counts, Ochiai similarity and cross-layer transition counts.
//
// Definitions ("Expert Coupling in MoE Pretraining", abstract: pairs of
// experts selected together, and next-layer experts predicted by this layer's;
// "Cobalt", "Key Observation": Ochiai over the experts' token sets):
//   C_l[i][j] = |{t : i, j in D_t^l}|,   S_l = C_ij / sqrt(C_ii C_jj),
//   M_l[i][j] = |{t : i in D_t^l, j in D_t^{l+1}}|.
//
// Design (sm_100a).  The work is a histogram: k(k+1)/2 counter increments per
// token and layer for C (upper triangle incl. diagonal) and k^2 per token and
// layer pair for M.  Each thread block owns one "group" -- (C of layer l, a band
// of triangle rows) or (M of layer pair l, a band of rows) -- small enough to
// live as uint32 counters in shared memory (about 64 KB, three blocks per SM),
// and one contiguous token slice; M blocks take q times shorter slices than C
// blocks so that both kinds do about the same number of increments.  Threads
// take one token at a time, load its k ids with vector loads, sort them with a
// compare-exchange network (C only) and issue shared-memory atomic adds.  M rows
// are padded to an odd stride, so that tokens incrementing the same column
// (a popular next-layer expert) in different rows hit different banks.  Only C
// blocks check ids for repeats (M blocks keep the range check that guards the
// histogram) unless C is not computed.  Blocks are numbered slice-major, so the
// blocks reading the same token slice run in the same wave and share it
// through L2.  Each block writes its counters once, coalesced, to a partial
// buffer; a second kernel sums the partials of each cell (integer, so the
// result does not depend on order), mirrors the triangle and evaluates Ochiai
// in fp64 with IEEE-rounded multiply, square root and divide.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "stats_mma.cuh"

namespace moe {
namespace {

constexpr int kHistThreads = 512;
constexpr int kMaxBands = 64;
constexpr int kBudgetCells = 16384;      // C: 64 KB of uint32 counters per block
constexpr int kBudgetWords = 16640;      // M: the same plus row padding
constexpr int kTargetBlocks = 148 * 3;   // one wave at three blocks per SM
constexpr int kMinSliceTokens = 2048;
constexpr int kReduceThreads = 256;

struct StatsGeom {
    int L, T, k, E;
    int Jc, Jt;          // groups: Jc = L*nbc (0 if no C wanted), Jt = (L-1)*nbt
    int nbc, nbt;        // bands of C (triangle rows) and of M (rows)
    int S, q;            // C slices S; M sub-slices S*q
    int rows_t;          // rows per M band
    int tstride;         // shared-memory row stride of an M band (odd)
    int max_words;       // shared memory words per block
    long long c_layer;   // partial words per C layer  = S * E(E+1)/2
    long long t_layer;   // partial words per M layer  = S*q * E*E
    long long c_total;   // Jc ? L * c_layer : 0
    int band_c[kMaxBands + 1];
};

__host__ __device__ inline long long tri_start(int i, int E)
{
    return (long long)i * E - (long long)i * (i - 1) / 2;
}

bool make_geom(int L, int T, int k, int E, bool want_c, bool want_t, StatsGeom &g)
{
    g = StatsGeom{};
    g.L = L; g.T = T; g.k = k; g.E = E;
    const long long tri_all = tri_start(E, E);
    // C bands: equal shares of the triangle, each within the counter budget
    int nbc = 0;
    if (want_c) {
        nbc = (int)((tri_all + kBudgetCells - 1) / kBudgetCells);
        for (;; ++nbc) {
            if (nbc > kMaxBands) return false;
            g.band_c[0] = 0;
            bool ok = true;
            int r = 0;
            for (int b = 1; b <= nbc; ++b) {
                long long want = tri_all * b / nbc;
                while (r < E && tri_start(r, E) < want) ++r;
                g.band_c[b] = (b == nbc) ? E : r;
                long long cells = tri_start(g.band_c[b], E) - tri_start(g.band_c[b - 1], E);
                if (cells > kBudgetCells || g.band_c[b] <= g.band_c[b - 1]) ok = false;
            }
            if (ok) break;
        }
    }
    // M bands: as few as fit the budget with rows padded to an odd stride
    int nbt = 0;
    g.tstride = E | 1;
    if (want_t && L > 1) {
        const int rows_fit = std::max(1, kBudgetWords / g.tstride);
        nbt = (E + rows_fit - 1) / rows_fit;
        g.rows_t = (E + nbt - 1) / nbt;
        nbt = (E + g.rows_t - 1) / g.rows_t;
        if (nbt > kMaxBands) return false;
    }
    g.nbc = nbc;
    g.nbt = nbt;
    g.Jc = want_c ? L * nbc : 0;
    g.Jt = (want_t && L > 1) ? (L - 1) * nbt : 0;
    if (g.Jc + g.Jt == 0) return false;
    // an M block does k^2/nbt increments per token, a C block about k(k+1)/2/nbc
    g.q = (g.Jc && g.Jt) ? std::max(1, (int)(2.0 * k * nbc / ((k + 1.0) * nbt) + 0.5)) : 1;
    const int per_slice = g.Jc + g.Jt * g.q;
    int S = (kTargetBlocks + per_slice / 2) / per_slice;
    S = std::max(1, std::min(S, std::max(1, T / kMinSliceTokens)));
    g.S = S;
    int mw = 0;
    for (int b = 0; b < nbc; ++b)
        mw = std::max(mw, (int)(tri_start(g.band_c[b + 1], E) - tri_start(g.band_c[b], E)));
    if (nbt) mw = std::max(mw, g.rows_t * g.tstride);
    g.max_words = mw;
    g.c_layer = (long long)S * tri_all;
    g.t_layer = (long long)S * g.q * E * E;
    g.c_total = g.Jc ? (long long)L * g.c_layer : 0;
    return true;
}

long long partial_words(const StatsGeom &g)
{
    return g.c_total + (g.Jt ? (long long)(g.L - 1) * g.t_layer : 0);
}

// Load token t's K ids; VEC selects 16- or 8-byte vector loads (the host checks
// the base alignment).
template <int K, bool VEC>
__device__ __forceinline__ void load_ids(const int32_t *__restrict__ p, int (&v)[K])
{
    if constexpr (VEC && K % 4 == 0) {
#pragma unroll
        for (int q = 0; q < K / 4; ++q) {
            int4 a = __ldg(reinterpret_cast<const int4 *>(p) + q);
            v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
        }
    } else if constexpr (VEC && K % 2 == 0) {
#pragma unroll
        for (int q = 0; q < K / 2; ++q) {
            int2 a = __ldg(reinterpret_cast<const int2 *>(p) + q);
            v[2 * q] = a.x; v[2 * q + 1] = a.y;
        }
    } else {
#pragma unroll
        for (int q = 0; q < K; ++q) v[q] = __ldg(p + q);
    }
}

__device__ __forceinline__ void cmpx(int &a, int &b)
{
    const int lo = min(a, b), hi = max(a, b);
    a = lo;
    b = hi;
}

// Ascending sort of K ids: Batcher's 19-comparator network for K = 8, a
// bubble network otherwise.
template <int K>
__device__ __forceinline__ void sort_ids(int (&v)[K])
{
    if constexpr (K == 8) {
        cmpx(v[0], v[1]); cmpx(v[2], v[3]); cmpx(v[4], v[5]); cmpx(v[6], v[7]);
        cmpx(v[0], v[2]); cmpx(v[1], v[3]); cmpx(v[4], v[6]); cmpx(v[5], v[7]);
        cmpx(v[1], v[2]); cmpx(v[5], v[6]);
        cmpx(v[0], v[4]); cmpx(v[1], v[5]); cmpx(v[2], v[6]); cmpx(v[3], v[7]);
        cmpx(v[2], v[4]); cmpx(v[3], v[5]);
        cmpx(v[1], v[2]); cmpx(v[3], v[4]); cmpx(v[5], v[6]);
    } else {
#pragma unroll
        for (int i = 0; i < K; ++i)
#pragma unroll
            for (int j = 0; j + 1 < K - i; ++j) cmpx(v[j], v[j + 1]);
    }
}

// 0 when the K ids are distinct and in [0, E), else the device error code.
template <int K>
__device__ __forceinline__ int check_ids(const int (&v)[K], int E)
{
    int bad_range = 0, bad_rep = 0;
#pragma unroll
    for (int a = 0; a < K; ++a) {
        bad_range |= (unsigned)v[a] >= (unsigned)E;
#pragma unroll
        for (int b = 0; b < a; ++b) bad_rep |= v[a] == v[b];
    }
    return bad_range ? MOE_DERR_ID_RANGE : (bad_rep ? MOE_DERR_ID_REPEAT : 0);
}

template <int K>
__device__ __forceinline__ bool ids_in_range(const int (&v)[K], int E)
{
    bool ok = true;
#pragma unroll
    for (int a = 0; a < K; ++a) ok &= (unsigned)v[a] < (unsigned)E;
    return ok;
}

template <int K, bool VEC>
__global__ void __launch_bounds__(kHistThreads)
stats_hist_kernel(const int32_t *__restrict__ ids, StatsGeom G, uint32_t *__restrict__ part, int32_t *err)
{
    extern __shared__ uint32_t hist[];
    const int per_slice = G.Jc + G.Jt * G.q;
    const int slice = blockIdx.x / per_slice;
    const int r = blockIdx.x % per_slice;
    const int T = G.T, E = G.E;
    const bool is_c = r < G.Jc;
    int l, r0, r1, cells, t0, t1;
    long long out;
    if (is_c) {
        l = r / G.nbc;
        const int band = r % G.nbc;
        r0 = G.band_c[band];
        r1 = G.band_c[band + 1];
        cells = (int)(tri_start(r1, E) - tri_start(r0, E));
        out = (long long)l * G.c_layer + (long long)G.S * tri_start(r0, E) + (long long)slice * cells;
        t0 = (int)((long long)T * slice / G.S);
        t1 = (int)((long long)T * (slice + 1) / G.S);
    } else {
        const int rr = r - G.Jc;
        const int grp = rr / G.q;
        const int sub = slice * G.q + rr % G.q;
        const int nsub = G.S * G.q;
        l = grp / G.nbt;
        const int band = grp % G.nbt;
        r0 = band * G.rows_t;
        r1 = min(E, r0 + G.rows_t);
        cells = (r1 - r0) * E;
        out = G.c_total + (long long)l * G.t_layer + (long long)nsub * r0 * E + (long long)sub * cells;
        t0 = (int)((long long)T * sub / nsub);
        t1 = (int)((long long)T * (sub + 1) / nsub);
    }
    const int words = is_c ? cells : (r1 - r0) * G.tstride;
    for (int c = threadIdx.x; c < words; c += blockDim.x) hist[c] = 0u;
    __syncthreads();

    const int32_t *lay = ids + (size_t)l * T * K;
    if (is_c) {
        const int base0 = (int)tri_start(r0, E);
        for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
            int v[K];
            load_ids<K, VEC>(lay + (size_t)t * K, v);
            sort_ids<K>(v);
            int bad = ((unsigned)v[0] >= (unsigned)E || (unsigned)v[K - 1] >= (unsigned)E) ? MOE_DERR_ID_RANGE : 0;
#pragma unroll
            for (int a = 0; a + 1 < K; ++a)
                if (!bad && v[a] == v[a + 1]) bad = MOE_DERR_ID_REPEAT;
            if (bad) {
                record_error(err, bad);
                continue;
            }
#pragma unroll
            for (int a = 0; a < K; ++a) {
                const int i = v[a];
                if (i >= r0 && i < r1) {
                    const int row = (int)tri_start(i, E) - base0 - i;
#pragma unroll
                    for (int b = a; b < K; ++b) atomicAdd(&hist[row + v[b]], 1u);
                }
            }
        }
    } else {
        const int32_t *nxt = lay + (size_t)T * K;
        const bool full_check = G.Jc == 0;   // C blocks report repeats when they run
        const int stride = G.tstride;
        for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
            int a[K], c[K];
            load_ids<K, VEC>(lay + (size_t)t * K, a);
            load_ids<K, VEC>(nxt + (size_t)t * K, c);
            if (full_check) {
                int bad = check_ids<K>(a, E);
                if (!bad) bad = check_ids<K>(c, E);
                if (bad) {
                    record_error(err, bad);
                    continue;
                }
            } else if (!ids_in_range<K>(a, E) || !ids_in_range<K>(c, E)) {
                record_error(err, MOE_DERR_ID_RANGE);
                continue;
            }
#pragma unroll
            for (int x = 0; x < K; ++x) {
                const int i = a[x];
                if (i >= r0 && i < r1) {
                    const int row = (i - r0) * stride;
#pragma unroll
                    for (int y = 0; y < K; ++y) atomicAdd(&hist[row + c[y]], 1u);
                }
            }
        }
    }
    __syncthreads();
    uint32_t *dst = part + out;
    if (is_c) {
        for (int c = threadIdx.x; c < cells; c += blockDim.x) dst[c] = hist[c];
    } else {
        for (int c = threadIdx.x; c < cells; c += blockDim.x) dst[c] = hist[(c / E) * G.tstride + c % E];
    }
}

// Sum of n partial words at base, base + stride, ... (8 loads in flight).
__device__ __forceinline__ uint32_t sum_strided(const uint32_t *__restrict__ part, long long base, long long stride, int n)
{
    uint32_t s = 0;
    int q = 0;
    for (; q + 8 <= n; q += 8) {
        uint32_t v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __ldg(part + base + (long long)(q + i) * stride);
#pragma unroll
        for (int i = 0; i < 8; ++i) s += v[i];
    }
    for (; q < n; ++q) s += __ldg(part + base + (long long)q * stride);
    return s;
}

__device__ __forceinline__ uint32_t c_cell_sum(const StatsGeom &G, const uint32_t *__restrict__ part, int l, int a, int b)
{
    // (a, b) with a <= b: find a's band, then sum the slices
    int band = 0;
    while (a >= G.band_c[band + 1]) ++band;
    const int r0 = G.band_c[band];
    const long long cells = tri_start(G.band_c[band + 1], G.E) - tri_start(r0, G.E);
    const long long base = (long long)l * G.c_layer + (long long)G.S * tri_start(r0, G.E)
                           + (tri_start(a, G.E) - tri_start(r0, G.E)) + (b - a);
    return sum_strided(part, base, cells, G.S);
}

// blockIdx.y selects the matrix: [0, L) C of layer y, [L, 2L-1) M of layer y-L.
// One output cell per thread.
__global__ void __launch_bounds__(kReduceThreads)
stats_reduce_kernel(StatsGeom G, const uint32_t *__restrict__ part, uint32_t *coact, float *ochiai, uint32_t *trans)
{
    extern __shared__ uint32_t diag[];
    const int E = G.E;
    const int m = blockIdx.y;
    const long long EE = (long long)E * E;
    const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (m < G.L) {
        if (!G.Jc) return;
        const int l = m;
        if (ochiai) {
            for (int e = threadIdx.x; e < E; e += blockDim.x) diag[e] = c_cell_sum(G, part, l, e, e);
            __syncthreads();
        }
        if (c < EE) {
            const int i = (int)(c / E), j = (int)(c % E);
            const uint32_t v = c_cell_sum(G, part, l, min(i, j), max(i, j));
            if (coact) coact[(long long)l * EE + c] = v;
            if (ochiai) {
                const double den = __dmul_rn((double)diag[i], (double)diag[j]);
                const double s = den > 0.0 ? __ddiv_rn((double)v, __dsqrt_rn(den)) : 0.0;
                ochiai[(long long)l * EE + c] = __double2float_rn(s);
            }
        }
    } else {
        if (!G.Jt || !trans || c >= EE) return;
        const int l = m - G.L;
        const int i = (int)(c / E), j = (int)(c % E);
        const int band = i / G.rows_t;
        const int r0 = band * G.rows_t;
        const int r1 = min(E, r0 + G.rows_t);
        const long long cells = (long long)(r1 - r0) * E;
        const int nsub = G.S * G.q;
        const long long base = G.c_total + (long long)l * G.t_layer + (long long)nsub * r0 * E
                               + (long long)(i - r0) * E + j;
        trans[(long long)l * EE + c] = sum_strided(part, base, cells, nsub);
    }
}

template <int K>
moe_status launch_hist(const int32_t *ids, const StatsGeom &g, uint32_t *part, int32_t *err, cudaStream_t s)
{
    const size_t smem = (size_t)g.max_words * sizeof(uint32_t);
    const int blocks = (g.Jc + g.Jt * g.q) * g.S;
    const bool vec = (K % 4 == 0) ? aligned16(ids) : ((K % 2 == 0) ? ((reinterpret_cast<uintptr_t>(ids) & 7u) == 0) : false);
    if (vec) {
        if (allow_smem(stats_hist_kernel<K, true>, smem) != cudaSuccess) return MOE_ERR_CUDA;
        stats_hist_kernel<K, true><<<blocks, kHistThreads, smem, s>>>(ids, g, part, err);
    } else {
        if (allow_smem(stats_hist_kernel<K, false>, smem) != cudaSuccess) return MOE_ERR_CUDA;
        stats_hist_kernel<K, false><<<blocks, kHistThreads, smem, s>>>(ids, g, part, err);
    }
    return launch_status();
}

}  // namespace
}  // namespace moe

using namespace moe;

namespace {
// 0: default -- the tensor cores for E >= 128 where the shape allows (on B200
// they measured faster than the histograms at E = 128 and 256 with k = 8),
// the histograms below (at E = 64 the operand tiles, padded to 128 experts,
// cost more than the counter increments); 1: histograms; 2: tensor cores
// where the shape allows
std::atomic<int> g_coact_method{0};

bool tensor_method(int method, int E) { return method == 2 || (method == 0 && E >= 128); }
}  // namespace

extern "C" int moe_coact_stats_method(int method)
{
    if (method < 0 || method > 2) return -1;
    return g_coact_method.exchange(method);
}

extern "C" int moe_coact_stats_path(int L, int T, int k, int E, int with_trans)
{
    if (L < 1 || T < 1 || k < 1 || k > 8 || E < k || E > 1024) return 0;
    const int method = g_coact_method.load();
    MmaGeom mg;
    if (tensor_method(method, E) && make_mma_geom(L, T, k, E, true, with_trans != 0, mg)) return 2;
    return 1;
}

extern "C" size_t moe_coact_stats_workspace(int L, int T, int k, int E, int with_trans)
{
    if (L < 1 || T < 0 || k < 1 || k > 8 || E < k || E > 1024) return 0;
    // the largest of the geometries a call may choose (with or without C, either method)
    long long words = 0;
    StatsGeom g;
    if (make_geom(L, T, k, E, true, with_trans != 0, g)) words = std::max(words, partial_words(g));
    if (with_trans && L > 1 && make_geom(L, T, k, E, false, true, g)) words = std::max(words, partial_words(g));
    MmaGeom mg;
    if (make_mma_geom(L, T, k, E, true, with_trans != 0, mg)) words = std::max(words, (long long)mma_partial_words(mg));
    if (with_trans && L > 1 && make_mma_geom(L, T, k, E, false, true, mg))
        words = std::max(words, (long long)mma_partial_words(mg));
    if (words == 0) return 0;
    return round_up((size_t)words * sizeof(uint32_t), 256) + 256;
}

extern "C" moe_status moe_coact_stats(const int32_t *ids, int L, int T, int k, int E,
                                      uint32_t *coact, float *ochiai, uint32_t *trans,
                                      int32_t *err, void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (L < 1 || T < 0 || k < 1 || k > 8 || E < k || E > 1024) return MOE_ERR_ARG;
    if ((long long)L * T * k >= (1ll << 31)) return MOE_ERR_ARG;
    if (!err || (T > 0 && !ids)) return MOE_ERR_ARG;
    if (L == 1) trans = nullptr;
    const bool want_c = coact || ochiai;
    const bool want_t = trans != nullptr;
    if (!want_c && !want_t) return MOE_OK;
    const size_t EE = (size_t)E * E;
    if (T == 0) {
        if (coact && cudaMemsetAsync(coact, 0, sizeof(uint32_t) * EE * L, stream) != cudaSuccess) return MOE_ERR_CUDA;
        if (ochiai && cudaMemsetAsync(ochiai, 0, sizeof(float) * EE * L, stream) != cudaSuccess) return MOE_ERR_CUDA;
        if (trans && cudaMemsetAsync(trans, 0, sizeof(uint32_t) * EE * (L - 1), stream) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    const int method = g_coact_method.load();
    MmaGeom mg;
    if (tensor_method(method, E) && aligned16(ids) && make_mma_geom(L, T, k, E, want_c, want_t, mg)) {
        const size_t need = mma_partial_words(mg) * sizeof(uint32_t);
        if (!ws || !aligned256(ws) || ws_bytes < need) return MOE_ERR_WORKSPACE;
        return coact_mma(ids, mg, static_cast<uint32_t *>(ws), coact, ochiai, trans, err, stream);
    }
    StatsGeom g;
    if (!make_geom(L, T, k, E, want_c, want_t, g)) return MOE_ERR_UNSUPPORTED;
    const size_t need = (size_t)partial_words(g) * sizeof(uint32_t);
    if (!ws || !aligned256(ws) || ws_bytes < need) return MOE_ERR_WORKSPACE;
    uint32_t *part = static_cast<uint32_t *>(ws);
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_hist<1>(ids, g, part, err, stream); break;
    case 2: st = launch_hist<2>(ids, g, part, err, stream); break;
    case 3: st = launch_hist<3>(ids, g, part, err, stream); break;
    case 4: st = launch_hist<4>(ids, g, part, err, stream); break;
    case 5: st = launch_hist<5>(ids, g, part, err, stream); break;
    case 6: st = launch_hist<6>(ids, g, part, err, stream); break;
    case 7: st = launch_hist<7>(ids, g, part, err, stream); break;
    case 8: st = launch_hist<8>(ids, g, part, err, stream); break;
    }
    if (st != MOE_OK) return st;
    note_launches(1);
    const int mats = L + (want_t ? L - 1 : 0);
    const int bx = (int)(((long long)EE + kReduceThreads - 1) / kReduceThreads);
    dim3 grid(bx, mats);
    const size_t smem = (size_t)E * sizeof(uint32_t);
    stats_reduce_kernel<<<grid, kReduceThreads, smem, stream>>>(g, part, coact, ochiai, trans);
    st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

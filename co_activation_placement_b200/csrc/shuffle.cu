// Token shuffling targets.
//
// "Expert Coupling in MoE Pretraining", abstract: under sequence parallelism
// each token moves, during the reduce-scatter after attention, to the GPU
// predicted to hold its next-layer experts.  The prediction used here: a token
// that picks e at layer l picks an expert on rank r at layer l+1 as often as
// the transition counts M_l say,
//   rank_score[e][r] = sum_{e' : p_{l+1}(e') = r} M_l[e][e'],
//   target_t = argmax_r sum_j rank_score[e_tj][r]   (lowest r on ties).
//
// moe_rank_score: one block per expert row e, a shared uint64 accumulator per
// rank (integer atomics: order-free).  moe_shuffle_targets: the E x G table
// sits in shared memory (one block per SM, so it is copied once per SM), with
// one extra row of zeros that the picks of an invalid token point to; a warp
// stages the picks of 32 tokens in shared memory and then scores them one at a
// time, every lane reading the token's picks with broadcast loads.  The argmax
// on (score desc, rank asc) is a maximum of the packed key
// (score << 6) | (63 - rank).  When G is even and k times the largest table
// entry stays below 2^26 (checked once per block while copying), lane l owns
// ranks 2l and 2l+1, reads both with one 8-byte load per pick, sums in 32 bits
// and takes the maximum with one redux.sync: 57 warp instructions per token
// against 170 for the general path (ncu counts on 131072 tokens, G = 64).
// Otherwise lane l owns ranks l and l+32 with uint64 sums, and the maximum is
// one redux.sync when the warp's sums fit 26 bits, five 64-bit shuffles if not.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kShuffleThreads = 512;

__global__ void __launch_bounds__(kThreads)
rank_score_kernel(const uint32_t *__restrict__ trans, const int32_t *__restrict__ e2r, int E, int G,
                  uint32_t *__restrict__ rs, int32_t *err)
{
    __shared__ unsigned long long acc[64];
    const int e = blockIdx.x;
    if (threadIdx.x < G) acc[threadIdx.x] = 0;
    __syncthreads();
    for (int f = threadIdx.x; f < E; f += kThreads) {
        const int r = __ldg(e2r + f);
        if ((unsigned)r >= (unsigned)G) {
            record_error(err, MOE_DERR_RANK_RANGE);
            continue;
        }
        const uint32_t v = __ldg(trans + (size_t)e * E + f);
        if (v) atomicAdd(&acc[r], (unsigned long long)v);
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const unsigned long long v = acc[threadIdx.x];
        rs[(size_t)e * G + threadIdx.x] = v > 0xffffffffull ? 0xffffffffu : (uint32_t)v;
    }
}

template <int K>
__global__ void __launch_bounds__(kShuffleThreads)
shuffle_targets_kernel(const int32_t *__restrict__ ids, int T, int E, int G, const uint32_t *__restrict__ rs_g,
                       int32_t *__restrict__ target, int32_t *err)
{
    extern __shared__ __align__(16) uint32_t tab[];   // [E+1][G] (row E zeros), then each warp's picks
    __shared__ uint32_t tab_max;
    int *picks_all = reinterpret_cast<int *>(tab + (((E + 1) * G + 3) & ~3));
    if (threadIdx.x == 0) tab_max = 0;
    for (int i = threadIdx.x; i < G; i += kShuffleThreads) tab[E * G + i] = 0u;
    __syncthreads();
    {   // copy the table: 16-byte vectors where the layout allows, 8 in flight per thread
        const int n = E * G;
        const bool vec = (n % 4 == 0) && ((reinterpret_cast<uintptr_t>(rs_g) & 15u) == 0);
        uint32_t mx = 0;
        if (vec) {
            const uint4 *src = reinterpret_cast<const uint4 *>(rs_g);
            uint4 *dst = reinterpret_cast<uint4 *>(tab);
            for (int i0 = threadIdx.x; i0 < n / 4; i0 += 8 * kShuffleThreads) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (i0 + u * kShuffleThreads < n / 4) v[u] = __ldg(src + i0 + u * kShuffleThreads);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (i0 + u * kShuffleThreads < n / 4) {
                        dst[i0 + u * kShuffleThreads] = v[u];
                        mx = max(max(mx, max(v[u].x, v[u].y)), max(v[u].z, v[u].w));
                    }
            }
        } else {
            for (int i = threadIdx.x; i < n; i += kShuffleThreads) {
                const uint32_t v = __ldg(rs_g + i);
                tab[i] = v;
                mx = max(mx, v);
            }
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if ((threadIdx.x & 31) == 0) atomicMax(&tab_max, mx);
    }
    __syncthreads();
    // sums of K entries fit 26 bits: 32-bit sums and one redux per token
    const bool narrow = (G % 2 == 0) && (unsigned long long)tab_max * K < (1ull << 26);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int KP = (K + 3) & ~3;                  // picks per token in shared memory, padded to int4
    int *picks = picks_all + warp * 32 * KP;
    const int nwarps = gridDim.x * (kShuffleThreads / 32);
    const int gw = blockIdx.x * (kShuffleThreads / 32) + warp;
    // a warp takes 32 tokens at a time: lane l loads token t0+l's picks into
    // shared memory, then the warp scores the 32 tokens one after another,
    // every lane reading the token's picks with broadcast loads
    for (int t0 = gw * 32; t0 < T; t0 += nwarps * 32) {
        const int tl = t0 + lane;
        bool ok = tl < T;
        {
            int e[KP];
#pragma unroll
            for (int j = 0; j < KP; ++j) {
                e[j] = (j < K && tl < T) ? __ldg(ids + (size_t)tl * K + j) : 0;
                if (j < K && (unsigned)e[j] >= (unsigned)E) { ok = false; }
            }
            if (tl < T && !ok) record_error(err, MOE_DERR_ID_RANGE);
            // an invalid token (or a padding pick) points to the zero row: score 0 everywhere, rank 0
#pragma unroll
            for (int j = 0; j < KP; ++j) picks[lane * KP + j] = (ok && j < K) ? e[j] : E;
        }
        __syncwarp();
        const int n = min(32, T - t0);
        int result = 0;
        if (narrow) {
            const bool mine = 2 * lane < G;
            const uint32_t k0 = (uint32_t)(63 - 2 * lane), k1 = (uint32_t)(62 - 2 * lane);
            for (int i = 0; i < n; ++i) {
                int e[KP];
#pragma unroll
                for (int q = 0; q < KP / 4; ++q) {
                    const int4 v = reinterpret_cast<const int4 *>(picks + i * KP)[q];
                    e[4 * q] = v.x; e[4 * q + 1] = v.y; e[4 * q + 2] = v.z; e[4 * q + 3] = v.w;
                }
                uint32_t s0 = 0, s1 = 0;
                if (mine) {
#pragma unroll
                    for (int j = 0; j < K; ++j) {
                        const uint2 v = reinterpret_cast<const uint2 *>(tab + (size_t)e[j] * G)[lane];
                        s0 += v.x;
                        s1 += v.y;
                    }
                }
                const uint32_t key = mine ? max((s0 << 6) | k0, (s1 << 6) | k1) : 0u;
                const int bi = 63 - (int)(__reduce_max_sync(0xffffffffu, key) & 63u);
                if (lane == i) result = bi;
            }
            if (tl < T) target[tl] = result;
            __syncwarp();
            continue;
        }
        for (int i = 0; i < n; ++i) {
            int e[KP];
#pragma unroll
            for (int q = 0; q < KP / 4; ++q) {
                const int4 v = reinterpret_cast<const int4 *>(picks + i * KP)[q];
                e[4 * q] = v.x; e[4 * q + 1] = v.y; e[4 * q + 2] = v.z; e[4 * q + 3] = v.w;
            }
            unsigned long long a0 = 0, a1 = 0;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const uint32_t *row = tab + (size_t)e[j] * G;
                if (lane < G) a0 += row[lane];
                if (lane + 32 < G) a1 += row[lane + 32];
            }
            // packed key (score << 6) | (63 - rank): the maximum is the best
            // rank, the lowest rank among equal scores
            int bi;
            if (__all_sync(0xffffffffu, (a0 | a1) < (1ull << 26))) {
                uint32_t key = lane < G ? (((uint32_t)a0 << 6) | (uint32_t)(63 - lane)) : 0u;
                if (lane + 32 < G) key = max(key, ((uint32_t)a1 << 6) | (uint32_t)(31 - lane));
                key = __reduce_max_sync(0xffffffffu, key);
                bi = 63 - (int)(key & 63u);
            } else {
                unsigned long long best = lane < G ? (a0 << 6) | (unsigned long long)(63 - lane) : 0ull;
                if (lane + 32 < G) best = max(best, (a1 << 6) | (unsigned long long)(31 - lane));
#pragma unroll
                for (int o = 16; o; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
                bi = 63 - (int)(best & 63u);
            }
            if (lane == i) result = bi;
        }
        if (tl < T) target[tl] = result;
        __syncwarp();
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_rank_score(const uint32_t *trans_l, const int32_t *next_expert_to_rank,
                                     int E, int G, uint32_t *rank_score, int32_t *err, cudaStream_t stream)
{
    if (E < 1 || G < 1 || G > 64 || !trans_l || !next_expert_to_rank || !rank_score || !err) return MOE_ERR_ARG;
    rank_score_kernel<<<E, kThreads, 0, stream>>>(trans_l, next_expert_to_rank, E, G, rank_score, err);
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

template <int K>
static moe_status launch_shuffle(const int32_t *ids, int T, int E, int G, const uint32_t *rs, int32_t *target,
                                 int32_t *err, cudaStream_t s)
{
    constexpr int KP = (K + 3) & ~3;
    const size_t smem = sizeof(uint32_t) * (size_t)(((E + 1) * G + 3) & ~3) + sizeof(int) * (kShuffleThreads / 32) * 32 * KP;
    if (allow_smem(shuffle_targets_kernel<K>, smem) != cudaSuccess) return MOE_ERR_CUDA;
    // one block per SM at most: every block first copies the whole table
    const long long need = ((long long)T + kShuffleThreads - 1) / kShuffleThreads;
    const int grid = (int)std::max<long long>(1, std::min<long long>(need, (long long)sm_count()));
    shuffle_targets_kernel<K><<<grid, kShuffleThreads, smem, s>>>(ids, T, E, G, rs, target, err);
    return launch_status();
}

extern "C" moe_status moe_shuffle_targets(const int32_t *ids, int T, int k, int E, int G,
                                          const uint32_t *rank_score, int32_t *target,
                                          int32_t *err, cudaStream_t stream)
{
    if (T < 0 || k < 1 || k > 8 || E < k || G < 1 || G > 64 || !err) return MOE_ERR_ARG;
    if ((long long)E * G > 16384) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!ids || !rank_score || !target) return MOE_ERR_ARG;
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_shuffle<1>(ids, T, E, G, rank_score, target, err, stream); break;
    case 2: st = launch_shuffle<2>(ids, T, E, G, rank_score, target, err, stream); break;
    case 3: st = launch_shuffle<3>(ids, T, E, G, rank_score, target, err, stream); break;
    case 4: st = launch_shuffle<4>(ids, T, E, G, rank_score, target, err, stream); break;
    case 5: st = launch_shuffle<5>(ids, T, E, G, rank_score, target, err, stream); break;
    case 6: st = launch_shuffle<6>(ids, T, E, G, rank_score, target, err, stream); break;
    case 7: st = launch_shuffle<7>(ids, T, E, G, rank_score, target, err, stream); break;
    case 8: st = launch_shuffle<8>(ids, T, E, G, rank_score, target, err, stream); break;
    }
    if (st == MOE_OK) note_launches(1);
    return st;
}

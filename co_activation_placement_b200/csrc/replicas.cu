// Communication-aware task assignment over expert replicas.
//
// "Cobalt", "Problem Formulation": a task (t, e) runs on a rank r_t^e holding
// a replica of e, and the cross-node cost V counts, per token, the distinct
// nodes other than the source's that its tasks reach; the communication-aware
// assignment "routes tokens to the fewest remote nodes possible".
//
// Exact per token: with at most 8 nodes, the smallest set S of remote nodes
// covering the token's experts (those without a replica on the source node) is
// found by enumerating the submasks of the candidate nodes (ties: smallest S
// as a bit pattern).  Then, pick by pick in j order, among the ranks hosting
// the expert on the source node (or, if none, on the nodes of S): rank s if
// it is one of them, else the lowest one an earlier pick already uses (no new
// row), else the lowest one.
// One thread per token; the replica table sits in shared memory.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxNodes = 8;

template <int K>
__global__ void __launch_bounds__(kThreads)
assign_replicas_kernel(const int32_t *__restrict__ ids, int T, int E, int G, int rpn,
                       const int32_t *__restrict__ replica_rank, const int32_t *__restrict__ n_rep,
                       const int32_t *__restrict__ src_rank, int32_t *__restrict__ pick_rank,
                       int32_t *__restrict__ n_remote, int32_t *err)
{
    extern __shared__ int32_t sm[];
    const int nodes = G / rpn, max_rep = 1 + nodes;
    int32_t *rep = sm;                          // [E][max_rep]
    uint32_t *nmask = reinterpret_cast<uint32_t *>(sm + E * max_rep);   // [E] nodes hosting e
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        uint32_t m = 0;
        const int n = min(max(__ldg(n_rep + e), 0), max_rep);
        for (int q = 0; q < max_rep; ++q) {
            int r = q < n ? __ldg(replica_rank + (size_t)e * max_rep + q) : -1;
            if (q < n && (unsigned)r >= (unsigned)G) {
                record_error(err, MOE_DERR_RANK_RANGE);
                r = -1;
            }
            rep[e * max_rep + q] = r;
            if (r >= 0) m |= 1u << (r / rpn);
        }
        nmask[e] = m;
    }
    __syncthreads();
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
        int v[K];
#pragma unroll
        for (int j = 0; j < K; ++j) v[j] = __ldg(ids + (size_t)t * K + j);
        bool bad = false;
#pragma unroll
        for (int a = 0; a < K; ++a) {
            bad |= (unsigned)v[a] >= (unsigned)E;
#pragma unroll
            for (int b = 0; b < a; ++b) bad |= v[a] == v[b];
        }
        int s = src_rank ? __ldg(src_rank + t) : t / (T / G);
        if ((unsigned)s >= (unsigned)G) bad = true;
        uint32_t need = 0;   // picks whose expert has no replica on the source node
        uint32_t cand = 0;   // remote nodes hosting one of those experts
        const int ns = bad ? 0 : s / rpn;
        uint32_t nm[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            nm[j] = bad ? 0u : nmask[v[j]];
            if (!((nm[j] >> ns) & 1u)) {
                need |= 1u << j;
                cand |= nm[j];
            }
        }
        cand &= ~(1u << ns);
        int best_pop = 99;
        uint32_t best = 0;
        if (!bad) {
            for (uint32_t sub = cand;; sub = (sub - 1) & cand) {
                bool ok = true;
#pragma unroll
                for (int j = 0; j < K; ++j)
                    if ((need >> j) & 1u) ok &= (nm[j] & sub) != 0;
                const int pop = __popc(sub);
                if (ok && (pop < best_pop || (pop == best_pop && sub < best))) {
                    best_pop = pop;
                    best = sub;
                }
                if (sub == 0) break;
            }
            if (best_pop == 99) bad = true;    // an expert with no replica at all
        }
        if (bad) {
            record_error(err, MOE_DERR_ID_RANGE);
#pragma unroll
            for (int j = 0; j < K; ++j) pick_rank[(size_t)t * K + j] = -1;
            if (n_remote) n_remote[t] = -1;
            continue;
        }
        unsigned long long used = 0;   // ranks already serving an earlier pick
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const int32_t *rl = rep + v[j] * max_rep;
            const bool any_ns = (nm[j] >> ns) & 1u;
            int pick = -1, used_pick = -1, low = -1;
            for (int q = 0; q < max_rep; ++q) {
                const int r = rl[q];
                if (r < 0) continue;
                const bool allowed = any_ns ? (r / rpn == ns) : ((best >> (r / rpn)) & 1u);
                if (!allowed) continue;
                if (r == s) pick = r;
                if (((used >> r) & 1ull) && (used_pick < 0 || r < used_pick)) used_pick = r;
                if (low < 0 || r < low) low = r;
            }
            if (pick < 0) pick = used_pick >= 0 ? used_pick : low;
            used |= 1ull << pick;
            pick_rank[(size_t)t * K + j] = pick;
        }
        if (n_remote) n_remote[t] = best_pop;
    }
}

template <int K>
moe_status launch_assign(const int32_t *ids, int T, int E, int G, int rpn, const int32_t *rr, const int32_t *nr,
                         const int32_t *src, int32_t *pick, int32_t *nrem, int32_t *err, cudaStream_t s)
{
    const int max_rep = 1 + G / rpn;
    const size_t smem = sizeof(int32_t) * (size_t)E * (max_rep + 1);
    if (allow_smem(assign_replicas_kernel<K>, smem) != cudaSuccess) return MOE_ERR_CUDA;
    const int grid = (int)std::max<long long>(1, std::min<long long>((T + kThreads - 1) / kThreads, sm_count() * 4LL));
    assign_replicas_kernel<K><<<grid, kThreads, smem, s>>>(ids, T, E, G, rpn, rr, nr, src, pick, nrem, err);
    return launch_status();
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_assign_replicas(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                          const int32_t *replica_rank, const int32_t *n_rep,
                                          const int32_t *src_rank, int32_t *pick_rank, int32_t *n_remote,
                                          int32_t *err, cudaStream_t stream)
{
    if (T < 0 || k < 1 || k > 8 || E < k || G < 1 || G > 64 || rpn < 1 || G % rpn != 0 || !err) return MOE_ERR_ARG;
    if (G / rpn > kMaxNodes) return MOE_ERR_UNSUPPORTED;
    if ((size_t)E * (G / rpn + 2) * sizeof(int32_t) > 200 * 1024) return MOE_ERR_UNSUPPORTED;
    if (!src_rank && T % G != 0) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!ids || !replica_rank || !n_rep || !pick_rank) return MOE_ERR_ARG;
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_assign<1>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 2: st = launch_assign<2>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 3: st = launch_assign<3>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 4: st = launch_assign<4>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 5: st = launch_assign<5>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 6: st = launch_assign<6>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 7: st = launch_assign<7>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    case 8: st = launch_assign<8>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err, stream); break;
    }
    if (st == MOE_OK) note_launches(1);
    return st;
}

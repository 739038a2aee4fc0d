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
//
// Under a load tolerance ("Cobalt", "Problem Formulation": the tasks of rank
// r, sum_e w_r^e, at most (1 + eps) K T / G) the assignment is the greedy in
// token order: before token t a rank whose task count has reached
// cap = floor((1 + eps) T k / G) is closed, and t is assigned as above over
// its experts' open replicas (all of them when none is open).  Token t's
// choice depends on every earlier token only through the set of closed
// ranks, which changes at most G times, so one cooperative launch computes
// it in rounds: every remaining token's choice under the current closed set,
// in parallel; per-block task counts per rank and their running sum over
// blocks locate the first token tau at which an open rank reaches the cap
// (a block-wide scan inside the block where that happens); the choices of
// tokens before tau are final, their tasks join the loads, the ranks at the
// cap close, and the next round starts at tau.  At most G + 1 rounds, each
// ending in a grid barrier with a bounded wait.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "waits.cuh"

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

// ---- load-capped assignment ---------------------------------------------

constexpr int kCapThreads = 512;
constexpr int kCapMaxBlocks = 1024;

struct CapHeader {
    GridBarrier bar;
    int tau[2];           // first token seeing a newly closed rank (by round parity)
    int rounds;           // rounds run
    int pad;
};

struct CapArgs {
    const int32_t *ids;
    int T, E, G, rpn;
    const int32_t *rr, *nr, *src;
    long long cap;
    int32_t *pick, *nrem;
    long long *rank_load;     // [G] out or null
    CapHeader *h;
    unsigned long long *load; // [G] tasks committed per rank
    int *blk;                 // [gridDim.x][G] tasks per rank of each block's tokens this round
    int32_t *err;
};

// Token t's choice over the usable replicas (uok[e]: usable ranks of e,
// unm[e]: their nodes): the fewest remote nodes, then the pick rule.
// Returns |S| or -1 for an invalid token (ids, source, an expert without
// replicas); the picks are written to pk.
template <int K>
__device__ __forceinline__ int choose_capped(const int (&v)[K], int s, int E, int G, int rpn, int max_rep,
                                             const int32_t *rep, const uint32_t *unm,
                                             const unsigned long long *uok, int (&pk)[K])
{
    bool bad = (unsigned)s >= (unsigned)G;
#pragma unroll
    for (int a = 0; a < K; ++a) {
        bad |= (unsigned)v[a] >= (unsigned)E;
#pragma unroll
        for (int b = 0; b < a; ++b) bad |= v[a] == v[b];
    }
    if (bad) return -1;
    const int ns = s / rpn;
    uint32_t need = 0, cand = 0, nm[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
        nm[j] = unm[v[j]];
        if (!((nm[j] >> ns) & 1u)) {
            need |= 1u << j;
            cand |= nm[j];
        }
    }
    cand &= ~(1u << ns);
    int best_pop = 99;
    uint32_t best = 0;
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
    if (best_pop == 99) return -1;
    unsigned long long used = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        const int32_t *rl = rep + v[j] * max_rep;
        const unsigned long long ok = uok[v[j]];
        const bool any_ns = (nm[j] >> ns) & 1u;
        int pick = -1, used_pick = -1, low = -1;
        for (int q = 0; q < max_rep; ++q) {
            const int r = rl[q];
            if (r < 0 || !((ok >> r) & 1ull)) continue;
            const bool allowed = any_ns ? (r / rpn == ns) : ((best >> (r / rpn)) & 1u);
            if (!allowed) continue;
            if (r == s) pick = r;
            if (((used >> r) & 1ull) && (used_pick < 0 || r < used_pick)) used_pick = r;
            if (low < 0 || r < low) low = r;
        }
        if (pick < 0) pick = used_pick >= 0 ? used_pick : low;
        used |= 1ull << pick;
        pk[j] = pick;
    }
    return best_pop;
}

// Inclusive block-wide sum scan of one value per thread (kCapThreads).
__device__ __forceinline__ int block_scan_incl(int x, int *warp_tot)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
        int t = lane < kCapThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kCapThreads / 32) warp_tot[lane] = t;
    }
    __syncthreads();
    const int before = w > 0 ? warp_tot[w - 1] : 0;
    __syncthreads();
    return x + before;
}

template <int K>
__global__ void __launch_bounds__(kCapThreads)
assign_capped_kernel(CapArgs a)
{
    extern __shared__ __align__(16) unsigned char csm[];
    const int E = a.E, G = a.G, rpn = a.rpn, T = a.T;
    const int nodes = G / rpn, max_rep = 1 + nodes;
    const int nb = gridDim.x, b = blockIdx.x, tid = threadIdx.x;
    unsigned long long *uok = reinterpret_cast<unsigned long long *>(csm);             // [E]
    unsigned long long *base = uok + E;                                                   // [G]
    int32_t *rep = reinterpret_cast<int32_t *>(base + G);                                 // [E][max_rep]
    uint32_t *unm = reinterpret_cast<uint32_t *>(rep + E * max_rep);                      // [E]
    int *hist = reinterpret_cast<int *>(unm + E);                                         // [G]
    __shared__ int warp_tot[32];
    __shared__ unsigned long long closed_s;
    __shared__ int tau_s, cross_s, tile_tot_s;

    for (int e = tid; e < E; e += blockDim.x) {
        const int n = min(max(__ldg(a.nr + e), 0), max_rep);
        for (int q = 0; q < max_rep; ++q) {
            int r = q < n ? __ldg(a.rr + (size_t)e * max_rep + q) : -1;
            if (q < n && (unsigned)r >= (unsigned)G) {
                if (b == 0) record_error(a.err, MOE_DERR_RANK_RANGE);
                r = -1;
            }
            rep[e * max_rep + q] = r;
        }
    }
    if (b == 0 && tid == 0) {
        a.h->tau[0] = T;
        a.h->tau[1] = T;
    }
    if (!grid_barrier(&a.h->bar, a.err)) return;

    int tc = 0;
    for (int rd = 0; rd <= G + 1; ++rd) {
        // (a) the closed ranks and each expert's usable replicas
        if (tid == 0) {
            unsigned long long c = 0;
            for (int r = 0; r < G; ++r)
                if ((long long)__ldcg(a.load + r) >= a.cap) c |= 1ull << r;
            closed_s = c;
        }
        for (int r = tid; r < G; r += blockDim.x) hist[r] = 0;
        __syncthreads();
        const unsigned long long closed = closed_s;
        for (int e = tid; e < E; e += blockDim.x) {
            unsigned long long all = 0, open = 0;
            for (int q = 0; q < max_rep; ++q) {
                const int r = rep[e * max_rep + q];
                if (r < 0) continue;
                all |= 1ull << r;
                if (!((closed >> r) & 1ull)) open |= 1ull << r;
            }
            const unsigned long long u = open ? open : all;
            uint32_t m = 0;
            for (int q = 0; q < max_rep; ++q) {
                const int r = rep[e * max_rep + q];
                if (r >= 0 && ((u >> r) & 1ull)) m |= 1u << (r / rpn);
            }
            uok[e] = u;
            unm[e] = m;
        }
        __syncthreads();
        // (b) every remaining token's choice; this block's tokens [lo, hi)
        const int lo = tc + (int)((long long)(T - tc) * b / nb);
        const int hi = tc + (int)((long long)(T - tc) * (b + 1) / nb);
        for (int t = lo + tid; t < hi; t += blockDim.x) {
            int v[K], pk[K];
#pragma unroll
            for (int j = 0; j < K; ++j) v[j] = __ldg(a.ids + (size_t)t * K + j);
            const int s = a.src ? __ldg(a.src + t) : t / (T / G);
            const int n = choose_capped<K>(v, s, E, G, rpn, max_rep, rep, unm, uok, pk);
            if (n < 0) {
                if (rd == 0) record_error(a.err, MOE_DERR_ID_RANGE);
#pragma unroll
                for (int j = 0; j < K; ++j) a.pick[(size_t)t * K + j] = -1;
                if (a.nrem) a.nrem[t] = -1;
                continue;
            }
#pragma unroll
            for (int j = 0; j < K; ++j) {
                a.pick[(size_t)t * K + j] = pk[j];
                atomicAdd(&hist[pk[j]], 1);
            }
            if (a.nrem) a.nrem[t] = n;
        }
        __syncthreads();
        for (int r = tid; r < G; r += blockDim.x) a.blk[(size_t)b * G + r] = hist[r];
        if (b == 0 && tid == 0) a.h->tau[(rd + 1) & 1] = T;
        if (!grid_barrier(&a.h->bar, a.err)) return;
        // (c) the loads at this block's first token; a rank that reaches the
        // cap inside the block's tokens gives the first token that sees it
        // closed
        for (int r = tid; r < G; r += blockDim.x) {
            unsigned long long x = __ldcg(a.load + r);
            for (int q = 0; q < b; ++q) x += (unsigned)__ldcg(a.blk + (size_t)q * G + r);
            base[r] = x;
        }
        __syncthreads();
        for (int r = 0; r < G; ++r) {
            if ((closed >> r) & 1ull) continue;
            const long long b0 = (long long)base[r];
            if (b0 >= a.cap || b0 + hist[r] < a.cap) continue;
            // the crossing lies in [lo, hi): scan the block's tokens in order
            const long long need = a.cap - b0;          // tasks on r that reach the cap
            long long run = 0;
            if (tid == 0) cross_s = -1;
            __syncthreads();
            for (int t0 = lo; t0 < hi; t0 += blockDim.x) {
                const int t = t0 + tid;
                int c = 0;
                if (t < hi) {
#pragma unroll
                    for (int j = 0; j < K; ++j) c += __ldcg(a.pick + (size_t)t * K + j) == r;
                }
                const int incl = block_scan_incl(c, warp_tot);
                // the one token whose tasks on r take the running count to need
                if (t < hi && run + incl >= need && run + incl - c < need) cross_s = t;
                if (tid == (int)blockDim.x - 1) tile_tot_s = incl;
                __syncthreads();
                const bool found = cross_s >= 0;
                run += tile_tot_s;
                __syncthreads();
                if (found) break;
            }
            if (tid == 0 && cross_s >= 0) atomicMin(&a.h->tau[rd & 1], cross_s + 1);
            __syncthreads();
        }
        if (!grid_barrier(&a.h->bar, a.err)) return;
        // (d) commit the tokens before tau
        if (tid == 0) tau_s = __ldcg(&a.h->tau[rd & 1]);
        __syncthreads();
        const int tau = tau_s;
        if (hi <= tau) {
            for (int r = tid; r < G; r += blockDim.x)
                if (hist[r]) atomicAdd(a.load + r, (unsigned long long)hist[r]);
        } else if (lo < tau) {
            __syncthreads();
            for (int r = tid; r < G; r += blockDim.x) hist[r] = 0;
            __syncthreads();
            for (int t = lo + tid; t < tau; t += blockDim.x)
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int r = __ldcg(a.pick + (size_t)t * K + j);
                    if (r >= 0) atomicAdd(&hist[r], 1);
                }
            __syncthreads();
            for (int r = tid; r < G; r += blockDim.x)
                if (hist[r]) atomicAdd(a.load + r, (unsigned long long)hist[r]);
        }
        if (!grid_barrier(&a.h->bar, a.err)) return;
        tc = tau;
        if (tc >= T) {
            if (b == 0 && tid == 0) a.h->rounds = rd + 1;
            break;
        }
        if (rd == G + 1) record_error(a.err, MOE_DERR_TIMEOUT);   // more rounds than ranks: not reachable
    }
    if (b == 0 && a.rank_load)
        for (int r = tid; r < G; r += blockDim.x) a.rank_load[r] = (long long)__ldcg(a.load + r);
}

template <int K>
moe_status launch_capped(CapArgs args, cudaStream_t s)
{
    auto kern = assign_capped_kernel<K>;
    const int max_rep = 1 + args.G / args.rpn;
    const size_t smem = sizeof(unsigned long long) * ((size_t)args.E + args.G) +
                        sizeof(int32_t) * ((size_t)args.E * max_rep + args.E + args.G);
    if (allow_smem(kern, smem) != cudaSuccess) return MOE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCapThreads, smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (per_sm < 1) return MOE_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)std::min(sm_count(), kCapMaxBlocks));   // one block per SM: co-resident
    cfg.blockDim = dim3(kCapThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args) != cudaSuccess) return MOE_ERR_CUDA;
    return launch_status();
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

extern "C" size_t moe_assign_replicas_capped_workspace(int G)
{
    if (G < 1 || G > 64) return 0;
    return 256 + 512 + round_up(sizeof(int) * (size_t)kCapMaxBlocks * G, 256);
}

extern "C" moe_status moe_assign_replicas_capped(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                                 const int32_t *replica_rank, const int32_t *n_rep,
                                                 const int32_t *src_rank, double eps, int32_t *pick_rank,
                                                 int32_t *n_remote, long long *rank_load, int32_t *err,
                                                 void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (T < 0 || k < 1 || k > 8 || E < k || G < 1 || G > 64 || rpn < 1 || G % rpn != 0 || !err) return MOE_ERR_ARG;
    if (!(eps >= 0.0)) return MOE_ERR_ARG;
    if (G / rpn > kMaxNodes) return MOE_ERR_UNSUPPORTED;
    if ((size_t)E * (G / rpn + 2) * sizeof(int32_t) + (size_t)(E + G) * 8 > 200 * 1024) return MOE_ERR_UNSUPPORTED;
    if (!src_rank && T % G != 0) return MOE_ERR_ARG;
    if (T == 0) {
        if (rank_load && cudaMemsetAsync(rank_load, 0, sizeof(long long) * G, stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!ids || !replica_rank || !n_rep || !pick_rank || !ws) return MOE_ERR_ARG;
    if (!aligned256(ws) || ws_bytes < moe_assign_replicas_capped_workspace(G)) return MOE_ERR_WORKSPACE;
    // the per-rank task cap, floor((1 + eps) T k / G) in fp64; none for eps = inf
    const double c = std::floor((1.0 + eps) * (double)((long long)T * k) / (double)G);
    char *w = static_cast<char *>(ws);
    CapArgs a{};
    a.ids = ids;
    a.T = T; a.E = E; a.G = G; a.rpn = rpn;
    a.rr = replica_rank; a.nr = n_rep; a.src = src_rank;
    a.cap = c >= 9.0e18 ? (long long)INT64_MAX : (long long)c;
    a.pick = pick_rank; a.nrem = n_remote; a.rank_load = rank_load;
    a.h = reinterpret_cast<CapHeader *>(w);
    a.load = reinterpret_cast<unsigned long long *>(w + 256);
    a.blk = reinterpret_cast<int *>(w + 256 + 512);
    a.err = err;
    if (cudaMemsetAsync(w, 0, 256 + 512, stream) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_capped<1>(a, stream); break;
    case 2: st = launch_capped<2>(a, stream); break;
    case 3: st = launch_capped<3>(a, stream); break;
    case 4: st = launch_capped<4>(a, stream); break;
    case 5: st = launch_capped<5>(a, stream); break;
    case 6: st = launch_capped<6>(a, stream); break;
    case 7: st = launch_capped<7>(a, stream); break;
    case 8: st = launch_capped<8>(a, stream); break;
    }
    if (st == MOE_OK) note_launches(1);
    return st;
}

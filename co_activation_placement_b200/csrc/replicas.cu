// Communication-aware task assignment over expert replicas.
//
// "Cobalt", "Problem Formulation": a task (t, e) runs on a rank r_t^e holding
// a replica of e, and the cross-node cost V counts, per token, the distinct
// nodes other than the source's that its tasks reach; the communication-aware
// assignment sends each token to as few remote nodes as it can.
//
// Exact per token: with at most 8 nodes, the smallest set S of remote nodes
// covering the token's experts (those without a replica on the source node) is
// found by trying the sets of candidate nodes by size, each size in
// increasing order (ties: smallest S as a bit pattern).  Then, pick by pick in
// j order, among the ranks hosting the expert on the source node (or, if
// none, on the nodes of S): rank s if it is one of them, else the lowest one
// an earlier pick already uses (no new row), else the lowest one.
// One thread per token; the replica table sits in shared memory.
//
// Under a load tolerance ("Cobalt", "Problem Formulation": the tasks of rank
// r, sum_e w_r^e, at most (1 + eps) K T / G) the assignment is the greedy in
// token order: before token t a rank whose task count has reached
// cap = floor((1 + eps) T k / G) is closed, and t is assigned as above over
// its experts' open replicas (all of them when none is open).  Token t's
// choice depends on every earlier token only through the set of closed
// ranks, which changes at most G times, so one cooperative launch computes
// it in rounds: the remaining tokens' choices under the current closed set,
// in parallel, one warp per token (after the first round only the tokens
// with a pick on a rank that just closed); per-block task counts per rank and their
// running sum over blocks locate the first token tau at which an open rank
// reaches the cap (a block-wide scan inside the block where that happens);
// the choices of tokens before tau are final, their tasks join the loads,
// the ranks at the cap close, and the next round starts at tau.  Every
// block finds tau and commits by itself from all blocks' counts, so a round
// takes one grid barrier (bounded wait); at most G + 1 rounds.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "waits.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxNodes = 8;

// The fewest remote nodes covering the needed picks: the smallest set S of
// the candidate nodes `cand` such that every pick j in `need` has a node of
// nm[j] in S; among sets of that size the smallest as a bit pattern.  A pick
// with one candidate node forces that node into every cover (F); the picks F
// leaves uncovered are covered by the fewest of their own candidate nodes,
// tried by size and within a size in increasing order (Gosper's successor on
// the candidates' positions, deposited back onto them), so the first cover
// found is the answer and S = F | that cover (F's bits are common to every
// minimum S, so the order of the covers is that of the S).  With one or two
// replicas per expert nearly every pick is forced and little is left to try.
// Returns |S| (best = S), or -1 when a needed pick has no candidate node.
template <int K>
__device__ __forceinline__ int fewest_nodes(uint32_t need, const uint32_t (&nm)[K], uint32_t cand, uint32_t &best)
{
    best = 0;
    if (need == 0) return 0;
    uint32_t forced = 0;
#pragma unroll
    for (int j = 0; j < K; ++j)
        if ((need >> j) & 1u) {
            const uint32_t c = nm[j] & cand;
            if (c == 0) return -1;
            if ((c & (c - 1u)) == 0) forced |= c;
        }
    uint32_t rest = 0, rc = 0, all = ~0u;
#pragma unroll
    for (int j = 0; j < K; ++j)
        if (((need >> j) & 1u) && (nm[j] & forced) == 0) {
            rest |= 1u << j;
            rc |= nm[j] & cand;
            all &= nm[j];
        }
    const int nf = __popc(forced);
    if (rest == 0) {
        best = forced;
        return nf;
    }
    all &= rc;
    if (all) {                                   // one node covers the rest: the lowest such
        best = forced | (all & (0u - all));
        return nf + 1;
    }
    const int m = __popc(rc);
    for (int p = 2; p <= m; ++p) {
        for (uint32_t x = (1u << p) - 1; x < (1u << m);) {
            uint32_t sub = 0, c = rc;
            for (uint32_t y = x; y; y >>= 1) {
                const uint32_t low = c & (0u - c);
                if (y & 1u) sub |= low;
                c ^= low;
            }
            bool ok = true;
#pragma unroll
            for (int j = 0; j < K; ++j)
                if ((rest >> j) & 1u) ok &= (nm[j] & sub) != 0;
            if (ok) {
                best = forced | sub;
                return nf + p;
            }
            const uint32_t lo = x & (0u - x), r = x + lo;
            x = (((r ^ x) >> 2) >> (__ffs(lo) - 1)) | r;
        }
    }
    return -1;
}

template <int K>
__global__ void __launch_bounds__(kThreads)
assign_replicas_kernel(const int32_t *__restrict__ ids, int T, int E, int G, int rpn,
                       const int32_t *__restrict__ replica_rank, const int32_t *__restrict__ n_rep,
                       const int32_t *__restrict__ src_rank, int32_t *__restrict__ pick_rank,
                       int32_t *__restrict__ n_remote, int32_t *err)
{
    extern __shared__ int32_t sm[];
    __shared__ int node_of[64];                 // rank -> node
    const int nodes = G / rpn, max_rep = 1 + nodes;
    int32_t *rep = sm;                          // [E][max_rep]
    for (int r = threadIdx.x; r < G; r += blockDim.x) node_of[r] = r / rpn;
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
        uint32_t best = 0;
        int best_pop = 0;
        if (!bad) {
            best_pop = fewest_nodes<K>(need, nm, cand, best);
            if (best_pop < 0) bad = true;      // an expert with no replica at all
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
                const int nr = node_of[r];
                const bool allowed = any_ns ? (nr == ns) : ((best >> nr) & 1u);
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

constexpr int kCapThreads = 1024;
constexpr size_t kCapSetSmem = 160 * 1024;   // dynamic shared memory allowed with the pick-rank sets
constexpr int kCapMaxBlocks = 256;      // grid limit: every block keeps a [G][blocks] table

struct CapHeader {
    GridBarrier bar;
    int rounds;           // rounds run
};

struct CapArgs {
    const int32_t *ids;
    int T, E, G, rpn;
    const int32_t *rr, *nr, *src;
    long long cap;
    int32_t *pick, *nrem;
    long long *rank_load;     // [G] out or null
    CapHeader *h;
    int *blk;                 // [2][gridDim.x][G] tasks per rank of each block's tokens (round parity)
    int32_t *err;
    int cache_tok;            // tokens per block whose pick-rank sets live in shared memory (0: none)
};

// x's bits deposited, lowest first, onto the set bits of mask (<= 8 of them).
__device__ __forceinline__ uint32_t deposit8(uint32_t x, uint32_t mask)
{
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t low = mask & (0u - mask);
        if (x & 1u) r |= low;
        mask ^= low;
        x >>= 1;
    }
    return r;
}

// A listed token's inputs, loaded by its warp ahead of its turn: lane j < K
// its pick j's expert and, after the first round, the rank it had.
struct TokenIn {
    int t, v, s, old;
};

template <int K>
__device__ __forceinline__ TokenIn load_token(int t, const CapArgs &a, int rd)
{
    const int lane = threadIdx.x & 31;
    TokenIn x{t, -1, 0, -1};
    if (t < 0) return x;
    if (lane < K) x.v = __ldg(a.ids + (size_t)t * K + lane);
    x.s = a.src ? __ldg(a.src + t) : t / (a.T / a.G);
    if (rd > 0 && lane < K) x.old = __ldcg(a.pick + (size_t)t * K + lane);
    return x;
}

// Token x.t assigned by one warp over the usable replicas (uok[e]: usable
// ranks of e, unm[e]: their nodes), the same rule as the uncapped kernel:
// lane j < K holds pick j.  The fewest remote nodes come from warp
// reductions: the forced nodes, then one node covering the rest, else every
// set of the remaining candidate nodes at once (lanes over sets, the minimum
// of (size, set)).  Then every lane finds its pick's candidate ranks; a pick
// with one candidate, or with rank s among them, is settled at once, and the
// others take, in j order, the lowest candidate an earlier pick uses, else
// the lowest.  Every step is warp-uniform.  Writes pick_rank[t][*] and
// n_remote[t] (-1 for an invalid token) and moves the token's tasks in
// `hist` from its previous choice (rd > 0) to the new one.
template <int K>
__device__ __forceinline__ void assign_token_warp(const TokenIn &x, const CapArgs &a, int rd, int max_rep,
                                                  const int32_t *rep, const int *node_of, const uint32_t *unm,
                                                  const unsigned long long *uok, int *hist,
                                                  unsigned long long *pm_s, int lo)
{
    const int lane = threadIdx.x & 31;
    constexpr unsigned kAll = 0xffffffffu, kPicks = (1u << K) - 1u;
    const int t = x.t, v = x.v, s = x.s;
    const unsigned same = __match_any_sync(kAll, v);
    bool bad = __any_sync(kAll, lane < K && ((unsigned)v >= (unsigned)a.E || __popc(same & kPicks) > 1)) ||
               (unsigned)s >= (unsigned)a.G;
    int pick = -1, pop = -1;
    if (!bad) {
        const int ns = node_of[s];
        const uint32_t nm = lane < K ? unm[v] : 0u;
        const bool need = lane < K && !((nm >> ns) & 1u);
        const uint32_t cand = __reduce_or_sync(kAll, need ? nm : 0u) & ~(1u << ns);
        const uint32_t c = nm & cand;
        uint32_t best = 0;
        pop = 0;
        if (__any_sync(kAll, need)) {
            if (__any_sync(kAll, need && c == 0)) {
                pop = -1;                        // an expert without replicas
            } else {
                const uint32_t forced = __reduce_or_sync(kAll, (need && (c & (c - 1u)) == 0) ? c : 0u);
                const bool rest = need && (nm & forced) == 0;
                best = forced;
                pop = __popc(forced);
                if (__any_sync(kAll, rest)) {
                    const uint32_t rc = __reduce_or_sync(kAll, rest ? c : 0u);
                    const uint32_t one = __reduce_and_sync(kAll, rest ? nm : ~0u) & rc;
                    if (one) {
                        best |= one & (0u - one);
                        pop += 1;
                    } else {
                        uint32_t nmv[K];
                        const unsigned restm = __ballot_sync(kAll, rest);
#pragma unroll
                        for (int j = 0; j < K; ++j) nmv[j] = __shfl_sync(kAll, nm, j);
                        const uint32_t nsets = 1u << __popc(rc);
                        unsigned key = kAll;
                        for (uint32_t q = (uint32_t)lane + 1u; q < nsets; q += 32u) {
                            const uint32_t sub = deposit8(q, rc);
                            bool ok = true;
#pragma unroll
                            for (int j = 0; j < K; ++j)
                                if ((restm >> j) & 1u) ok &= (nmv[j] & sub) != 0;
                            if (ok) key = min(key, ((unsigned)__popc(q) << 8) | q);
                        }
                        key = __reduce_min_sync(kAll, key);
                        best |= deposit8(key & 0xffu, rc);
                        pop += (int)(key >> 8);
                    }
                }
            }
        }
        if (pop < 0) {
            bad = true;
        } else {
            // candidate ranks of pick j: usable replicas on the source node,
            // or (none there) on the nodes of S
            unsigned long long cm = 0;
            if (lane < K) {
                const unsigned long long ok = uok[v];
                const bool any_ns = (nm >> ns) & 1u;
                for (int q = 0; q < max_rep; ++q) {
                    const int r = rep[v * max_rep + q];
                    if (r >= 0 && ((ok >> r) & 1ull)) {
                        const int nr = node_of[r];
                        if (any_ns ? nr == ns : ((best >> nr) & 1u)) cm |= 1ull << r;
                    }
                }
                if ((cm >> s) & 1ull) pick = s;
                else if ((cm & (cm - 1ull)) == 0) pick = __ffsll((long long)cm) - 1;
            }
            for (unsigned open = __ballot_sync(kAll, lane < K && pick < 0); open; open &= open - 1u) {
                const int j = __ffs(open) - 1;   // picks before j are settled
                const unsigned long long mine = (lane < j) ? (1ull << pick) : 0ull;
                const unsigned long long used = ((unsigned long long)__reduce_or_sync(kAll, (unsigned)(mine >> 32)) << 32) |
                                                __reduce_or_sync(kAll, (unsigned)mine);
                if (lane == j) {
                    const unsigned long long u = cm & used;
                    pick = __ffsll((long long)(u ? u : cm)) - 1;
                }
            }
        }
    }
    if (bad && rd == 0 && lane == 0) record_error(a.err, MOE_DERR_ID_RANGE);
    if (lane < K) {
        if (x.old >= 0) atomicSub(&hist[x.old], 1);
        a.pick[(size_t)t * K + lane] = bad ? -1 : pick;
        if (!bad) atomicAdd(&hist[pick], 1);
    }
    if (lane == 0 && a.nrem) a.nrem[t] = bad ? -1 : pop;
    if (pm_s) {   // the block's copy of the token's pick-rank set
        const unsigned long long bit = (lane < K && !bad) ? 1ull << pick : 0ull;
        const unsigned lo32 = __reduce_or_sync(kAll, (unsigned)bit);
        const unsigned hi32 = __reduce_or_sync(kAll, (unsigned)(bit >> 32));
        if (lane == 0) pm_s[t - lo] = ((unsigned long long)hi32 << 32) | lo32;
    }
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

// The block holding token t under the fixed partition [T q / nb, T (q + 1) / nb).
__device__ __forceinline__ int block_of(int t, int T, int nb)
{
    int q = (int)((long long)t * nb / T);
    while (q + 1 < nb && (int)((long long)T * (q + 1) / nb) <= t) ++q;
    while (q > 0 && (int)((long long)T * q / nb) > t) --q;
    return q;
}

// Block b owns the tokens [T b / nb, T (b + 1) / nb) for the whole launch and
// keeps, in shared memory, the tasks per rank of its tokens not yet committed
// (those at or after tc).  A round re-evaluates only the tokens with an
// expert whose usable replicas changed with the ranks closed last round: for
// any other token the options, and so the choice, are the same as before.
template <int K>
__global__ void __launch_bounds__(kCapThreads)
assign_capped_kernel(CapArgs a)
{
    extern __shared__ __align__(16) unsigned char csm[];
    const int E = a.E, G = a.G, rpn = a.rpn, T = a.T;
    const int nodes = G / rpn, max_rep = 1 + nodes;
    const int nb = gridDim.x, b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned long long *uok = reinterpret_cast<unsigned long long *>(csm);             // [E]
    int32_t *rep = reinterpret_cast<int32_t *>(uok + E);                                  // [E][max_rep]
    uint32_t *unm = reinterpret_cast<uint32_t *>(rep + E * max_rep);                      // [E]
    int *chg = reinterpret_cast<int *>(unm + E);                                          // [E]
    int *pre = chg + E;                                                                   // [G][stride]
    const int stride = nb | 1;                // odd: the transposed writes spread over the banks
    // the ranks of each of this block's tokens' picks as one 64-bit set
    // (when they fit): a token none of whose picks sits on a rank that just
    // closed keeps its choice, and the set tells that without global loads
    const size_t pm_off = ((size_t)E * 8 + 4 * ((size_t)E * max_rep + 2 * (size_t)E + (size_t)G * stride) + 7) &
                          ~(size_t)7;
    unsigned long long *pm_s = a.cache_tok ? reinterpret_cast<unsigned long long *>(csm + pm_off) : nullptr;
    __shared__ int warp_tot[32];
    __shared__ unsigned closed_w[2];
    __shared__ unsigned long long lds[64];    // tasks committed per rank (the same in every block)
    __shared__ unsigned long long tot_s[64];  // open tokens' tasks per rank, all blocks
    __shared__ unsigned long long rc[64];     // tasks per rank of the partly committed block
    __shared__ long long run_s[64];           // a candidate rank's tasks in qb's tokens scanned so far
    __shared__ int hist[64];                  // this block's uncommitted tasks per rank
    __shared__ int node_of[64];               // rank -> node
    __shared__ int qx_s[64];                  // first block (from q0) where the rank reaches the cap
    __shared__ int list_s[kCapThreads];       // tokens of a tile to assign
    __shared__ int nlist_s;
    __shared__ int cross_s, qmin_s;
    __shared__ unsigned long long cand_s;     // the ranks that reach the cap in block q0 + qmin_s

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
        uok[e] = 0;
    }
    if (tid == 0) nlist_s = 0;
    for (int r = tid; r < 64; r += blockDim.x) {
        lds[r] = 0;
        hist[r] = 0;
        node_of[r] = r / rpn;
    }
    const int lo = (int)((long long)T * b / nb), hi = (int)((long long)T * (b + 1) / nb);
    if (!grid_barrier(&a.h->bar, a.err)) return;

    int tc = 0, any_chg = 0;
    unsigned long long closed_before = 0;
    for (int rd = 0; rd <= G + 1; ++rd) {
        int *blk = a.blk + (size_t)(rd & 1) * kCapMaxBlocks * G;
        const int q0 = block_of(tc, T, nb);             // the block holding tc
        // (a) the closed ranks, each expert's usable replicas, and whether
        // they changed since the last round
        if (tid < 64) {
            const unsigned bl = __ballot_sync(0xffffffffu, tid < G && (long long)lds[tid] >= a.cap);
            if (lane == 0) closed_w[warp] = bl;
        }
        __syncthreads();
        const unsigned long long closed = ((unsigned long long)closed_w[1] << 32) | closed_w[0];
        const unsigned long long closing = closed & ~closed_before;   // ranks closed since the last round
        closed_before = closed;
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
                if (r >= 0 && ((u >> r) & 1ull)) m |= 1u << node_of[r];
            }
            chg[e] = rd == 0 || u != uok[e];
            any_chg |= chg[e];
            uok[e] = u;
            unm[e] = m;
        }
        // no expert's usable replicas changed: no choice changes this round
        const bool some_chg = __syncthreads_or(any_chg) != 0;
        any_chg = 0;
        // (b) round 0: the choices are those of the uncapped assignment
        // (no rank is open-and-closed yet: every replica is usable), which
        // the launch before this one wrote; count them
        if (rd == 0)
            for (int t0 = lo; t0 < hi; t0 += kCapThreads) {
                const int t = t0 + tid;
                unsigned long long pm = 0;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int r = t < hi ? __ldcg(a.pick + (size_t)t * K + j) : -1;
                    const unsigned same = __match_any_sync(0xffffffffu, r);
                    if (r >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[r], __popc(same));
                    if (r >= 0) pm |= 1ull << r;
                }
                if (pm_s && t < hi) pm_s[t - lo] = pm;
            }
        // later rounds: the choices of this block's open tokens whose options
        // changed: a tile of tokens (one per thread) is checked, the changed
        // ones are listed in shared memory, and the warps assign the listed
        // tokens one token per warp at a time
        for (int t0 = max(lo, tc); rd > 0 && some_chg && t0 < hi; t0 += kCapThreads) {
            const int t = t0 + tid;
            // a token's choice can change only through a pick on a rank that
            // just closed, of an expert whose usable replicas changed: while
            // every pick stays usable the old node set stays feasible, and
            // with fewer options it stays the smallest (and so do the picks);
            // options grow only when an expert's last open replica closes,
            // and that replica was then its pick
            bool dirty = false;
            if (t < hi && (!pm_s || (pm_s[t - lo] & closing) != 0)) {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int e = __ldg(a.ids + (size_t)t * K + j);
                    const int r = __ldcg(a.pick + (size_t)t * K + j);
                    if ((unsigned)e < (unsigned)E && r >= 0)
                        dirty |= chg[e] != 0 && ((closing >> r) & 1ull);
                }
            }
            const unsigned bal = __ballot_sync(0xffffffffu, dirty);
            int at = 0;
            if (lane == 0 && bal) at = atomicAdd(&nlist_s, __popc(bal));
            at = __shfl_sync(0xffffffffu, at, 0);
            if (dirty) list_s[at + __popc(bal & ((1u << lane) - 1u))] = t;
            __syncthreads();
            const int n = nlist_s;
            // each warp's next token is loaded while it assigns the current one
            TokenIn cur = load_token<K>(warp < n ? list_s[warp] : -1, a, rd);
            for (int i = warp; i < n; i += kCapThreads / 32) {
                const int i2 = i + kCapThreads / 32;
                const TokenIn nxt = load_token<K>(i2 < n ? list_s[i2] : -1, a, rd);
                assign_token_warp<K>(cur, a, rd, max_rep, rep, node_of, unm, uok, hist, pm_s, lo);
                cur = nxt;
            }
            __syncthreads();
            if (tid == 0) nlist_s = 0;
            __syncthreads();
        }
        __syncthreads();
        for (int r = tid; r < G; r += blockDim.x) blk[(size_t)b * G + r] = hist[r];
        if (!grid_barrier(&a.h->bar, a.err)) return;
        // (c) every block alike, from all blocks' counts: per rank the running
        // sum over the blocks with open tokens (q0 on, in token order), the
        // first block in which an open rank reaches the cap, the token inside
        // it at which that happens (tau - 1), and the commit of the tokens
        // before tau in this block's copy of the loads.  One grid barrier a
        // round: the counts are double-buffered by round, and the picks read
        // here (tokens before tau) are final.
        const int nq = nb - q0;                       // blocks with open tokens
        {
            // thread (qq, r) copies rows qq, qq + P, ... of column r (one
            // division per thread, not per element)
            const int P = kCapThreads / G, qq = tid / G, r = tid - qq * G;
            if (qq < P)
                for (int q = qq; q < nq; q += P) pre[r * stride + q] = __ldcg(blk + (size_t)(q0 + q) * G + r);
        }
        __syncthreads();
        for (int r = warp; r < G; r += kCapThreads / 32) {
            // exclusive running sums in place; the first block where the
            // committed tasks plus the running sum reach the cap
            const bool open = (long long)lds[r] < a.cap;
            const long long need = a.cap - (long long)lds[r];
            long long run = 0;
            int qx = nq;
            for (int c0 = 0; c0 < nq; c0 += 32) {
                const int q = c0 + lane;
                const int v = q < nq ? pre[r * stride + q] : 0;
                int incl = v;                         // 32 blocks' tasks: at most T k < 2^31
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (q < nq) pre[r * stride + q] = (int)(run + incl - v);
                const unsigned hit = __ballot_sync(0xffffffffu, open && q < nq && run + incl >= need);
                if (qx == nq && hit) qx = c0 + __ffs(hit) - 1;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) {
                qx_s[r] = qx;
                tot_s[r] = (unsigned long long)run;
            }
        }
        __syncthreads();
        if (warp == 0) {
            int m = nq;
            if (lane < G) m = min(m, qx_s[lane]);
            if (lane + 32 < G) m = min(m, qx_s[lane + 32]);
            m = (int)__reduce_min_sync(0xffffffffu, (unsigned)m);
            // the ranks that reach the cap inside that block
            const unsigned c0 = __ballot_sync(0xffffffffu, lane < G && qx_s[lane] == m);
            const unsigned c1 = __ballot_sync(0xffffffffu, lane + 32 < G && qx_s[lane + 32] == m);
            if (lane == 0) {
                qmin_s = m;
                cand_s = ((unsigned long long)c1 << 32) | c0;
            }
        }
        __syncthreads();
        const int qm = qmin_s;
        int tau = T;
        if (qm < nq) {
            const int qb = q0 + qm;                   // the block holding the first crossing
            const int first = max((int)((long long)T * qb / nb), tc);
            const int last = (int)((long long)T * (qb + 1) / nb);
            const unsigned long long cand = cand_s;
            if (tid == 0) cross_s = last;
            for (int r = tid; r < G; r += blockDim.x) {
                rc[r] = 0;
                run_s[r] = 0;
            }
            __syncthreads();
            // one pass over qb's tokens, a tile at a time, the picks loaded
            // once: per candidate rank the token whose tasks take the rank's
            // running count to its remaining room (the earliest over the
            // ranks is the crossing, tau - 1), then the commit of the tile's
            // tokens before tau (a warp's lanes on one rank add once: the
            // picks crowd onto the hot ranks)
            for (int t0 = first; t0 < last; t0 += kCapThreads) {
                const int t = t0 + tid;
                int pk[K];
#pragma unroll
                for (int j = 0; j < K; ++j) pk[j] = t < last ? __ldcg(a.pick + (size_t)t * K + j) : -1;
                for (unsigned long long cm = cand; cm; cm &= cm - 1ull) {
                    const int r = __ffsll((long long)cm) - 1;
                    const long long need = a.cap - (long long)lds[r] - pre[r * stride + qm];
                    int c = 0;
#pragma unroll
                    for (int j = 0; j < K; ++j) c += pk[j] == r;
                    const int incl = block_scan_incl(c, warp_tot);
                    const long long run = run_s[r];
                    if (t < last && run + incl >= need && run + incl - c < need) atomicMin(&cross_s, t);
                    __syncthreads();
                    if (tid == kCapThreads - 1) run_s[r] = run + incl;
                }
                __syncthreads();
                const int cross = cross_s;
                const int upto = min(cross + 1, last);
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int r = t < upto ? pk[j] : -1;
                    const unsigned same = __match_any_sync(0xffffffffu, r);
                    if (r >= 0 && lane == __ffs(same) - 1) atomicAdd(&rc[r], (unsigned long long)__popc(same));
                }
                if (cross < last) break;              // the same in every thread
            }
            __syncthreads();
            tau = cross_s + 1;
            for (int r = tid; r < G; r += blockDim.x) {
                lds[r] += (unsigned long long)pre[r * stride + qm] + rc[r];
                if (b == qb) hist[r] -= (int)rc[r];
            }
        } else {
            for (int r = tid; r < G; r += blockDim.x) lds[r] += tot_s[r];   // no rank closes: all final
        }
        if (hi <= tau)
            for (int r = tid; r < G; r += blockDim.x) hist[r] = 0;
        __syncthreads();
        tc = tau;
        if (tc >= T) {
            if (b == 0 && tid == 0) a.h->rounds = rd + 1;
            break;
        }
        if (rd == G + 1) record_error(a.err, MOE_DERR_TIMEOUT);   // more rounds than ranks: not reachable
    }
    if (b == 0 && a.rank_load)
        for (int r = tid; r < G; r += blockDim.x) a.rank_load[r] = (long long)lds[r];
}

template <int K>
moe_status launch_capped(CapArgs args, cudaStream_t s)
{
    auto kern = assign_capped_kernel<K>;
    const int max_rep = 1 + args.G / args.rpn;
    const int nb = std::min(coop_grid(), kCapMaxBlocks);
    size_t smem = sizeof(unsigned long long) * (size_t)args.E +
                  sizeof(int32_t) * ((size_t)args.E * max_rep + 2 * (size_t)args.E + (size_t)args.G * (nb | 1));
    // the per-token pick-rank sets of a block's tokens, when they fit
    const size_t tpb = ((size_t)args.T + nb - 1) / nb;
    const size_t with_sets = round_up(smem, 8) + sizeof(unsigned long long) * tpb;
    args.cache_tok = 0;
    if (with_sets <= kCapSetSmem) {
        args.cache_tok = (int)tpb;
        smem = with_sets;
    }
    if (allow_smem(kern, smem) != cudaSuccess) return MOE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCapThreads, smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (per_sm < 1) return MOE_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)nb);        // at most one block per SM: co-resident
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
    return 256 + round_up(sizeof(int) * 2 * (size_t)kCapMaxBlocks * G, 256);
}

extern "C" moe_status moe_assign_replicas_capped(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                                 const int32_t *replica_rank, const int32_t *n_rep,
                                                 const int32_t *src_rank, double eps, int32_t *pick_rank,
                                                 int32_t *n_remote, long long *rank_load, int32_t *err,
                                                 void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (T < 0 || k < 1 || k > 8 || E < k || G < 1 || G > 64 || rpn < 1 || G % rpn != 0 || !err) return MOE_ERR_ARG;
    if (!(eps >= 0.0) || (long long)T * k >= (1ll << 31)) return MOE_ERR_ARG;   // task counts are int32
    if (G / rpn > kMaxNodes) return MOE_ERR_UNSUPPORTED;
    if ((size_t)E * (G / rpn + 3) * sizeof(int32_t) + (size_t)E * 8 +
            (size_t)G * (std::min(coop_grid(), kCapMaxBlocks) | 1) * sizeof(int32_t) > 200 * 1024)
        return MOE_ERR_UNSUPPORTED;
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
    a.blk = reinterpret_cast<int *>(w + 256);
    a.err = err;
    if (cudaMemsetAsync(w, 0, 256, stream) != cudaSuccess) return MOE_ERR_CUDA;
    // the first round's choices -- every replica usable -- are the uncapped
    // assignment: one thread per token over the whole GPU, then the rounds
    moe_status st = MOE_ERR_ARG;
    switch (k) {
#define MOE_CAPPED_CASE(KK)                                                                                  \
    case KK:                                                                                                 \
        st = launch_assign<KK>(ids, T, E, G, rpn, replica_rank, n_rep, src_rank, pick_rank, n_remote, err,   \
                               stream);                                                                      \
        if (st == MOE_OK) st = launch_capped<KK>(a, stream);                                                 \
        break;
    MOE_CAPPED_CASE(1) MOE_CAPPED_CASE(2) MOE_CAPPED_CASE(3) MOE_CAPPED_CASE(4)
    MOE_CAPPED_CASE(5) MOE_CAPPED_CASE(6) MOE_CAPPED_CASE(7) MOE_CAPPED_CASE(8)
#undef MOE_CAPPED_CASE
    }
    if (st == MOE_OK) note_launches(2);
    return st;
}

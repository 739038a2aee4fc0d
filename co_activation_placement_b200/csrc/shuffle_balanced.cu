// Capacity-balanced token shuffle.
//
// "Expert Coupling in MoE Pretraining", abstract: under sequence parallelism
// every token moves, during the reduce-scatter that follows attention, to the
// GPU predicted to hold its next-layer experts.  A reduce-scatter hands every
// rank an equal shard, so here every rank receives at most `capacity` tokens.
// Token t scores rank r with S_t(r) = sum_j rank_score[e_tj][r] (as the
// unconstrained target); the result is the assignment reached by taking all
// (t, r) pairs in the order S desc, t asc, r asc and accepting a pair when t
// has no rank yet and r still has room.
//
// That greedy is sequential over T*G pairs.  Its result is also the unique
// stable assignment for "tokens prefer ranks by (S desc, r asc), ranks prefer
// tokens by (S desc, t asc)" (both orders come from one ordering of the pairs),
// so it is computed here by token-proposing deferred acceptance, run in rounds
// by one persistent cooperative kernel:
//   A  every free token proposes to its best rank among those that could still
//      take it: a rank with room, or a full rank whose weakest holder ranks
//      below the token (key > theta_r).  A proposal to any other rank would be
//      rejected, now and later (theta_r only rises), so skipping it changes
//      nothing but the number of rounds.  Proposals are counted per rank in
//      shared memory, then once per block in global memory.
//   C  each rank (owned by one block for the whole kernel) gathers its
//      proposals from the round's list into shared memory next to its
//      holders, keeps the best `capacity` of them -- a radix select of the
//      capacity-th largest key, from the highest byte in which the candidates
//      differ -- and returns the rest to the free list.
// A key packs (S_t(r) << 28) | (2^28 - 1 - t): one uint64 comparison orders
// a rank's candidates by S desc then t asc, and for one token orders ranks by
// S (equal S: the lower rank is preferred explicitly).
//
// Rounds take two grid barriers (after A and after C).  Every wait is bounded (2 s of
// %globaltimer); a block that gives up records MOE_DERR_TIMEOUT, raises an
// abort flag that releases every other waiting block, and returns.  The grid
// is launched cooperatively, so all blocks are co-resident and the barriers
// complete.
#include <algorithm>

#include "common.cuh"
#include "waits.cuh"

namespace moe {
namespace {

constexpr int kBalThreads = 512;
constexpr int kBalWarps = kBalThreads / 32;
constexpr int kKeyShift = 28;
constexpr unsigned long long kTokMask = (1ull << kKeyShift) - 1;
constexpr int kScratchKeys = 4096;          // boundary-bin scratch of the selection (32 KB)

struct BalHeader {            // cleared before every launch
    GridBarrier bar;
    int nfree[2];             // free tokens for the round of that parity
    int pad[2];
    long long proposals;
    int cnt[2][64];           // proposals per rank, round parity
    unsigned long long theta[64];   // weakest holder's key of a full rank; 0 while it has room
};

struct BalLayout {
    size_t hdr, fl0, fl1, prop_r, prop_key, bucket, hold0, hold1, total;
};

BalLayout bal_layout(long long T, int G, long long Cc)
{
    BalLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = round_up(o + std::max<size_t>(bytes, 1), 256); return at; };
    L.hdr = take(sizeof(BalHeader));
    L.fl0 = take(sizeof(int) * T);
    L.fl1 = take(sizeof(int) * T);
    L.prop_r = take(sizeof(int) * T);
    L.prop_key = take(sizeof(unsigned long long) * T);
    L.bucket = take(sizeof(unsigned long long) * T);
    L.hold0 = take(sizeof(unsigned long long) * G * Cc);
    L.hold1 = take(sizeof(unsigned long long) * G * Cc);
    L.total = o;
    return L;
}

struct BalArgs {
    const int32_t *ids;
    int T, E, G, Cc;
    int stage;                // keys the shared-memory staging area holds
    int scratch;              // keys the boundary-bin scratch area holds
    const uint32_t *rs;
    int32_t *target;
    long long *info;
    BalHeader *h;
    int *fl[2];
    int *prop_r;
    unsigned long long *prop_key, *bucket, *hold[2];
    int32_t *err;
};

__device__ __forceinline__ unsigned long long block_min(unsigned long long v, unsigned long long *red)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = lane < kBalWarps ? red[lane] : ~0ull;
#pragma unroll
    for (int o = 16; o; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int K>
__global__ void __launch_bounds__(kBalThreads, 1) shuffle_balanced_kernel(BalArgs a)
{
    extern __shared__ __align__(16) uint32_t tab[];   // rank_score [E][G], then the staging area
    __shared__ unsigned long long theta_s[64], hmin_s[64], red_s[kBalWarps];
    __shared__ int cnt_s[64], base_s[64], tot_s[64], hn_s[64], hsel_s[64];
    __shared__ unsigned int hist_s[256];
    __shared__ int kept_s, digit_s, need_s, gather_s, bin_s;
    constexpr int KP = (K + 3) & ~3;                  // picks per staged token, padded to int4
    __shared__ __align__(16) int picks_s[kBalWarps][32 * KP];
    __shared__ int tok_s[kBalWarps][32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = a.G, E = a.E, Cc = a.Cc;
    BalHeader *h = a.h;
    unsigned long long *stage = reinterpret_cast<unsigned long long *>(tab + ((E * G + 1) & ~1));
    unsigned long long *scr = stage + a.stage;        // boundary-bin scratch, a.scratch keys
    for (int i = tid; i < E * G; i += kBalThreads) tab[i] = __ldg(a.rs + i);
    if (tid < 64) { hn_s[tid] = 0; hsel_s[tid] = 0; hmin_s[tid] = ~0ull; }
    __syncthreads();

    const long long round_limit = (long long)a.T * G + 1;
    long long proposals = 0;
    // time in each phase (info[2..5]): proposing and waiting at barriers as
    // block 0 sees them, gathering and selecting as the slowest block's total
    const bool clk = a.info && tid == 0;
    unsigned long long t_a = 0, t_b = 0, t_c = 0, t_w = 0, t_mark = clk ? gtimer_ns() : 0;
    auto lap = [&](unsigned long long &acc) {
        if (clk) {
            const unsigned long long now = gtimer_ns();
            acc += now - t_mark;
            t_mark = now;
        }
    };
    int rd = 0;
    for (;; ++rd) {
        const int p = rd & 1;
        const int nF = rd == 0 ? a.T : __ldcg(&h->nfree[p]);
        proposals += nF;
        if (blockIdx.x == 0) {   // counters of the next round (unused in this one)
            if (tid < 64) h->cnt[p ^ 1][tid] = 0;
            if (tid == 0) h->nfree[p ^ 1] = 0;
        }
        // ---- A: proposals
        if (tid < 64) {
            theta_s[tid] = tid < G ? __ldcg(&h->theta[tid]) : 0ull;
            cnt_s[tid] = 0;
        }
        __syncthreads();
        const int *fl = p ? a.fl[1] : a.fl[0];
        // a warp scores `per` free tokens one after another: up to 32, fewer
        // when the free list is short, so that every warp shares the work
        const int nwt = gridDim.x * kBalWarps;
        const int per = min(32, max(1, (nF + nwt - 1) / nwt));
        const int stride = nwt * per;
        for (int i0 = (blockIdx.x * kBalWarps + warp) * per; i0 < nF; i0 += stride) {
            const int i = i0 + lane;
            const bool mine = lane < per && i < nF;
            int t = 0;
            int e[K];
            bool ok = mine;
            if (mine) t = rd == 0 ? i : __ldcg(fl + i);
#pragma unroll
            for (int j = 0; j < K; ++j) {
                e[j] = mine ? __ldg(a.ids + (size_t)t * K + j) : 0;
                if ((unsigned)e[j] >= (unsigned)E) { ok = false; e[j] = 0; }
            }
            if (mine && !ok) record_error(a.err, MOE_DERR_ID_RANGE);
            // stage the warp's tokens and picks (-1: a token with an invalid
            // pick, which then scores 0 everywhere) for broadcast reads
            int *pk = picks_s[warp];
            if (lane < per) {
                tok_s[warp][lane] = t;
#pragma unroll
                for (int j = 0; j < KP; ++j) pk[lane * KP + j] = (j < K && ok) ? e[j] : -1;
            }
            __syncwarp();
            const int n = min(per, nF - i0);
            int my_r = 0;
            unsigned long long my_key = 0;
            for (int q = 0; q < n; ++q) {
                const int tq = tok_s[warp][q];
                int ev[KP];
#pragma unroll
                for (int c4 = 0; c4 < KP / 4; ++c4) {
                    const int4 v = reinterpret_cast<const int4 *>(pk + q * KP)[c4];
                    ev[4 * c4] = v.x; ev[4 * c4 + 1] = v.y; ev[4 * c4 + 2] = v.z; ev[4 * c4 + 3] = v.w;
                }
                const bool good = ev[0] >= 0;
                unsigned long long s0 = 0, s1 = 0;
                if (good) {
#pragma unroll
                    for (int j = 0; j < K; ++j) {
                        const uint32_t *row = tab + (size_t)ev[j] * G;
                        if (lane < G) s0 += row[lane];
                        if (lane + 32 < G) s1 += row[lane + 32];
                    }
                }
                // one packed value per rank: (S + 1) << 6 | (63 - r), or 0 for a
                // rank that would reject the token (its key <= theta_r); the
                // warp maximum is the best acceptable rank (equal S: lower r):
                // one redux.sync when every S fits 25 bits, else 64-bit shuffles
                const unsigned long long low = kTokMask - (unsigned long long)tq;
                const bool ok0 = lane < G && ((s0 << kKeyShift) | low) > theta_s[lane];
                const bool ok1 = lane + 32 < G && ((s1 << kKeyShift) | low) > theta_s[lane + 32];
                unsigned long long best;
                if (__all_sync(0xffffffffu, (s0 | s1) < (1ull << 25))) {
                    uint32_t v = ok0 ? (((uint32_t)s0 + 1u) << 6) | (uint32_t)(63 - lane) : 0u;
                    if (ok1) v = max(v, (((uint32_t)s1 + 1u) << 6) | (uint32_t)(31 - lane));
                    best = __reduce_max_sync(0xffffffffu, v);
                } else {
                    best = ok0 ? ((s0 + 1) << 6) | (unsigned long long)(63 - lane) : 0ull;
                    if (ok1) best = max(best, ((s1 + 1) << 6) | (unsigned long long)(31 - lane));
#pragma unroll
                    for (int o = 16; o; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
                }
                if (lane == q) {
                    my_r = 63 - (int)(best & 63u);
                    my_key = best ? (((best >> 6) - 1) << kKeyShift) | low : 0ull;
                }
            }
            __syncwarp();
            if (mine) {
                if (my_key == 0) {            // no rank can take it: impossible while T <= G*capacity
                    record_error(a.err, MOE_DERR_RANK_RANGE);
                    atomicExch(&h->bar.abort, 1u);
                    my_r = 0;
                }
                __stcg(a.prop_r + i, my_r);
                __stcg(a.prop_key + i, my_key);
            }
            // one add per rank and warp: proposals crowd onto the hot ranks
            const int cr = mine ? my_r : -1;
            const unsigned same = __match_any_sync(0xffffffffu, cr);
            if (cr >= 0 && lane == __ffs(same) - 1) atomicAdd(&cnt_s[cr], __popc(same));
        }
        __syncthreads();
        if (tid < G && cnt_s[tid]) atomicAdd(&h->cnt[p][tid], cnt_s[tid]);
        lap(t_a);
        if (!grid_barrier(&h->bar, a.err)) return;
        lap(t_w);

        // proposals per rank and their exclusive prefix (a rank's segment of
        // the bucket array, used when its candidates exceed shared memory)
        if (warp == 0) {
            const int c0 = lane < G ? __ldcg(&h->cnt[p][lane]) : 0;
            const int c1 = lane + 32 < G ? __ldcg(&h->cnt[p][lane + 32]) : 0;
            int s0 = c0, s1 = c1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v0 = __shfl_up_sync(0xffffffffu, s0, o);
                const int v1 = __shfl_up_sync(0xffffffffu, s1, o);
                if (lane >= o) { s0 += v0; s1 += v1; }
            }
            const int total0 = __shfl_sync(0xffffffffu, s0, 31);
            base_s[lane] = s0 - c0;
            base_s[lane + 32] = total0 + s1 - c1;
            tot_s[lane] = c0;
            tot_s[lane + 32] = c1;
        }
        __syncthreads();

        // ---- C: every rank keeps its best Cc candidates
        const int pn = p ^ 1;
        for (int r = blockIdx.x; r < G; r += gridDim.x) {
            const int np = tot_s[r];
            if (np == 0) continue;
            const int hn = hn_s[r];
            const int sel = hsel_s[r];
            unsigned long long *cur = (sel ? a.hold[1] : a.hold[0]) + (size_t)r * Cc;
            unsigned long long *alt = (sel ? a.hold[0] : a.hold[1]) + (size_t)r * Cc;
            unsigned long long *B = a.bucket + base_s[r];
            const int n = hn + np;
            const bool append = n <= Cc;
            const bool staged = !append && n <= a.stage;
            // the rank's proposals, gathered from the round's proposal list:
            // after the holders (appended, or staged in shared memory), or
            // into the rank's bucket segment when they do not fit
            unsigned long long *dst = append ? cur + hn : staged ? stage + hn : B;
            unsigned long long lo = ~0ull, hi = 0;
            if (tid == 0) gather_s = 0;
            __syncthreads();
            for (int i0 = 0; i0 < nF; i0 += 8 * kBalThreads) {
                int rr[8];
                unsigned long long kk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + u * kBalThreads + tid;
                    rr[u] = i < nF ? __ldcg(a.prop_r + i) : -1;
                    kk[u] = i < nF ? __ldcg(a.prop_key + i) : 0ull;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const bool m = rr[u] == r;
                    const unsigned int mk = __ballot_sync(0xffffffffu, m);
                    if (mk == 0) continue;
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&gather_s, __popc(mk));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (m) {
                        const unsigned long long v = kk[u];
                        const int slot = base + __popc(mk & ((1u << lane) - 1u));
                        if (staged) dst[slot] = v; else __stcg(dst + slot, v);
                        lo = min(lo, v);
                        hi = max(hi, v);
                    }
                }
            }
            lap(t_b);
            if (append) {
                lo = block_min(lo, red_s);
                if (tid == 0) {
                    hmin_s[r] = min(hmin_s[r], lo);
                    hn_s[r] = n;
                    if (n == Cc) __stcg(&h->theta[r], hmin_s[r]);
                }
                __syncthreads();
                continue;
            }
            // the holders join the candidates (copied when staged)
            for (int x0 = tid; x0 < hn; x0 += 4 * kBalThreads) {
                unsigned long long v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int x = x0 + u * kBalThreads;
                    v[u] = x < hn ? __ldcg(cur + x) : 0ull;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int x = x0 + u * kBalThreads;
                    if (x < hn) {
                        if (staged) stage[x] = v[u];
                        lo = min(lo, v[u]);
                        hi = max(hi, v[u]);
                    }
                }
            }
            lo = block_min(lo, red_s);
            hi = ~block_min(~hi, red_s);
            auto cand = [&](int x) -> unsigned long long {
                return staged ? stage[x] : __ldcg(x < hn ? cur + x : B + (x - hn));
            };
            // radix select of the Cc-th largest key, one byte at a time from
            // the highest byte in which the candidates differ (lo != hi: the
            // keys are distinct and n > Cc >= 1)
            const int top = (63 - __clzll((long long)(lo ^ hi))) & ~7;
            unsigned long long pmask = top == 56 ? 0ull : ~((1ull << (top + 8)) - 1);
            unsigned long long prefix = lo & pmask;
            int need = Cc;
            // once the candidates left in the boundary bin fit the scratch
            // area, they are collected there and later passes scan only them
            bool collected = false;
            int m = n;
            for (int shift = top; shift >= 0; shift -= 8) {
                if (tid < 256) hist_s[tid] = 0;
                __syncthreads();
                const int len = collected ? m : n;
                for (int x0 = tid; x0 < len; x0 += 8 * kBalThreads) {   // 8 loads in flight
                    unsigned long long v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int x = x0 + u * kBalThreads;
                        v[u] = x < len ? (collected ? scr[x] : cand(x)) : 0ull;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (x0 + u * kBalThreads < len && (v[u] & pmask) == prefix)
                            atomicAdd(&hist_s[(v[u] >> shift) & 255u], 1u);
                }
                __syncthreads();
                if (warp == 0) {
                    // lane l owns digits 255-8l down to 248-8l (descending)
                    unsigned int c[8], sum = 0;
#pragma unroll
                    for (int u = 0; u < 8; ++u) { c[u] = hist_s[255 - 8 * lane - u]; sum += c[u]; }
                    unsigned int incl = sum;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const unsigned int v = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    const unsigned int excl = incl - sum;
                    if (excl < (unsigned)need && incl >= (unsigned)need) {
                        unsigned int acc = excl;
                        int d = 255 - 8 * lane;
                        unsigned int cd = c[0];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            if (acc + c[u] >= (unsigned)need) { d = 255 - 8 * lane - u; cd = c[u]; break; }
                            acc += c[u];
                        }
                        digit_s = d;
                        need_s = need - (int)acc;
                        bin_s = (int)cd;
                    }
                }
                __syncthreads();
                prefix |= (unsigned long long)digit_s << shift;
                pmask |= 0xffull << shift;
                need = need_s;
                const int in_bin = bin_s;
                if (!collected && shift > 0 && in_bin <= a.scratch) {
                    if (tid == 0) gather_s = 0;
                    __syncthreads();
                    for (int x0 = 0; x0 < n; x0 += 8 * kBalThreads) {
                        unsigned long long v[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int x = x0 + u * kBalThreads + tid;
                            v[u] = x < n ? cand(x) : 0ull;
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const bool in = x0 + u * kBalThreads + tid < n && (v[u] & pmask) == prefix;
                            const unsigned int mk = __ballot_sync(0xffffffffu, in);
                            if (mk == 0) continue;
                            int base = 0;
                            if (lane == 0) base = atomicAdd(&gather_s, __popc(mk));
                            base = __shfl_sync(0xffffffffu, base, 0);
                            if (in) scr[base + __popc(mk & ((1u << lane) - 1u))] = v[u];
                        }
                    }
                    __syncthreads();
                    collected = true;
                    m = in_bin;
                }
            }
            const unsigned long long theta = prefix;   // keys are distinct: exactly Cc keys >= theta
            if (tid == 0) kept_s = 0;
            __syncthreads();
            int *fl_next = pn ? a.fl[1] : a.fl[0];
            for (int x0 = 0; x0 < n; x0 += 8 * kBalThreads) {
                unsigned long long vv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int x = x0 + u * kBalThreads + tid;
                    vv[u] = x < n ? cand(x) : 0ull;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int x = x0 + u * kBalThreads + tid;
                    const unsigned long long v = vv[u];
                    const bool keep = x < n && v >= theta;
                    const bool rej = x < n && v < theta;
                    const unsigned int mk = __ballot_sync(0xffffffffu, keep);
                    const unsigned int mr = __ballot_sync(0xffffffffu, rej);
                    int kb = 0, rb = 0;
                    if (lane == 0) {
                        if (mk) kb = atomicAdd(&kept_s, __popc(mk));
                        if (mr) rb = atomicAdd(&h->nfree[pn], __popc(mr));
                    }
                    kb = __shfl_sync(0xffffffffu, kb, 0);
                    rb = __shfl_sync(0xffffffffu, rb, 0);
                    const unsigned int below = (1u << lane) - 1u;
                    if (keep) {
                        const int slot = kb + __popc(mk & below);
                        if (slot < Cc) __stcg(alt + slot, v);
                    }
                    if (rej) __stcg(fl_next + rb + __popc(mr & below), (int)(kTokMask - (v & kTokMask)));
                }
            }
            __syncthreads();
            if (tid == 0) {
                if (kept_s != Cc) {           // impossible: keys are distinct
                    record_error(a.err, MOE_DERR_ROW_RANGE);
                    atomicExch(&h->bar.abort, 1u);
                }
                hn_s[r] = Cc;
                hsel_s[r] = sel ^ 1;
                hmin_s[r] = theta;
                __stcg(&h->theta[r], theta);
            }
            __syncthreads();
        }
        lap(t_c);
        if (!grid_barrier(&h->bar, a.err) || __ldcg(&h->bar.abort)) return;
        lap(t_w);
        if (__ldcg(&h->nfree[pn]) == 0) break;
        if (rd + 1 >= round_limit) {           // cannot happen: each round is a new rank for every free token
            if (blockIdx.x == 0 && tid == 0) record_error(a.err, MOE_DERR_TIMEOUT);
            break;
        }
    }
    // every token is held by exactly one rank
    for (int r = blockIdx.x; r < G; r += gridDim.x) {
        const unsigned long long *cur = (hsel_s[r] ? a.hold[1] : a.hold[0]) + (size_t)r * Cc;
        for (int x = tid; x < hn_s[r]; x += kBalThreads)
            a.target[kTokMask - (__ldcg(cur + x) & kTokMask)] = r;
    }
    if (clk) {
        atomicMax(reinterpret_cast<unsigned long long *>(a.info + 3), t_b);
        atomicMax(reinterpret_cast<unsigned long long *>(a.info + 4), t_c);
        if (blockIdx.x == 0) {
            a.info[0] = rd + 1;
            a.info[1] = proposals;
            a.info[2] = (long long)t_a;
            a.info[5] = (long long)t_w;
        }
    }
}

template <int K>
moe_status launch_balanced(BalArgs args, cudaStream_t s)
{
    auto kern = shuffle_balanced_kernel<K>;
    // dynamic shared memory: the score table, then as many staged keys as the
    // rest of the block's shared memory holds (at most the candidates a rank
    // can have: capacity + proposals <= 2T), then the boundary-bin scratch
    int dev = 0, optin = 0;
    cudaFuncAttributes fa{};
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(kern)) != cudaSuccess)
        return MOE_ERR_CUDA;
    const size_t table = sizeof(uint32_t) * (size_t)((args.E * args.G + 1) & ~1);
    const long long room = (long long)optin - (long long)fa.sharedSizeBytes - (long long)table - 1024;
    if (room < 0) return MOE_ERR_UNSUPPORTED;
    args.scratch = (int)std::min<long long>(kScratchKeys, room / 16);
    args.stage = (int)std::min<long long>(room / 8 - args.scratch, 2LL * args.T);
    const size_t smem = table + sizeof(unsigned long long) * ((size_t)args.stage + args.scratch);
    if (allow_smem(kern, smem) != cudaSuccess) return MOE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBalThreads, smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (per_sm < 1) return MOE_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)coop_grid());    // at most one block per SM: co-resident by construction
    cfg.blockDim = dim3(kBalThreads);
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

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" size_t moe_shuffle_balanced_workspace(int T, int G, int capacity)
{
    if (T < 0 || G < 1 || G > 64 || capacity < 0) return 0;
    const long long Cc = std::min<long long>(capacity, T);
    return bal_layout(T, G, Cc).total;
}

extern "C" moe_status moe_shuffle_balanced(const int32_t *ids, int T, int k, int E, int G,
                                           const uint32_t *rank_score, int capacity, int32_t *target,
                                           long long *info, void *ws, size_t ws_bytes, int32_t *err,
                                           cudaStream_t stream)
{
    if (T < 0 || k < 1 || k > 8 || E < k || G < 1 || G > 64 || capacity < 0 || !err) return MOE_ERR_ARG;
    if ((long long)G * capacity < T) return MOE_ERR_ARG;
    if ((long long)E * G > 16384 || T >= (1 << 27)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) {
        if (info && cudaMemsetAsync(info, 0, 6 * sizeof(long long), stream) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!ids || !rank_score || !target || !ws) return MOE_ERR_ARG;
    const int Cc = std::min(capacity, T);
    const BalLayout L = bal_layout(T, G, Cc);
    if (!aligned256(ws) || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    char *w = static_cast<char *>(ws);
    BalArgs a{};
    a.ids = ids;
    a.T = T; a.E = E; a.G = G; a.Cc = Cc;
    a.rs = rank_score;
    a.target = target;
    a.info = info;
    a.h = reinterpret_cast<BalHeader *>(w + L.hdr);
    a.fl[0] = reinterpret_cast<int *>(w + L.fl0);
    a.fl[1] = reinterpret_cast<int *>(w + L.fl1);
    a.prop_r = reinterpret_cast<int *>(w + L.prop_r);
    a.prop_key = reinterpret_cast<unsigned long long *>(w + L.prop_key);
    a.bucket = reinterpret_cast<unsigned long long *>(w + L.bucket);
    a.hold[0] = reinterpret_cast<unsigned long long *>(w + L.hold0);
    a.hold[1] = reinterpret_cast<unsigned long long *>(w + L.hold1);
    a.err = err;
    if (cudaMemsetAsync(a.h, 0, sizeof(BalHeader), stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (info && cudaMemsetAsync(info, 0, 6 * sizeof(long long), stream) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status st = MOE_ERR_ARG;
    switch (k) {
    case 1: st = launch_balanced<1>(a, stream); break;
    case 2: st = launch_balanced<2>(a, stream); break;
    case 3: st = launch_balanced<3>(a, stream); break;
    case 4: st = launch_balanced<4>(a, stream); break;
    case 5: st = launch_balanced<5>(a, stream); break;
    case 6: st = launch_balanced<6>(a, stream); break;
    case 7: st = launch_balanced<7>(a, stream); break;
    case 8: st = launch_balanced<8>(a, stream); break;
    }
    if (st == MOE_OK) note_launches(1);
    return st;
}

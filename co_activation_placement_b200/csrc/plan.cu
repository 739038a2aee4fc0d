// Deduplicated, rank-major dispatch plan.
//
// "Expert Coupling in MoE Pretraining", abstract: a dispatcher that sends each
// token to each GPU once.  "Cobalt", "Problem Formulation": the cross-node
// cost V = sum_t |{N(r_t^e) : e in D_t} \ {N(s_t)}| under node-level
// deduplication; here r_t^e = p(e) (one replica per expert).
//
// Rows are the pairs (t, r), r in m_t = {p(e) : e in D_t}, ordered by
// (r, s_t, t).  The order is produced without sorting keys:
//   1. (only when source ranks are given) a stable counting sort of the tokens
//      by s_t -> perm; with contiguous shards perm is the identity;
//   2. the token sequence in perm order is cut into chunks of kChunk tokens
//      that never straddle a source shard.  Each chunk's block computes m_t
//      (bitmask of destination ranks), the summary terms and its per-rank row
//      counts;
//   3. each chunk's block sums the counts of the chunks before it and of all
//      chunks per rank (its first row per rank), then ranks its rows per
//      destination, stable in perm order: a warp transposes its 32 x G
//      destination bit matrix with five shuffle stages, so lane d holds the
//      ballot of rank d; a row's rank in the warp is a popcount of that word
//      below the lane, and warps are ordered by a prefix over the block.  It
//      writes row_token, row_jmask and row_of.  One more block of the same
//      launch scans the counts over chunks for the rank segment offsets and
//      counts[s][r] (chunks of one shard are adjacent) and the summary.
// All arithmetic is integer; the result is unique and does not depend on
// scheduling.  No kernel waits on another block.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "waits.cuh"

namespace moe {
namespace {

constexpr int kChunk = 1024;  // tokens per block, one per thread
constexpr int kWarps = kChunk / 32;

struct PlanWsHeader {
    unsigned int done_src;        // blocks finished in plan_src_count
    unsigned int pad[3];
    unsigned long long acc[4];    // R, R_remote, local, V
    GridBarrier bar;              // the single-launch plan's grid barrier
};

struct PlanWs {
    PlanWsHeader *hdr;
    int32_t *soff;       // [G+1] first perm position of each source shard
    int32_t *scnt;       // [G]   tokens per source shard
    int32_t *cpre;       // [G+1] first chunk of each shard; cpre[G] = active chunks
    int32_t *perm;       // [T]
    int32_t *sblk;       // [Bs][G]
    int32_t *sblk_pref;  // [Bs+1][G]
    int32_t *blk;        // [Bc][G]
    int32_t *blk_pref;   // [Bc+1][G]
};

inline int src_blocks(int T) { return (T + kChunk - 1) / kChunk; }
inline int chunk_blocks(int T, int G, bool with_src)
{
    if (with_src) return (T + kChunk - 1) / kChunk + G;
    const int shard = T / G;
    return G * std::max(1, (shard + kChunk - 1) / kChunk);
}

size_t carve(void *ws, int T, int G, bool with_src, PlanWs *out)
{
    char *p = static_cast<char *>(ws);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *q = p ? p + off : nullptr;
        off = round_up(off + bytes, 256);
        return q;
    };
    PlanWs w{};
    w.hdr = reinterpret_cast<PlanWsHeader *>(take(sizeof(PlanWsHeader)));
    w.soff = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (G + 1)));
    w.scnt = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * G));
    w.cpre = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (G + 1)));
    const int Bs = src_blocks(T), Bc = chunk_blocks(T, G, with_src);
    if (with_src) {
        w.perm = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * std::max(T, 1)));
        w.sblk = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * Bs * G));
        w.sblk_pref = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (Bs + 1) * G));
    }
    w.blk = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)Bc * G));
    w.blk_pref = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)(Bc + 1) * G));
    if (out) *out = w;
    return off;
}

template <int K>
__device__ __forceinline__ void load_token(const int32_t *__restrict__ p, int (&v)[K])
{
#pragma unroll
    for (int q = 0; q < K; ++q) v[q] = __ldg(p + q);
}

template <int K>
__device__ __forceinline__ int token_error(const int (&v)[K], int E)
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

__device__ __forceinline__ int clamp_rank(int r, int G, int32_t *err)
{
    if ((unsigned)r >= (unsigned)G) {
        record_error(err, MOE_DERR_RANK_RANGE);
        return 0;
    }
    return r;
}

// Transpose the warp's 32 x 32 bit matrix (lane r holds row r): afterwards
// lane c holds column c, i.e. bit r of lane c's result = bit c of lane r's
// input -- the ballot of bit c, for all 32 c at once (five butterfly stages).
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane)
{
    constexpr uint32_t kMask[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int st = 0; st < 5; ++st) {
        const int j = 16 >> st;
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
        x = (lane & j) ? ((x & ~kMask[st]) | ((y & ~kMask[st]) >> j)) : ((x & kMask[st]) | ((y & kMask[st]) << j));
    }
    return x;
}

// Last block: exclusive scan of a [B][G] column table (rows b, column d) into
// pref[b][d] and tot[d] (shared).  Called by all threads of one block.
__device__ void scan_columns(const int32_t *tab, int32_t *pref, int B, int G, int32_t *tot_sh, int32_t *seg_sh)
{
    const int nseg = blockDim.x / G;   // >= 1 since G <= 64 < blockDim
    const int d = threadIdx.x % G, q = threadIdx.x / G;
    const int per = (B + nseg - 1) / nseg;
    const int b0 = min(B, q * per), b1 = min(B, b0 + per);
    constexpr int kBatch = 8;          // independent L2 loads in flight per thread
    if (q < nseg) {
        int s = 0;
        for (int b = b0; b < b1; b += kBatch) {
            int v[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) v[i] = b + i < b1 ? __ldcg(tab + (size_t)(b + i) * G + d) : 0;
#pragma unroll
            for (int i = 0; i < kBatch; ++i) s += v[i];
        }
        seg_sh[q * G + d] = s;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        int run = 0;
        for (int qq = 0; qq < nseg; ++qq) {
            int v = seg_sh[qq * G + threadIdx.x];
            seg_sh[qq * G + threadIdx.x] = run;
            run += v;
        }
        tot_sh[threadIdx.x] = run;
    }
    __syncthreads();
    if (q < nseg) {
        int run = seg_sh[q * G + d];
        for (int b = b0; b < b1; b += kBatch) {
            int v[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) v[i] = b + i < b1 ? __ldcg(tab + (size_t)(b + i) * G + d) : 0;
#pragma unroll
            for (int i = 0; i < kBatch; ++i)
                if (b + i < b1) {
                    pref[(size_t)(b + i) * G + d] = run;
                    run += v[i];
                }
        }
    }
    if (threadIdx.x < G) pref[(size_t)B * G + threadIdx.x] = tot_sh[threadIdx.x];
    __syncthreads();
}

// ---- step 1: stable counting sort of tokens by source rank ---------------

__global__ void __launch_bounds__(kChunk)
plan_src_count_kernel(const int32_t *__restrict__ src_rank, int T, int G, PlanWs w, int32_t *err)
{
    __shared__ int32_t hist[64];
    __shared__ int32_t tot[64];
    __shared__ int32_t seg[kChunk];
    __shared__ bool last;
    pdl_release();                        // the scatter's prologue reads only src_rank
    if (threadIdx.x < G) hist[threadIdx.x] = 0;
    __syncthreads();
    const int t = blockIdx.x * kChunk + threadIdx.x;
    const int s = t < T ? clamp_rank(__ldg(src_rank + t), G, err) : -1;
    // one add per rank and warp (shuffle targets crowd onto a few ranks)
    const unsigned same = __match_any_sync(0xffffffffu, s);
    if (s >= 0 && (int)(threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[s], __popc(same));
    __syncthreads();
    if (threadIdx.x < G) w.sblk[(size_t)blockIdx.x * G + threadIdx.x] = hist[threadIdx.x];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&w.hdr->done_src, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    scan_columns(w.sblk, w.sblk_pref, gridDim.x, G, tot, seg);
    if (threadIdx.x == 0) {
        int run = 0, ch = 0;
        for (int s = 0; s < G; ++s) {
            w.soff[s] = run;
            w.scnt[s] = tot[s];
            w.cpre[s] = ch;
            run += tot[s];
            ch += (tot[s] + kChunk - 1) / kChunk;
        }
        w.soff[G] = run;
        w.cpre[G] = ch;
        w.hdr->done_src = 0;
    }
}

__global__ void __launch_bounds__(kChunk)
plan_src_scatter_kernel(const int32_t *__restrict__ src_rank, int T, int G, PlanWs w)
{
    __shared__ int32_t wcnt[kWarps][64];
    __shared__ int32_t wbase[kWarps][64];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kWarps * 64; i += kChunk) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * kChunk + threadIdx.x;
    const bool act = t < T;
    int s = act ? __ldg(src_rank + t) : G;       // inactive lanes get key G
    if (act && (unsigned)s >= (unsigned)G) s = 0; // same clamp as the count kernel
    const unsigned peers = __match_any_sync(0xffffffffu, s);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (act && rank == 0) wcnt[wid][s] = __popc(peers);
    __syncthreads();
    if (threadIdx.x < G) {
        int run = 0;
        for (int q = 0; q < kWarps; ++q) {
            wbase[q][threadIdx.x] = run;
            run += wcnt[q][threadIdx.x];
        }
    }
    __syncthreads();
    pdl_wait();                           // the counts and their scan
    pdl_release();
    if (act) {
        const int pos = __ldcg(w.soff + s) + __ldcg(w.sblk_pref + (size_t)blockIdx.x * G + s) + wbase[wid][s] + rank;
        w.perm[pos] = t;
    }
}

// ---- step 2: destination sets, summary terms, per-chunk row counts ---------

struct ChunkRange {
    int s, p0, p1;   // source shard, perm positions [p0, p1)
    bool active;
};

// Shard table of the source-sorted order, staged in shared memory once per
// block (G + 1 entries each) so that locating a chunk costs no global loads.
struct ShardTable {
    int32_t soff[65], scnt[64], cpre[65];
};

__device__ __forceinline__ void load_shards(ShardTable &sh, int G, bool with_src, const PlanWs &w)
{
    if (!with_src) return;
    for (int i = threadIdx.x; i <= G; i += blockDim.x) {
        sh.soff[i] = __ldcg(w.soff + i);
        sh.cpre[i] = __ldcg(w.cpre + i);
        if (i < G) sh.scnt[i] = __ldcg(w.scnt + i);
    }
}

// Chunk b of the token sequence (call after load_shards and a barrier).
__device__ __forceinline__ ChunkRange chunk_range(int b, int T, int G, bool with_src, const ShardTable &sh)
{
    ChunkRange c;
    if (with_src) {
        if (b >= sh.cpre[G]) { c.active = false; c.s = 0; c.p0 = c.p1 = 0; return c; }
        int lo = 0, hi = G - 1;   // last shard s with cpre[s] <= b
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sh.cpre[mid] <= b) lo = mid; else hi = mid - 1;
        }
        const int s = lo;
        c.s = s;
        c.p0 = sh.soff[s] + (b - sh.cpre[s]) * kChunk;
        c.p1 = min(sh.soff[s] + sh.scnt[s], c.p0 + kChunk);
        c.active = true;
    } else {
        const int shard = T / G;
        const int nch = max(1, (shard + kChunk - 1) / kChunk);
        c.s = b / nch;
        c.p0 = c.s * shard + (b % nch) * kChunk;
        c.p1 = min((c.s + 1) * shard, c.p0 + kChunk);
        c.active = true;
    }
    return c;
}

// Serving rank of each of a token's K picks: p(e) from the placement, or,
// with PICKS, the per-(token, pick) ranks of a replica assignment.  Returns a
// device error code (0 when the ranks are usable).
template <int K, bool PICKS>
__device__ __forceinline__ int serving_ranks(const int (&v)[K], const int32_t *e2r_sh,
                                             const int32_t *__restrict__ picks, int t, int G, int (&r)[K])
{
    int bad = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if constexpr (PICKS) {
            r[j] = __ldg(picks + (size_t)t * K + j);
            if ((unsigned)r[j] >= (unsigned)G) {
                bad = MOE_DERR_RANK_RANGE;
                r[j] = 0;
            }
        } else {
            r[j] = e2r_sh[v[j]];
        }
    }
    return bad;
}

template <int K, bool PICKS>
__global__ void __launch_bounds__(kChunk, 2)
plan_count_kernel(const int32_t *__restrict__ ids, int T, int E, int G, int rpn,
                  const int32_t *__restrict__ e2r_g, const int32_t *__restrict__ picks, bool with_src, PlanWs w,
                  moe_plan P, int32_t *err)
{
    extern __shared__ int32_t e2r[];           // [E] (unused with PICKS)
    __shared__ int32_t cnt[64];
    __shared__ unsigned long long red[4][kWarps];
    __shared__ ShardTable sh;
    __shared__ int32_t node_s[64];              // node of each rank (no division per pick)
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (!PICKS)
        for (int e = threadIdx.x; e < E; e += kChunk) e2r[e] = clamp_rank(__ldg(e2r_g + e), G, err);
    if (threadIdx.x < 64) {
        cnt[threadIdx.x] = 0;
        node_s[threadIdx.x] = threadIdx.x / rpn;
    }
    load_shards(sh, G, with_src, w);      // from the source count, two launches back: complete
    __syncthreads();
    pdl_wait();                           // the source permutation
    pdl_release();

    const ChunkRange c = chunk_range(blockIdx.x, T, G, with_src, sh);
    uint32_t my[4] = {0, 0, 0, 0};             // per token at most 64: warp sums fit 32 bits
    const int p = c.p0 + threadIdx.x;
    unsigned long long m = 0;
    if (c.active && p < c.p1) {
        const int t = with_src ? __ldcg(w.perm + p) : p;
        int v[K], rk[K];
        load_token<K>(ids + (size_t)t * K, v);
        int bad = token_error<K>(v, E);
        if (!bad) bad = serving_ranks<K, PICKS>(v, e2r, picks, t, G, rk);
        unsigned long long nodes = 0;
        if (bad) {
            record_error(err, bad);
        } else {
            int local = 0;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const int r = rk[j];
                m |= 1ull << r;
                nodes |= 1ull << node_s[r];
                local += r == c.s;
            }
            my[0] = __popcll(m);
            my[1] = __popcll(m & ~(1ull << c.s));
            my[2] = local;
            my[3] = __popcll(nodes & ~(1ull << node_s[c.s]));
        }
        P.dest_mask[t] = m;
    }
    {   // rows per rank: lane d counts column d (and d+32) of the warp's destination bits
        const uint32_t clo = warp_transpose32((uint32_t)m, lane);
        const uint32_t chi = warp_transpose32((uint32_t)(m >> 32), lane);
        if (lane < G && clo) atomicAdd(&cnt[lane], __popc(clo));
        if (lane + 32 < G && chi) atomicAdd(&cnt[lane + 32], __popc(chi));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t x = __reduce_add_sync(0xffffffffu, my[i]);
        if (lane == 0) red[i][wid] = x;
    }
    __syncthreads();
    if (threadIdx.x < 4) {
        unsigned long long x = 0;
        for (int q = 0; q < kWarps; ++q) x += red[threadIdx.x][q];
        if (x) atomicAdd(&w.hdr->acc[threadIdx.x], x);
    }
    if (threadIdx.x < G) w.blk[(size_t)blockIdx.x * G + threadIdx.x] = cnt[threadIdx.x];
}

// ---- step 3: stable per-destination ranks and row writes -----------------

// The first row of chunk b for every rank, base[d] (shared): the rows of
// ranks below d, then those of rank d in chunks before b -- both column sums
// of the [B][G] per-chunk counts, taken in one pass by the whole block
// (thread (q, d) sums rows q, q + nseg, ... of column d).  Ends with a
// barrier.
__device__ __forceinline__ void chunk_bases(const int32_t *blk, int B, int b, int G, int32_t *base, int32_t *ptot,
                                            int32_t *pbef)
{
    const int nseg = blockDim.x / G, d = threadIdx.x % G, q = threadIdx.x / G;
    if (q < nseg) {
        int tot = 0, bef = 0;
        constexpr int kBatch = 8;             // independent L2 loads in flight per thread
        for (int r0 = q; r0 < B; r0 += kBatch * nseg) {
            int v[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                const int row = r0 + i * nseg;
                v[i] = row < B ? __ldcg(blk + (size_t)row * G + d) : 0;
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                tot += v[i];
                if (r0 + i * nseg < b) bef += v[i];
            }
        }
        ptot[q * G + d] = tot;
        pbef[q * G + d] = bef;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        // exclusive prefix over ranks of the totals, plus the rows before b
        const int lane = threadIdx.x;
        int t0 = 0, t1 = 0, b0 = 0, b1 = 0;
        for (int qq = 0; qq < nseg; ++qq) {
            if (lane < G) { t0 += ptot[qq * G + lane]; b0 += pbef[qq * G + lane]; }
            if (lane + 32 < G) { t1 += ptot[qq * G + lane + 32]; b1 += pbef[qq * G + lane + 32]; }
        }
        int s0 = t0, s1 = t1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(0xffffffffu, s0, o);
            const int y1 = __shfl_up_sync(0xffffffffu, s1, o);
            if (lane >= o) { s0 += y0; s1 += y1; }
        }
        const int all0 = __shfl_sync(0xffffffffu, s0, 31);
        if (lane < G) base[lane] = s0 - t0 + b0;
        if (lane + 32 < G) base[lane + 32] = all0 + s1 - t1 + b1;
    }
    __syncthreads();
}

// The plan's tables from the per-chunk counts (one block, beside the row
// writes of the others): the exclusive scan of the counts over chunks per
// rank, the rank segments, offsets[d][s] (first row of shard s in rank d's
// segment), counts[s][d], offsets[G*G] = R and the summary.
template <int K>
__device__ void write_tables(int B, int G, bool with_src, const ShardTable &sh, const PlanWs &w, const moe_plan &P,
                             int T, int32_t *tot, int32_t *seg)
{
    scan_columns(w.blk, w.blk_pref, B, G, tot, seg);
    if (threadIdx.x == 0) {
        int run = 0;
        for (int d = 0; d < G; ++d) { seg[d] = run; run += tot[d]; }   // seg[d] = first row of rank d
        P.offsets[G * G] = run;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * G; i += blockDim.x) {
        const int d = i / G, s = i % G;   // offsets in (d, s) order
        int b0, b1;
        if (with_src) { b0 = sh.cpre[s]; b1 = sh.cpre[s + 1]; }
        else { const int nch = B / G; b0 = s * nch; b1 = b0 + nch; }
        const int a0 = __ldcg(w.blk_pref + (size_t)b0 * G + d);
        const int a1 = __ldcg(w.blk_pref + (size_t)b1 * G + d);
        P.offsets[d * G + s] = seg[d] + a0;
        P.counts[s * G + d] = a1 - a0;
    }
    if (threadIdx.x < 4) P.summary[threadIdx.x] = (int64_t)__ldcg(&w.hdr->acc[threadIdx.x]);
    if (threadIdx.x == 4) P.summary[4] = (int64_t)T * K;
}

// A token's row_of entries (K ints) as whole vectors where the alignment
// allows: one 16-byte store per 4 picks, else 8-byte, else 4-byte.
template <int K>
__device__ __forceinline__ void store_row_of(int32_t *dst, const int (&x)[K], bool vec_ok)
{
    if constexpr (K % 4 == 0) {
        if (vec_ok) {
#pragma unroll
            for (int q = 0; q < K / 4; ++q)
                reinterpret_cast<int4 *>(dst)[q] = make_int4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            return;
        }
    } else if constexpr (K % 2 == 0) {
        if (vec_ok) {
#pragma unroll
            for (int q = 0; q < K / 2; ++q) reinterpret_cast<int2 *>(dst)[q] = make_int2(x[2 * q], x[2 * q + 1]);
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < K; ++j) dst[j] = x[j];
}

// The rows of one chunk.  On entry (after a block barrier): thread i holds
// its token t (act: a position of the chunk), destination set m (0 for an
// invalid token, whose row_of becomes -1) and serving ranks r; wcnt[w][d] is
// the exclusive prefix over the block's warps of the rows for rank d,
// colw[w][d] the lanes of warp w with a row for d, bcnt[d] the chunk's rows
// for d and base[d] the chunk's first row of rank d.  A row's place in its
// rank's run is its warp's prefix plus the earlier lanes of the warp that
// have that rank (stable in token order).  The chunk's rows of rank d fill
// one run [base[d], base[d] + bcnt[d]) of the output, so they are staged in
// shared memory in (d, token order) -- thread, pick mask and rank packed in
// one word -- and copied out with consecutive threads on consecutive rows;
// row_of goes out per token in whole vectors.
template <int K>
__device__ __forceinline__ void write_chunk_rows(int t, bool act, unsigned long long m, const int (&r)[K], int G,
                                                 const int32_t *base, const int32_t *bcnt, int32_t (*wcnt)[64],
                                                 uint32_t (*colw)[64], int32_t *boff, int32_t *tok_s,
                                                 uint32_t *rows_s, const moe_plan &P)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid < 32) {   // boff[d]: the chunk's rows of ranks below d
        const int c0 = lane < G ? bcnt[lane] : 0, c1 = lane + 32 < G ? bcnt[lane + 32] : 0;
        int s0 = c0, s1 = c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v0 = __shfl_up_sync(0xffffffffu, s0, o);
            const int v1 = __shfl_up_sync(0xffffffffu, s1, o);
            if (lane >= o) { s0 += v0; s1 += v1; }
        }
        const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
        boff[lane] = s0 - c0;
        boff[lane + 32] = tot0 + s1 - c1;
        if (lane == 31) boff[64] = tot0 + s1;
    }
    tok_s[tid] = t;
    __syncthreads();
    int rowj[K];
#pragma unroll
    for (int j = 0; j < K; ++j) rowj[j] = -1;
    const unsigned lt = (1u << lane) - 1u;
    for (unsigned long long q = m; q; q &= q - 1) {
        const int d = __ffsll((long long)q) - 1;
        const int within = wcnt[wid][d] + __popc(colw[wid][d] & lt);
        unsigned jm = 0;
#pragma unroll
        for (int j = 0; j < K; ++j)
            if (r[j] == d) {
                jm |= 1u << j;
                rowj[j] = base[d] + within;
            }
        rows_s[boff[d] + within] = ((uint32_t)tid << 14) | (jm << 6) | (uint32_t)d;
    }
    if (act) {
        const bool vec_ok = (reinterpret_cast<uintptr_t>(P.row_of) & (K % 4 == 0 ? 15 : 7)) == 0;
        store_row_of<K>(P.row_of + (size_t)t * K, rowj, vec_ok);
    }
    __syncthreads();
    const int n = boff[64];
    for (int i = tid; i < n; i += blockDim.x) {
        const uint32_t v = rows_s[i];
        const int d = (int)(v & 63u);
        const int pos = base[d] + (i - boff[d]);
        P.row_token[pos] = tok_s[v >> 14];
        P.row_jmask[pos] = (uint8_t)((v >> 6) & 255u);
    }
}

template <int K, bool PICKS>
__global__ void __launch_bounds__(kChunk, 2)
plan_scatter_kernel(const int32_t *__restrict__ ids, int T, int E, int G,
                    const int32_t *__restrict__ e2r_g, const int32_t *__restrict__ picks, bool with_src, PlanWs w,
                    moe_plan P)
{
    extern __shared__ int32_t e2r[];           // [E] (unused with PICKS), then the staged rows
    uint32_t *rows_s = reinterpret_cast<uint32_t *>(e2r + (PICKS ? 0 : E));   // [kChunk * K]
    __shared__ int32_t base[64];               // first row of this chunk per rank
    __shared__ int32_t bcnt[64], boff[65];     // the chunk's rows per rank and their exclusive prefix
    __shared__ int32_t tok_s[kChunk];
    __shared__ int32_t wcnt[kWarps][64];       // rows per (warp, rank), then their exclusive prefix
    __shared__ uint32_t colw[kWarps][64];      // lanes of the warp with a row for the rank
    __shared__ int32_t part[2][kChunk];        // column sums: per (segment, rank) partials
    __shared__ ShardTable sh;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    // prologue, before the counts are complete: the shard table and the
    // source permutation (written two and more launches back), the tokens'
    // destination sets and their per-warp ranks
    load_shards(sh, G, with_src, w);
    __syncthreads();
    const int B = gridDim.x - 1;               // chunks; the last block writes the tables
    if (blockIdx.x == B) {
        pdl_wait();
        write_tables<K>(B, G, with_src, sh, w, P, T, &part[0][0], &part[1][0]);
        return;
    }
    const ChunkRange c = chunk_range(blockIdx.x, T, G, with_src, sh);
    if (!c.active) {
        pdl_wait();
        return;
    }
    if (!PICKS)
        for (int e = threadIdx.x; e < E; e += kChunk) {
            const int r = __ldg(e2r_g + e);
            e2r[e] = (unsigned)r >= (unsigned)G ? 0 : r;
        }
    __syncthreads();

    const int p = c.p0 + threadIdx.x;
    const bool act = p < c.p1;
    int t = 0, v[K], r[K];
    unsigned long long m = 0;             // stays 0 for an invalid token: its row_of is all -1
    if (act) {
        t = with_src ? __ldcg(w.perm + p) : p;
        load_token<K>(ids + (size_t)t * K, v);
        if (token_error<K>(v, E) == 0 && serving_ranks<K, PICKS>(v, e2r, picks, t, G, r) == 0) {
#pragma unroll
            for (int j = 0; j < K; ++j) m |= 1ull << r[j];
        }
    }
    // column d of the warp's 32 x G destination bit matrix: which lanes send to rank d
    const uint32_t clo = warp_transpose32((uint32_t)m, lane);
    const uint32_t chi = warp_transpose32((uint32_t)(m >> 32), lane);
    if (lane < G) {
        colw[wid][lane] = clo;
        wcnt[wid][lane] = __popc(clo);
    }
    if (lane + 32 < G) {
        colw[wid][lane + 32] = chi;
        wcnt[wid][lane + 32] = __popc(chi);
    }
    __syncthreads();
    if (threadIdx.x < G) {
        int run = 0;
        for (int q = 0; q < kWarps; ++q) {
            const int x = wcnt[q][threadIdx.x];
            wcnt[q][threadIdx.x] = run;
            run += x;
        }
        bcnt[threadIdx.x] = run;
    }
    // the picks' ranks (< 64) as bytes while the bases are summed: fewer
    // registers live across that pass
    uint32_t rpk[(K + 3) / 4];
#pragma unroll
    for (int q = 0; q < (K + 3) / 4; ++q) rpk[q] = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) rpk[j / 4] |= (m ? (uint32_t)r[j] & 255u : 0u) << (8 * (j % 4));
    pdl_wait();                           // the per-chunk counts
    chunk_bases(w.blk, B, blockIdx.x, G, base, &part[0][0], &part[1][0]);
#pragma unroll
    for (int j = 0; j < K; ++j) r[j] = (int)((rpk[j / 4] >> (8 * (j % 4))) & 255u);
    write_chunk_rows<K>(t, act, m, r, G, base, bcnt, wcnt, colw, boff, tok_s, rows_s, P);
}

// ---- the whole plan in one cooperative launch ------------------------------
//
// The same three steps in one kernel, the cross-block scans replaced by grid
// barriers: every block derives the shard table and the per-rank totals from
// the per-chunk counts itself (a column sum over the chunks), so no single
// block's serial tail sits on the critical path.  Blocks loop over chunks
// when there are more chunks than co-resident blocks.  Used when the caller
// selects it (moe_plan_dispatch_method) and the chunk count is small enough
// for the column sums to stay cheap.

constexpr int kFusedMaxChunks = 512;

struct FusedArgs {
    const int32_t *ids;
    int T, E, G, rpn;
    const int32_t *e2r_g, *picks, *src;
    PlanWs w;
    moe_plan P;
    int32_t *err;
    int Bs;               // source-count chunks (with source ranks)
};

// sum over rows b < B of tab[b][d] for d < G, into out[d] (shared); all
// threads of the block; part: blockDim.x ints of shared scratch
__device__ __forceinline__ void column_sums(const int32_t *tab, int B, int G, int32_t *out, int32_t *part)
{
    const int nseg = blockDim.x / G, d = threadIdx.x % G, q = threadIdx.x / G;
    if (q < nseg) {
        int s = 0;
        for (int b = q; b < B; b += nseg) s += __ldcg(tab + (size_t)b * G + d);
        part[q * G + d] = s;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        int x = 0;
        for (int qq = 0; qq < nseg; ++qq) x += part[qq * G + threadIdx.x];
        out[threadIdx.x] = x;
    }
    __syncthreads();
}

template <int K, bool PICKS>
__global__ void __launch_bounds__(kChunk, 1)
plan_fused_kernel(FusedArgs a)
{
    extern __shared__ int32_t e2r[];           // [E] (unused with PICKS), then the staged rows
    uint32_t *rows_s = reinterpret_cast<uint32_t *>(e2r + (PICKS ? 0 : a.E));   // [kChunk * K]
    __shared__ int32_t cnt[64], base[64], tot[64], seg[64];
    __shared__ int32_t bcnt[64], boff[65];
    __shared__ int32_t tok_s[kChunk];
    __shared__ int32_t node_s[64];             // node of each rank (no division per pick)
    __shared__ int32_t part[kChunk];
    __shared__ int32_t wcnt[kWarps][64];       // rows per (warp, rank), then their exclusive prefix
    __shared__ uint32_t colw[kWarps][64];      // lanes of the warp with a row for the rank
    __shared__ unsigned long long red[4][kWarps];
    __shared__ ShardTable sh;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int T = a.T, E = a.E, G = a.G;
    const bool with_src = a.src != nullptr;
    GridBarrier *bar = &a.w.hdr->bar;
    if (!PICKS)
        for (int e = tid; e < E; e += kChunk) e2r[e] = clamp_rank(__ldg(a.e2r_g + e), G, a.err);
    if (tid < 64) node_s[tid] = tid / a.rpn;

    // ---- step 1 (source ranks given): counting sort of the tokens by s_t
    if (with_src) {
        for (int b = blockIdx.x; b < a.Bs; b += gridDim.x) {
            if (tid < 64) cnt[tid] = 0;
            __syncthreads();
            const int t = b * kChunk + tid;
            if (t < T) atomicAdd(&cnt[clamp_rank(__ldg(a.src + t), G, a.err)], 1);
            __syncthreads();
            if (tid < G) a.w.sblk[(size_t)b * G + tid] = cnt[tid];
            __syncthreads();
        }
        if (!grid_barrier(bar, a.err)) return;
        column_sums(a.w.sblk, a.Bs, G, tot, part);
        if (tid == 0) {
            int run = 0, ch = 0;
            for (int s = 0; s < G; ++s) {
                sh.soff[s] = run;
                sh.scnt[s] = tot[s];
                sh.cpre[s] = ch;
                run += tot[s];
                ch += (tot[s] + kChunk - 1) / kChunk;
            }
            sh.soff[G] = run;
            sh.cpre[G] = ch;
        }
        __syncthreads();
        for (int b = blockIdx.x; b < a.Bs; b += gridDim.x) {
            column_sums(a.w.sblk, b, G, base, part);      // tokens of each shard in earlier chunks
            for (int i = tid; i < kWarps * 64; i += kChunk) (&wcnt[0][0])[i] = 0;
            __syncthreads();
            const int t = b * kChunk + tid;
            const bool act = t < T;
            int s = act ? __ldg(a.src + t) : G;
            if (act && (unsigned)s >= (unsigned)G) s = 0;
            const unsigned peers = __match_any_sync(0xffffffffu, s);
            const int rk = __popc(peers & ((1u << lane) - 1u));
            if (act && rk == 0) wcnt[wid][s] = __popc(peers);
            __syncthreads();
            if (tid < G) {
                int run = 0;
                for (int q = 0; q < kWarps; ++q) {
                    const int x = wcnt[q][tid];
                    wcnt[q][tid] = run;
                    run += x;
                }
            }
            __syncthreads();
            if (act) a.w.perm[sh.soff[s] + base[s] + wcnt[wid][s] + rk] = t;
            __syncthreads();
        }
        if (!grid_barrier(bar, a.err)) return;
    }
    const int shard = with_src ? 0 : T / G;
    const int nch = with_src ? 0 : max(1, (shard + kChunk - 1) / kChunk);
    const int B = with_src ? sh.cpre[G] : G * nch;

    // ---- step 2: destination sets, summary terms, per-chunk row counts
    unsigned long long my[4] = {0, 0, 0, 0};
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        if (tid < 64) cnt[tid] = 0;
        __syncthreads();
        const ChunkRange c = chunk_range(b, T, G, with_src, sh);
        const int p = c.p0 + tid;
        unsigned long long m = 0;
        if (p < c.p1) {
            const int t = with_src ? __ldcg(a.w.perm + p) : p;
            int v[K], rk[K];
            load_token<K>(a.ids + (size_t)t * K, v);
            int bad = token_error<K>(v, E);
            if (!bad) bad = serving_ranks<K, PICKS>(v, e2r, a.picks, t, G, rk);
            if (bad) {
                record_error(a.err, bad);
            } else {
                unsigned long long nodes = 0;
                int local = 0;
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int r = rk[j];
                    m |= 1ull << r;
                    nodes |= 1ull << node_s[r];
                    local += r == c.s;
                }
                my[0] += __popcll(m);
                my[1] += __popcll(m & ~(1ull << c.s));
                my[2] += local;
                my[3] += __popcll(nodes & ~(1ull << node_s[c.s]));
            }
            a.P.dest_mask[t] = m;
        }
        const uint32_t clo = warp_transpose32((uint32_t)m, lane);
        const uint32_t chi = warp_transpose32((uint32_t)(m >> 32), lane);
        if (lane < G && clo) atomicAdd(&cnt[lane], __popc(clo));
        if (lane + 32 < G && chi) atomicAdd(&cnt[lane + 32], __popc(chi));
        __syncthreads();
        if (tid < G) a.w.blk[(size_t)b * G + tid] = cnt[tid];
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        unsigned long long x = my[i];
        for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) red[i][wid] = x;
    }
    __syncthreads();
    if (tid < 4) {
        unsigned long long x = 0;
        for (int q = 0; q < kWarps; ++q) x += red[tid][q];
        if (x) atomicAdd(&a.w.hdr->acc[tid], x);
    }
    if (!grid_barrier(bar, a.err)) return;

    // ---- step 3: rank segments, then every chunk's rows
    column_sums(a.w.blk, B, G, tot, part);
    if (tid == 0) {
        int run = 0;
        for (int d = 0; d < G; ++d) { seg[d] = run; run += tot[d]; }
        if (blockIdx.x == 0) a.P.offsets[G * G] = run;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        // offsets in (d, s) order and counts[s][d]: running sums over the
        // chunks of each rank's column, read at the shards' chunk boundaries
        if (tid < G) {
            const int d = tid;
            int run = 0, b = 0;
            for (int s = 0; s < G; ++s) {
                const int b1 = with_src ? sh.cpre[s + 1] : (s + 1) * nch;
                const int at = run;
                for (; b < b1; ++b) run += __ldcg(a.w.blk + (size_t)b * G + d);
                a.P.offsets[d * G + s] = seg[d] + at;
                a.P.counts[s * G + d] = run - at;
            }
        }
        if (tid < 4) a.P.summary[tid] = (int64_t)__ldcg(&a.w.hdr->acc[tid]);
        if (tid == 4) a.P.summary[4] = (int64_t)T * K;
    }
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        column_sums(a.w.blk, b, G, base, part);       // rows of each rank in earlier chunks
        if (tid < G) base[tid] += seg[tid];
        const ChunkRange c = chunk_range(b, T, G, with_src, sh);
        const int p = c.p0 + tid;
        const bool act = p < c.p1;
        int t = 0, v[K], r[K];
        unsigned long long m = 0;
        if (act) {
            t = with_src ? __ldcg(a.w.perm + p) : p;
            load_token<K>(a.ids + (size_t)t * K, v);
            if (token_error<K>(v, E) == 0 && serving_ranks<K, PICKS>(v, e2r, a.picks, t, G, r) == 0) {
#pragma unroll
                for (int j = 0; j < K; ++j) m |= 1ull << r[j];
            }
        }
        const uint32_t clo = warp_transpose32((uint32_t)m, lane);
        const uint32_t chi = warp_transpose32((uint32_t)(m >> 32), lane);
        if (lane < G) {
            colw[wid][lane] = clo;
            wcnt[wid][lane] = __popc(clo);
        }
        if (lane + 32 < G) {
            colw[wid][lane + 32] = chi;
            wcnt[wid][lane + 32] = __popc(chi);
        }
        __syncthreads();
        if (tid < G) {
            int run = 0;
            for (int q = 0; q < kWarps; ++q) {
                const int x = wcnt[q][tid];
                wcnt[q][tid] = run;
                run += x;
            }
            bcnt[tid] = run;
        }
        __syncthreads();
        write_chunk_rows<K>(t, act, m, r, G, base, bcnt, wcnt, colw, boff, tok_s, rows_s, a.P);
        __syncthreads();
    }
}

// The single-launch plan when the shape allows it; MOE_ERR_UNSUPPORTED
// otherwise (the caller then runs the separate kernels).
template <int K, bool PICKS>
moe_status launch_plan_fused(const int32_t *ids, int T, int E, int G, int rpn, const int32_t *e2r,
                             const int32_t *picks, const int32_t *src_rank, const moe_plan &P, int32_t *err,
                             const PlanWs &w, cudaStream_t s)
{
    const bool with_src = src_rank != nullptr;
    const int Bs = with_src ? src_blocks(T) : 0;
    const int Bc = chunk_blocks(T, G, with_src);
    if (Bc > kFusedMaxChunks || Bs > kFusedMaxChunks) return MOE_ERR_UNSUPPORTED;
    auto kern = plan_fused_kernel<K, PICKS>;
    const size_t smem = sizeof(int32_t) * ((PICKS ? 0 : (size_t)E) + (size_t)kChunk * K);
    if (allow_smem(kern, smem) != cudaSuccess) return MOE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kChunk, smem) != cudaSuccess) return MOE_ERR_CUDA;
    if (per_sm < 1) return MOE_ERR_UNSUPPORTED;
    FusedArgs a{};
    a.ids = ids; a.T = T; a.E = E; a.G = G; a.rpn = rpn;
    a.e2r_g = e2r; a.picks = picks; a.src = src_rank;
    a.w = w; a.P = P; a.err = err; a.Bs = Bs;
    const int grid = std::min(std::max(Bc, Bs), sm_count() * per_sm);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kChunk);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

// 0: separate kernels (they run beside other kernels without waiting on one
// another); 1: one cooperative launch when the chunk count allows
std::atomic<int> g_plan_method{0};

// Step 1 alone: the tokens' stable order by source rank, into the workspace.
// The first kernel starts after everything before it on the stream; the
// second may start early and waits inside for the first's counts.
moe_status launch_sources(const int32_t *src_rank, int T, int G, int32_t *err, const PlanWs &w, cudaStream_t s)
{
    const int Bs = src_blocks(T);
    plan_src_count_kernel<<<Bs, kChunk, 0, s>>>(src_rank, T, G, w, err);
    if (launch_pdl(plan_src_scatter_kernel, dim3(Bs), dim3(kChunk), 0, s, src_rank, T, G, w) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_status();
}

template <int K, bool PICKS>
moe_status launch_plan(const int32_t *ids, int T, int E, int G, int rpn, const int32_t *e2r, const int32_t *picks,
                       const int32_t *src_rank, bool presorted, const moe_plan &P, int32_t *err, const PlanWs &w,
                       cudaStream_t s)
{
    if (g_plan_method.load() == 1 && !presorted) {
        const moe_status fs = launch_plan_fused<K, PICKS>(ids, T, E, G, rpn, e2r, picks, src_rank, P, err, w, s);
        if (fs != MOE_ERR_UNSUPPORTED) return fs;
    }
    const bool with_src = src_rank != nullptr;
    const size_t smem = PICKS ? 0 : sizeof(int32_t) * (size_t)E;
    int launched = 0;
    // the first kernel starts after everything before the call; each later
    // one may start early (programmatic dependent launch) and waits inside
    // for its predecessor before reading what that one writes
    if (with_src && !presorted) {
        if (launch_sources(src_rank, T, G, err, w, s) != MOE_OK) return MOE_ERR_CUDA;
        launched += 2;
    }
    const int Bc = chunk_blocks(T, G, with_src);
    const size_t smem_sc = smem + sizeof(int32_t) * (size_t)kChunk * K;     // plus the staged rows
    if (allow_smem(plan_count_kernel<K, PICKS>, smem) != cudaSuccess) return MOE_ERR_CUDA;
    if (allow_smem(plan_scatter_kernel<K, PICKS>, smem_sc) != cudaSuccess) return MOE_ERR_CUDA;
    if (with_src && !presorted) {
        if (launch_pdl(plan_count_kernel<K, PICKS>, dim3(Bc), dim3(kChunk), smem, s, ids, T, E, G, rpn, e2r, picks,
                       with_src, w, P, err) != cudaSuccess)
            return MOE_ERR_CUDA;
    } else {
        plan_count_kernel<K, PICKS><<<Bc, kChunk, smem, s>>>(ids, T, E, G, rpn, e2r, picks, with_src, w, P, err);
    }
    if (launch_pdl(plan_scatter_kernel<K, PICKS>, dim3(Bc + 1), dim3(kChunk), smem_sc, s, ids, T, E, G, e2r, picks,
                   with_src, w, P) != cudaSuccess)
        return MOE_ERR_CUDA;
    launched += 2;
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(launched);
    return st;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_plan_dispatch_method(int method)
{
    if (method < 0 || method > 1) return -1;
    return g_plan_method.exchange(method);
}

extern "C" size_t moe_plan_dispatch_workspace(int T, int k, int G, int with_src_rank)
{
    (void)k;
    if (T < 0 || G < 1 || G > 64) return 0;
    return carve(nullptr, T, G, with_src_rank != 0, nullptr) + 256;
}

namespace {

moe_status plan_entry(const int32_t *ids, int T, int k, int E, int G, int rpn, const int32_t *expert_to_rank,
                      const int32_t *pick_rank, const int32_t *src_rank, bool presorted, const moe_plan *plan,
                      int32_t *err, void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (presorted && !src_rank) return MOE_ERR_ARG;
    if (T < 0 || k < 1 || k > 8 || E < k || G < 1 || G > 64 || rpn < 1 || G % rpn != 0) return MOE_ERR_ARG;
    if ((long long)T * k >= (1ll << 31)) return MOE_ERR_ARG;
    if (E > 12 * 1024) return MOE_ERR_UNSUPPORTED;
    if (!plan || !err || (!expert_to_rank && !pick_rank)) return MOE_ERR_ARG;
    if (!plan->counts || !plan->offsets || !plan->summary) return MOE_ERR_ARG;
    if (T > 0 && (!ids || !plan->dest_mask || !plan->row_token || !plan->row_jmask || !plan->row_of))
        return MOE_ERR_ARG;
    if (!src_rank && T % G != 0) return MOE_ERR_ARG;
    if (T == 0) {
        if (cudaMemsetAsync(plan->counts, 0, sizeof(int32_t) * G * G, stream) != cudaSuccess ||
            cudaMemsetAsync(plan->offsets, 0, sizeof(int32_t) * (G * G + 1), stream) != cudaSuccess ||
            cudaMemsetAsync(plan->summary, 0, sizeof(int64_t) * 5, stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    PlanWs w;
    const size_t need = carve(ws, T, G, src_rank != nullptr, &w);
    if (!ws || !aligned256(ws) || ws_bytes < need) return MOE_ERR_WORKSPACE;
    // (a presorted plan keeps the source order moe_plan_sources left in the
    // workspace; only the header's counters are reset)
    if (cudaMemsetAsync(w.hdr, 0, sizeof(PlanWsHeader), stream) != cudaSuccess) return MOE_ERR_CUDA;
    const int32_t *e2r = expert_to_rank;
    const int32_t *pk = pick_rank;
#define MOE_PLAN_CASE(KK)                                                                                  \
    case KK:                                                                                               \
        return pk ? launch_plan<KK, true>(ids, T, E, G, rpn, e2r, pk, src_rank, presorted, *plan, err, w,   \
                                          stream)                                                          \
                  : launch_plan<KK, false>(ids, T, E, G, rpn, e2r, pk, src_rank, presorted, *plan, err, w,  \
                                           stream);
    switch (k) {
        MOE_PLAN_CASE(1)
        MOE_PLAN_CASE(2)
        MOE_PLAN_CASE(3)
        MOE_PLAN_CASE(4)
        MOE_PLAN_CASE(5)
        MOE_PLAN_CASE(6)
        MOE_PLAN_CASE(7)
        MOE_PLAN_CASE(8)
    }
#undef MOE_PLAN_CASE
    return MOE_ERR_ARG;
}

}  // namespace

extern "C" moe_status moe_plan_dispatch(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                        const int32_t *expert_to_rank, const int32_t *src_rank,
                                        const moe_plan *plan, int32_t *err,
                                        void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (!expert_to_rank) return MOE_ERR_ARG;
    return plan_entry(ids, T, k, E, G, rpn, expert_to_rank, nullptr, src_rank, false, plan, err, ws, ws_bytes,
                      stream);
}

extern "C" moe_status moe_plan_sources(const int32_t *src_rank, int T, int G, int32_t *err, void *ws,
                                       size_t ws_bytes, cudaStream_t stream)
{
    if (T < 0 || G < 1 || G > 64 || !err) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!src_rank) return MOE_ERR_ARG;
    PlanWs w;
    const size_t need = carve(ws, T, G, true, &w);
    if (!ws || !aligned256(ws) || ws_bytes < need) return MOE_ERR_WORKSPACE;
    if (cudaMemsetAsync(w.hdr, 0, sizeof(PlanWsHeader), stream) != cudaSuccess) return MOE_ERR_CUDA;
    const moe_status st = launch_sources(src_rank, T, G, err, w, stream);
    if (st == MOE_OK) note_launches(2);
    return st;
}

extern "C" moe_status moe_plan_dispatch_presorted(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                                  const int32_t *expert_to_rank, const int32_t *src_rank,
                                                  const moe_plan *plan, int32_t *err,
                                                  void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (!expert_to_rank) return MOE_ERR_ARG;
    return plan_entry(ids, T, k, E, G, rpn, expert_to_rank, nullptr, src_rank, true, plan, err, ws, ws_bytes,
                      stream);
}

extern "C" moe_status moe_plan_dispatch_ranks(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                              const int32_t *pick_rank, const int32_t *src_rank,
                                              const moe_plan *plan, int32_t *err,
                                              void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (!pick_rank) return MOE_ERR_ARG;
    return plan_entry(ids, T, k, E, G, rpn, nullptr, pick_rank, src_rank, false, plan, err, ws, ws_bytes, stream);
}

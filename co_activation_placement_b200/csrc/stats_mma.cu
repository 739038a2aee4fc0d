// Co-activation and transition counts on the tensor cores (tcgen05, sm_100a).
//
// "Expert Coupling in MoE Pretraining", abstract, and "Cobalt", "Key
// Observation": C_l[i][j] counts the tokens that select experts i and j at
// layer l, M_l[i][j] the tokens that select i at layer l and j at layer l+1.
// With X_l the E x T one-hot matrix (X_l[e][t] = 1 iff token t selects e at
// layer l) these are the products
//     C_l = X_l X_l^T,     M_l = X_l X_{l+1}^T,
// an exact integer contraction over tokens.  Each thread block owns one job
// (C_l, M_l, or both from one tile of X_l; with E <= 128 both products of two
// consecutive layers, see coact_quad_kernel) and one token slice.  Per stage of
// 128 tokens eight builder warps write the stage's X tiles into shared
// memory and arrive on its "full" mbarrier; a ninth warp waits on it, issues
// tcgen05.mma kind::i8 (u8 x u8 -> s32, M = 128, K = 32 per instruction)
// accumulating in tensor memory, and commits them to the stage's "empty"
// mbarrier, which the builders wait on before rewriting the stage.  Three
// stages, no block-wide barrier inside the loop.  At the end warps 0-3 read
// the 128-lane accumulator with tcgen05.ld, stage it in shared memory row by
// row and add it into the job's count matrices with bulk asynchronous
// reductions (cp.reduce.async.bulk .add.u32, integer: order-free); a second
// kernel copies the counts out and evaluates Ochiai in fp64 exactly as the
// shared-memory histogram path does.
//
// Operand layout (MN-major, 128-byte swizzle).  A tile of X holds the stage's
// 128 tokens as rows of expert bytes: token u's row is its one-hot vector,
// one byte per expert, E padded to R = 128 or 256 ("rows").  Experts
// 128a..128a+127 form the tile's a-th 16 KB block ("atom"); inside it token u
// owns bytes [128 u, 128 u + 128), and its 16-byte chunk c (experts
// 16c..16c+15 of the atom) sits at chunk position c ^ (u % 8), the 128-byte
// swizzle.  A lane writes its own token's row: zeros with 16-byte stores
// (eight lanes of a store cover all 32 banks, so these are conflict-free),
// then one byte store per pick.  A token with a repeated or out-of-range pick
// keeps an empty row and reports the data error.  For the MMA both operands
// are MN-major (the experts contiguous): 32 tokens are 4 groups of 8 rows
// 1024 bytes apart (stride byte offset) and the next 128 experts lie one
// atom, 16 KB, further on (leading byte offset).  The N = 256 operand
// [X_l; X_{l+1}] of a job that computes C_l and M_l in one MMA is tile A
// followed by tile B, i.e. two atoms 16 KB apart.
//
// Every wait on an mbarrier is bounded (2 s of %globaltimer); a block that
// gives up records MOE_DERR_TIMEOUT, waits (bounded again) for its last
// commit, frees its tensor memory and returns.
#include <algorithm>

#include "common.cuh"
#include "stats_mma.cuh"
#include "waits.cuh"

namespace moe {
namespace {

constexpr int kBuildThreads = 256;        // 8 warps write the X tiles
constexpr int kMmaWarp = kBuildThreads / 32;   // warp 8 issues the MMAs
constexpr int kMmaThreads = kBuildThreads + 32;
constexpr int kTok = 128;                 // tokens per stage
constexpr int kStages = 3;
constexpr int kMmaReduceThreads = 256;
constexpr int kAtom = kTok * 128;         // bytes of 128 experts x 128 tokens

// Shared-memory matrix descriptor of an MN-major operand in the 128-byte
// swizzle layout: start address, leading byte offset (the next 128 experts:
// one atom, 16 KB), stride byte offset (the next 8 tokens: 1024 bytes),
// descriptor version 1, layout type 2 (128-byte swizzle).  Start addresses
// are multiples of 1024, so the base-offset field stays 0.
__device__ __forceinline__ uint64_t smem_desc_mn(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)(kAtom >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor of kind::i8: s32 accumulator, u8 A and B, both
// MN-major, N columns, M = 128 rows.
__host__ __device__ constexpr uint32_t idesc_u8_mn(int N)
{
    return (2u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_u8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc)
{
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        :
        : "r"(tmem_d), "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}

// Token t's K ids: 16-byte loads when K % 4 == 0, 8-byte when K % 2 == 0
// (the host checks that ids is 16-byte aligned), else 4-byte.
template <int K>
__device__ __forceinline__ void load_k(const int32_t *__restrict__ p, int (&v)[K])
{
    if constexpr (K % 4 == 0) {
#pragma unroll
        for (int q = 0; q < K / 4; ++q) {
            const int4 a = __ldg(reinterpret_cast<const int4 *>(p) + q);
            v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
        }
    } else if constexpr (K % 2 == 0) {
#pragma unroll
        for (int q = 0; q < K / 2; ++q) {
            const int2 a = __ldg(reinterpret_cast<const int2 *>(p) + q);
            v[2 * q] = a.x; v[2 * q + 1] = a.y;
        }
    } else {
#pragma unroll
        for (int j = 0; j < K; ++j) v[j] = __ldg(p + j);
    }
}

// 0 when the token's K picks are distinct and in [0, E), else the device
// error code: the range check, then the pairs compared (a sorting network
// costs about as much for K <= 8).
template <int K>
__device__ __forceinline__ int token_check(const int (&v)[K], int E)
{
    bool in_range = true, rep = false;
#pragma unroll
    for (int a = 0; a < K; ++a) {
        in_range &= (unsigned)v[a] < (unsigned)E;
#pragma unroll
        for (int b = 0; b < a; ++b) rep |= v[a] == v[b];
    }
    return !in_range ? MOE_DERR_ID_RANGE : (rep ? MOE_DERR_ID_REPEAT : 0);
}

template <int K, int ROWS>
__global__ void __launch_bounds__(kMmaThreads, 1)
coact_mma_kernel(const int32_t *__restrict__ ids, MmaGeom G, uint32_t *cnt_c, uint32_t *cnt_m, int32_t *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    // full[s]: the builders wrote stage s; empty[s]: the MMAs that read it are
    // done; done: every MMA of the block is done
    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], done_bar;
    __shared__ uint32_t tmem_base_s;

    constexpr int kMt = ROWS / 128;           // 128-row M tiles (= atoms per tile)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int job = blockIdx.x / G.S, slice = blockIdx.x % G.S;
    // a job: C of layer la (has_c) and/or M of layer la (has_m, tile B = layer lb)
    bool has_c, has_m;
    int la;
    if (G.paired) {
        la = job;
        has_c = true;
        has_m = job < G.L - 1;
    } else if (job < G.nc) {
        la = job;
        has_c = true;
        has_m = false;
    } else {
        la = job - G.nc;
        has_c = false;
        has_m = true;
    }
    const int lb = has_m ? la + 1 : la;
    const int T = G.T, E = G.E;
    const int t0 = (int)((long long)T * slice / G.S), t1 = (int)((long long)T * (slice + 1) / G.S);
    const int nchunks = (t1 - t0 + kTok - 1) / kTok;
    constexpr int tile = ROWS * kTok;                  // bytes per X tile
    // stage s: tile A at s * per_stage, tile B right after it (M products)
    const int per_stage = has_m ? 2 * tile : tile;
    // C_l and M_l in one MMA (paired jobs have one 128-row tile): tile B
    // (X_{l+1}) follows tile A (X_l), so the two form one N = 256 MN-major
    // operand [X_l; X_{l+1}]; D's columns [0, 128) are C_l's, [128, 256) M_l's
    const bool stacked = ROWS == 128 && has_c && has_m;
    const uint32_t m_off = stacked ? (uint32_t)ROWS : 0u;   // TMEM column of the M accumulator

    // zero the tiles once: the chunks past E stay zero, the others are
    // rewritten whole every stage
    for (int i = tid * 16; i < kStages * per_stage; i += kMmaThreads * 16)
        *reinterpret_cast<uint4 *>(sm + i) = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        for (int q = 0; q < kStages; ++q) {
            mbar_init(&full_bar[q], kBuildThreads / 32);
            mbar_init(&empty_bar[q], 1);
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&tmem_base_s)), "r"((uint32_t)G.cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_s;
    bool ok = true;

    if (warp < kMmaWarp) {
        // ---- builders.  With tile B (has_m): warps 0-3 write tile A (layer
        // la), warps 4-7 tile B (layer lb), warp w the tokens 32 (w % 4) + lane
        // of the stage.  Without it, warps w and w + 4 share tile A's rows:
        // the first writes the low half of the used chunks, the second the
        // high half.
        const int u = (warp & 3) * 32 + lane;
        const int nch = (E + 15) >> 4;                 // chunks holding experts < E
        int c_lo = 0, c_hi = nch, my_layer = la, my_tile = 0;
        if (has_m) {
            if (warp >= 4) { my_layer = lb; my_tile = tile; }
        } else {
            c_lo = warp >= 4 ? nch / 2 : 0;
            c_hi = warp >= 4 ? nch : nch / 2;
        }
        const int32_t *lay = ids + (size_t)my_layer * T * K;
        // ids of the stage being built (cur) and of the next two (n1, n2): the
        // loads for stage c+2 are issued before stage c waits and builds
        int cur_v[K], n1_v[K], n2_v[K];
        auto fetch = [&](int c, int (&v)[K]) {
            const int t = t0 + c * kTok + u;
            if (c < nchunks && t < t1) load_k<K>(lay + (size_t)t * K, v);
        };
        fetch(0, cur_v);
        fetch(1, n1_v);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages, n = c / kStages;
            fetch(c + 2, n2_v);
            const int t = t0 + c * kTok + u;
            int bad = 0;
            if (t < t1) {
                bad = token_check<K>(cur_v, E);
                if (bad) record_error(err, bad);
            }
            const bool set = t < t1 && !bad;
            if (c >= kStages && !mbar_wait(&empty_bar[s], (n - 1) & 1)) { ok = false; break; }
            uint8_t *row = sm + s * per_stage + my_tile + u * 128;
            // clear the row's chunks, then set the token's bytes (same thread:
            // the stores land in program order)
#pragma unroll
            for (int ch = 0; ch < ROWS / 16; ++ch)
                if (ch >= c_lo && ch < c_hi)
                    *reinterpret_cast<uint4 *>(row + (ch >> 3) * kAtom + (((ch ^ u) & 7) << 4)) = make_uint4(0, 0, 0, 0);
            if (set) {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const int e = cur_v[j], ch = e >> 4;
                    if (ch >= c_lo && ch < c_hi) row[(ch >> 3) * kAtom + (((ch ^ u) & 7) << 4) + (e & 15)] = 1;
                }
            }
            // the stores become visible to the tensor cores; one arrival per warp
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_bar[s]);
#pragma unroll
            for (int j = 0; j < K; ++j) { cur_v[j] = n1_v[j]; n1_v[j] = n2_v[j]; }
        }
    } else {
        // ---- MMA warp: per full stage, one lane issues 4 k-steps of 32 tokens
        // (x the M tiles) into each accumulator and commits them to the
        // stage's empty barrier
        constexpr uint32_t idesc = idesc_u8_mn(ROWS);
        constexpr uint32_t idesc2 = ROWS == 128 ? idesc_u8_mn(256) : 0u;   // stacked jobs have ROWS = 128
        const uint32_t base = smem_addr(sm);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages, n = c / kStages;
            if (!mbar_wait(&full_bar[s], n & 1)) { ok = false; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            if (lane == 0) {
                const uint32_t a0 = base + s * per_stage;
                const uint32_t b0 = a0 + tile;
#pragma unroll
                for (int ks = 0; ks < kTok / 32; ++ks) {
                    const uint32_t koff = (uint32_t)(ks * 32 * 128);     // 32 token rows
                    const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
                    const uint64_t dA = smem_desc_mn(a0 + koff);          // all rows of tile A as the N operand
                    const uint64_t dB = smem_desc_mn(b0 + koff);
#pragma unroll
                    for (int mi = 0; mi < kMt; ++mi) {
                        const uint64_t da = smem_desc_mn(a0 + koff + (uint32_t)(mi * kAtom));
                        if (stacked) {
                            mma_u8(tmem, da, dA, idesc2, acc);
                        } else if (has_c) {
                            mma_u8(tmem + (uint32_t)(mi * ROWS), da, dA, idesc, acc);
                        } else {
                            mma_u8(tmem + (uint32_t)(mi * ROWS), da, dB, idesc, acc);
                        }
                    }
                }
                mma_commit(&empty_bar[s]);
            }
            __syncwarp();
        }
        if (ok && lane == 0 && nchunks > 0) mma_commit(&done_bar);   // tracks every MMA issued before it
    }
    if (!ok) record_error(err, MOE_DERR_TIMEOUT);

    // epilogue: warp w (< 4) reads TMEM lanes 32w..32w+31 = rows of each M
    // tile.  The block's counts are added into the job's count matrices in
    // global memory by bulk asynchronous reductions: a thread stages its row
    // in shared memory (rows 16 bytes longer than E words, so that the 16-byte
    // stores of a warp fall in distinct banks) and adds it with one
    // cp.reduce.async.bulk (element-wise adds performed in L2, atomic with
    // respect to the other blocks' adds).
    if (warp < 4) {
        bool ready = ok;
        if (nchunks > 0) ready = mbar_wait(&done_bar, 0) && ready;
        ready = __all_sync(0xffffffffu, ready);
        if (!ready && lane == 0) record_error(err, MOE_DERR_TIMEOUT);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int pitch = E + 4;                          // staged row, in words
        uint32_t *srow = reinterpret_cast<uint32_t *>(sm) + (size_t)(warp * 32 + lane) * pitch;
        for (int q = 0; ready && nchunks > 0 && q < 2; ++q) {
            if (q == 0 ? !has_c : !has_m) continue;
            const uint32_t col0 = q == 0 ? 0u : m_off;
            uint32_t *dst = (q == 0 ? cnt_c : cnt_m) + (size_t)la * E * E;
            for (int mi = 0; mi < kMt; ++mi) {
                const int row = mi * 128 + warp * 32 + lane;
                for (int c0 = 0; c0 < E; c0 += 16) {
                    uint32_t r[16];
                    const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + col0 + (uint32_t)(mi * ROWS + c0);
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                        : "r"(ta));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    if (row < E) {
                        uint4 *o = reinterpret_cast<uint4 *>(srow + c0);
                        o[0] = make_uint4(r[0], r[1], r[2], r[3]);
                        o[1] = make_uint4(r[4], r[5], r[6], r[7]);
                        o[2] = make_uint4(r[8], r[9], r[10], r[11]);
                        o[3] = make_uint4(r[12], r[13], r[14], r[15]);
                    }
                }
                if (row < E) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.u32 [%0], [%1], %2;"
                                 ::"l"(dst + (size_t)row * E), "r"(smem_addr(srow)), "r"((uint32_t)(E * 4))
                                 : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    // the staged row is rewritten next: wait until the add has read it
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                }
            }
        }
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)G.cols)
                     : "memory");
}

// Two consecutive layers per block.  When C_l and M_l fit one N = 256
// accumulator (E <= 128), a block owning layers la and la + 1 fills all 512
// tensor-memory columns with the products of both: [C_la | M_la] at columns
// 0-255 from A = X_la and B = [X_la; X_la+1], [C_la+1 | M_la+1] at 256-511
// from A = X_la+1 and B = [X_la+1; X_la+2].  A stage then holds the three
// tiles X_la, X_la+1, X_la+2 one atom apart, each written once, so that the
// eight layers of a sweep are built 11 times per token instead of 15 (one
// block a job: X_l for job l and again as the stacked half of job l - 1).
// Four builder warps per tile (a lane per token of the stage, its row written
// as in the one-layer kernel) and one MMA warp; one block per SM.
constexpr int kQuadTiles = 3;
constexpr int kQuadWarpsPerTile = 4;
constexpr int kQuadBuildThreads = kQuadTiles * kQuadWarpsPerTile * 32;
constexpr int kQuadMmaWarp = kQuadBuildThreads / 32;
constexpr int kQuadThreads = kQuadBuildThreads + 32;
constexpr int kQuadStages = 4;
constexpr int kQuadStage = kQuadTiles * kAtom;     // bytes per stage

template <int K>
__global__ void __launch_bounds__(kQuadThreads, 1)
coact_quad_kernel(const int32_t *__restrict__ ids, MmaGeom G, uint32_t *cnt_c, uint32_t *cnt_m, int32_t *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t full_bar[kQuadStages], empty_bar[kQuadStages], done_bar;
    __shared__ uint32_t tmem_base_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int job = blockIdx.x / G.S, slice = blockIdx.x % G.S;
    const int la = 2 * job;
    const int nt = min(kQuadTiles, G.L - la);          // tiles: layers la .. la + nt - 1
    const int nj = min(2, G.L - la);                   // C products: layers la .. la + nj - 1
    const int T = G.T, E = G.E;
    const int t0 = (int)((long long)T * slice / G.S), t1 = (int)((long long)T * (slice + 1) / G.S);
    const int nchunks = (t1 - t0 + kTok - 1) / kTok;

    for (int i = tid * 16; i < kQuadStages * kQuadStage; i += kQuadThreads * 16)
        *reinterpret_cast<uint4 *>(sm + i) = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        for (int q = 0; q < kQuadStages; ++q) {
            mbar_init(&full_bar[q], kQuadWarpsPerTile * nt);   // one arrival per active builder warp
            mbar_init(&empty_bar[q], 1);
        }
        mbar_init(&done_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kQuadMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr(&tmem_base_s)), "r"((uint32_t)G.cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_s;
    bool ok = true;

    if (warp < kQuadMmaWarp) {
        // ---- builders: warp w writes tile w / 4 (layer la + w / 4), tokens
        // 32 (w % 4) + lane of the stage; warps of a missing tile sit out
        const int tt = warp / kQuadWarpsPerTile;
        if (tt < nt) {
            const int u = (warp % kQuadWarpsPerTile) * 32 + lane;
            const int nch = (E + 15) >> 4;
            const int32_t *lay = ids + (size_t)(la + tt) * T * K;
            int cur_v[K], n1_v[K], n2_v[K];
            auto fetch = [&](int c, int (&v)[K]) {
                const int t = t0 + c * kTok + u;
                if (c < nchunks && t < t1) load_k<K>(lay + (size_t)t * K, v);
            };
            fetch(0, cur_v);
            fetch(1, n1_v);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kQuadStages, n = c / kQuadStages;
                fetch(c + 2, n2_v);
                const int t = t0 + c * kTok + u;
                int bad = 0;
                if (t < t1) {
                    bad = token_check<K>(cur_v, E);
                    if (bad) record_error(err, bad);
                }
                const bool set = t < t1 && !bad;
                if (c >= kQuadStages && !mbar_wait(&empty_bar[s], (n - 1) & 1)) { ok = false; break; }
                uint8_t *row = sm + s * kQuadStage + tt * kAtom + u * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    if (ch < nch) *reinterpret_cast<uint4 *>(row + (((ch ^ u) & 7) << 4)) = make_uint4(0, 0, 0, 0);
                if (set) {
#pragma unroll
                    for (int j = 0; j < K; ++j) {
                        const int e = cur_v[j];
                        row[((((e >> 4) ^ u) & 7) << 4) + (e & 15)] = 1;
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_bar[s]);
#pragma unroll
                for (int j = 0; j < K; ++j) { cur_v[j] = n1_v[j]; n1_v[j] = n2_v[j]; }
            }
        }
    } else {
        // ---- MMA warp: per full stage and k-step of 32 tokens, product j
        // reads tile j as A and tiles j, j + 1 as the N = 256 operand (N = 128
        // without layer la + j + 1)
        constexpr uint32_t idesc1 = idesc_u8_mn(128), idesc2 = idesc_u8_mn(256);
        const uint32_t base = smem_addr(sm);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kQuadStages, n = c / kQuadStages;
            if (!mbar_wait(&full_bar[s], n & 1)) { ok = false; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            if (lane == 0) {
                const uint32_t a0 = base + s * kQuadStage;
#pragma unroll
                for (int ks = 0; ks < kTok / 32; ++ks) {
                    const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
                    for (int j = 0; j < nj; ++j) {
                        const uint64_t d = smem_desc_mn(a0 + (uint32_t)(j * kAtom + ks * 32 * 128));
                        mma_u8(tmem + (uint32_t)(256 * j), d, d, j + 1 < nt ? idesc2 : idesc1, acc);
                    }
                }
                mma_commit(&empty_bar[s]);
            }
            __syncwarp();
        }
        if (ok && lane == 0 && nchunks > 0) mma_commit(&done_bar);
    }
    if (!ok) record_error(err, MOE_DERR_TIMEOUT);

    // epilogue: warps 0-3 read TMEM lanes 32 w .. 32 w + 31 (rows of every
    // product) and add each row into its count matrix by a bulk asynchronous
    // reduction, as in the one-layer kernel
    if (warp < 4) {
        bool ready = ok;
        if (nchunks > 0) ready = mbar_wait(&done_bar, 0) && ready;
        ready = __all_sync(0xffffffffu, ready);
        if (!ready && lane == 0) record_error(err, MOE_DERR_TIMEOUT);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int pitch = E + 4;
        const int row = warp * 32 + lane;
        uint32_t *srow = reinterpret_cast<uint32_t *>(sm) + (size_t)row * pitch;
        for (int q = 0; ready && nchunks > 0 && q < 2 * nj; ++q) {
            const int j = q >> 1;
            const bool is_m = q & 1;
            if (is_m && j + 1 >= nt) continue;           // no layer la + j + 1
            const uint32_t col0 = (uint32_t)(256 * j + (is_m ? 128 : 0));
            uint32_t *dst = (is_m ? cnt_m : cnt_c) + (size_t)(la + j) * E * E;
            for (int c0 = 0; c0 < E; c0 += 16) {
                uint32_t r[16];
                const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + col0 + (uint32_t)c0;
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                    "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                    : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                      "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                      "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                    : "r"(ta));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (row < E) {
                    uint4 *o = reinterpret_cast<uint4 *>(srow + c0);
                    o[0] = make_uint4(r[0], r[1], r[2], r[3]);
                    o[1] = make_uint4(r[4], r[5], r[6], r[7]);
                    o[2] = make_uint4(r[8], r[9], r[10], r[11]);
                    o[3] = make_uint4(r[12], r[13], r[14], r[15]);
                }
            }
            if (row < E) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.u32 [%0], [%1], %2;"
                             ::"l"(dst + (size_t)row * E), "r"(smem_addr(srow)), "r"((uint32_t)(E * 4))
                             : "memory");
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
        }
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == kQuadMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)G.cols)
                     : "memory");
}

// blockIdx.y = product: C of layer y (y < nc), M of layer y - nc otherwise.
// The counts were summed over the blocks by the bulk reductions; this copies
// them out and evaluates Ochiai in fp64 (IEEE multiply, square root and
// divide, one rounding to fp32), exactly as the histogram path does.
__global__ void __launch_bounds__(kMmaReduceThreads)
coact_mma_finish_kernel(MmaGeom G, const uint32_t *__restrict__ cnt, uint32_t *coact, float *ochiai, uint32_t *trans)
{
    extern __shared__ uint32_t mdiag[];
    const int E = G.E, p = blockIdx.y;
    const size_t EE = (size_t)E * E;
    const size_t c = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t *m = cnt + (size_t)p * EE;
    if (p < G.nc) {
        if (ochiai) {
            for (int e = threadIdx.x; e < E; e += blockDim.x) mdiag[e] = __ldg(m + (size_t)e * E + e);
            __syncthreads();
        }
        if (c < EE) {
            const int i = (int)(c / E), j = (int)(c % E);
            const uint32_t v = __ldg(m + c);
            if (coact) coact[(size_t)p * EE + c] = v;
            if (ochiai) {
                const double den = __dmul_rn((double)mdiag[i], (double)mdiag[j]);
                const double s = den > 0.0 ? __ddiv_rn((double)v, __dsqrt_rn(den)) : 0.0;
                ochiai[(size_t)p * EE + c] = __double2float_rn(s);
            }
        }
    } else if (c < EE && trans) {
        trans[(size_t)(p - G.nc) * EE + c] = __ldg(m + c);
    }
}

template <int K, int ROWS>
moe_status launch_mma(const int32_t *ids, const MmaGeom &g, uint32_t *part, int32_t *err, cudaStream_t s)
{
    const size_t smem = mma_smem_bytes(g);
    if (allow_smem(coact_mma_kernel<K, ROWS>, smem) != cudaSuccess) return MOE_ERR_CUDA;
    coact_mma_kernel<K, ROWS><<<g.J * g.S, kMmaThreads, smem, s>>>(ids, g, part, part + (size_t)g.nc * g.E * g.E,
                                                                   err);
    return launch_status();
}

template <int K>
moe_status launch_quad(const int32_t *ids, const MmaGeom &g, uint32_t *part, int32_t *err, cudaStream_t s)
{
    const size_t smem = mma_smem_bytes(g);
    if (allow_smem(coact_quad_kernel<K>, smem) != cudaSuccess) return MOE_ERR_CUDA;
    coact_quad_kernel<K><<<g.J * g.S, kQuadThreads, smem, s>>>(ids, g, part, part + (size_t)g.nc * g.E * g.E, err);
    return launch_status();
}

template <int K>
moe_status launch_mma_rows(const int32_t *ids, const MmaGeom &g, uint32_t *part, int32_t *err, cudaStream_t s)
{
    if (g.quad) return launch_quad<K>(ids, g, part, err, s);
    return g.rows == 128 ? launch_mma<K, 128>(ids, g, part, err, s) : launch_mma<K, 256>(ids, g, part, err, s);
}

}  // namespace

bool make_mma_geom(int L, int T, int k, int E, bool want_c, bool want_t, MmaGeom &g)
{
    g = MmaGeom{};
    if (E % 16 != 0 || E < 32 || E > 256 || k < 1 || k > 8 || T < 1) return false;
    g.L = L; g.T = T; g.k = k; g.E = E;
    g.rows = (E + 127) / 128 * 128;
    g.mt = g.rows / 128;
    g.nc = want_c ? L : 0;
    const int nm = (want_t && L > 1) ? L - 1 : 0;
    g.P = g.nc + nm;
    if (g.P == 0) return false;
    // C_l and M_l share layer l's tile when both accumulators fit tensor memory
    g.paired = g.nc > 0 && nm > 0 && g.mt == 1 && 2 * g.rows <= 512;
    // two consecutive layers' C and M per block (all 512 columns)
    g.quad = g.paired && g.rows == 128;
    g.J = g.quad ? (L + 1) / 2 : (g.paired ? L : g.P);
    // paired implies one 128-row tile (2 * mt * E <= 512); its C and M share one
    // N = 2 * rows accumulator; otherwise one product of mt tiles of N = rows
    const int acc_cols = g.quad ? 4 * g.rows : (g.paired ? 2 * g.rows : g.mt * g.rows);
    int cols = 32;
    while (cols < acc_cols) cols <<= 1;
    g.cols = cols;
    // blocks resident per SM: what tensor memory (512 columns) and shared
    // memory (228 KB, 1 KB reserved per block, 1 KB static) allow, at most 4;
    // slices fill one wave of resident blocks
    const int smem_kb = (int)((mma_smem_bytes(g) + 1023) / 1024) + 2;
    const int per_sm = std::max(1, std::min(std::min(4, 512 / cols), 228 / smem_kb));
    const int target = sm_count() * per_sm;
    int S = target / g.J;
    S = std::max(1, std::min(S, (T + kTok - 1) / kTok));
    g.S = S;
    return true;
}

size_t mma_smem_bytes(const MmaGeom &g)
{
    const bool any_m = g.P > g.nc;
    const size_t stages = g.quad ? (size_t)kQuadStages * kQuadStage
                                 : (size_t)kStages * (any_m ? 2 : 1) * g.rows * kTok;
    const size_t staged_rows = (size_t)128 * (g.E + 4) * sizeof(uint32_t);   // the epilogue's rows
    return std::max(stages, staged_rows);
}

size_t mma_partial_words(const MmaGeom &g)
{
    return (size_t)g.P * g.E * g.E;          // every product's counts, summed in place
}

moe_status coact_mma(const int32_t *ids, const MmaGeom &g, uint32_t *part, uint32_t *coact, float *ochiai,
                     uint32_t *trans, int32_t *err, cudaStream_t stream)
{
    // the count matrices start at zero: every block adds its tokens' counts
    if (cudaMemsetAsync(part, 0, mma_partial_words(g) * sizeof(uint32_t), stream) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status st = MOE_ERR_ARG;
    switch (g.k) {
    case 1: st = launch_mma_rows<1>(ids, g, part, err, stream); break;
    case 2: st = launch_mma_rows<2>(ids, g, part, err, stream); break;
    case 3: st = launch_mma_rows<3>(ids, g, part, err, stream); break;
    case 4: st = launch_mma_rows<4>(ids, g, part, err, stream); break;
    case 5: st = launch_mma_rows<5>(ids, g, part, err, stream); break;
    case 6: st = launch_mma_rows<6>(ids, g, part, err, stream); break;
    case 7: st = launch_mma_rows<7>(ids, g, part, err, stream); break;
    case 8: st = launch_mma_rows<8>(ids, g, part, err, stream); break;
    }
    if (st != MOE_OK) return st;
    note_launches(1);
    const size_t EE = (size_t)g.E * g.E;
    dim3 grid((unsigned)((EE + kMmaReduceThreads - 1) / kMmaReduceThreads), (unsigned)g.P);
    coact_mma_finish_kernel<<<grid, kMmaReduceThreads, sizeof(uint32_t) * g.E, stream>>>(g, part, coact, ochiai,
                                                                                          trans);
    st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

}  // namespace moe

// Co-activation and transition counts on the tensor cores (tcgen05, sm_100a).
//
// "Expert Coupling in MoE Pretraining", abstract, and "Cobalt", "Key
// Observation": C_l[i][j] counts the tokens that select experts i and j at
// layer l, M_l[i][j] the tokens that select i at layer l and j at layer l+1.
// With X_l the E x T one-hot matrix (X_l[e][t] = 1 iff token t selects e at
// layer l) these are the products
//     C_l = X_l X_l^T,     M_l = X_l X_{l+1}^T,
// an exact integer contraction over tokens.  Each thread block owns one
// product and one token slice.  Per stage of 128 tokens it writes the ones of
// its X tiles into shared memory (and clears the previous stage's ones, so a
// tile is zeroed only once), then one thread issues tcgen05.mma kind::i8
// (u8 x u8 -> s32, K-major operands, M = 128, N = E, K = 32 per instruction)
// accumulating in tensor memory.  The work is split by warp: eight warps
// write the tiles of a stage and arrive on its "full" mbarrier; a ninth warp
// waits on it, issues the stage's MMAs and commits them to its "empty"
// mbarrier, which the writers wait on before reusing the stage.  Three stages,
// no block-wide barrier inside the loop.  At the end warps 0-3 read the
// 128-lane accumulator with tcgen05.ld and store the block's partial counts;
// a second kernel sums the slices (integer: order-free) and evaluates Ochiai
// in fp64 exactly as the shared-memory histogram path does.
//
// Operand layout (K-major, 128-byte swizzle): an X tile of R rows (experts, R
// a multiple of 128) and 128 tokens stores row r as 128 bytes, token u at
//     r * 128 + (((u / 16) ^ (r % 8)) * 16) + (u % 16),
// 8-row groups 1024 bytes apart; tiles start on 1024-byte boundaries.  The
// MMA for tokens 32q..32q+31 starts its descriptors 32 q bytes into the rows.
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

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle
// layout: rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte
// offset 64 x 16 B), leading byte offset unused (1), descriptor version 1,
// layout type 2 (128-byte swizzle).  addr may sit 32 k-bytes into a row: the
// swizzle acts on the absolute address bits, as for the tile's own stores.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)64 << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
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

// Byte of (expert row e, token slot u) in an X tile: rows of 128 bytes (the
// stage's 128 tokens), the 16-byte chunk index XORed with e % 8 (the 128-byte
// swizzle, which spreads a column's bytes over all banks).
__device__ __forceinline__ int tile_byte(int e, int u)
{
    return e * 128 + ((((u >> 4) ^ e) & 7) << 4) + (u & 15);
}

template <int K>
__device__ __forceinline__ bool ids_in_range(const int (&v)[K], int E)
{
    bool ok = true;
#pragma unroll
    for (int a = 0; a < K; ++a) ok &= (unsigned)v[a] < (unsigned)E;
    return ok;
}

template <int K>
__global__ void __launch_bounds__(kMmaThreads, 1)
coact_mma_kernel(const int32_t *__restrict__ ids, MmaGeom G, uint32_t *__restrict__ part, int32_t *err)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    // full[s]: the builders wrote stage s; empty[s]: the MMAs that read it are
    // done; done: every MMA of the block is done
    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], done_bar;
    __shared__ uint32_t tmem_base_s;

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
    const int T = G.T, E = G.E, rows = G.rows;
    const int t0 = (int)((long long)T * slice / G.S), t1 = (int)((long long)T * (slice + 1) / G.S);
    const int nchunks = (t1 - t0 + kTok - 1) / kTok;
    const int tile = rows * kTok;                      // bytes per X tile
    // stage s: tile A at s * per_stage, tile B right after it (M products)
    const int per_stage = has_m ? 2 * tile : tile;
    // C_l and M_l in one MMA: tile B (X_{l+1}) follows tile A (X_l), so the
    // 2*rows rows from tile A on are one N = 2*rows operand [X_l; X_{l+1}]
    // (single 128-row tile, rows <= 128); D's columns [0, rows) are C_l's,
    // [rows, 2 rows) M_l's
    const bool stacked = has_c && has_m && G.mt == 1;
    // TMEM column of the M accumulator
    const uint32_t m_off = stacked ? (uint32_t)rows : (has_c ? (uint32_t)(G.mt * E) : 0u);

    // zero the tiles once; later stages only set and clear their own ones
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
        // ---- builders: token slot u = tid % 128; threads < 128 write tile A
        // (layer la), threads >= 128 tile B (layer lb, M only).  A token with
        // an invalid pick leaves its column of that tile empty: it then adds
        // nothing to the products that tile enters.  Repeats are checked for
        // the layers whose C this launch computes (all layers when C is not
        // wanted).
        const int u = tid & (kTok - 1);
        const bool writer = tid < kTok || has_m;
        const int my_layer = (tid < kTok) ? la : lb;
        const int my_tile = (tid < kTok) ? 0 : tile;
        const bool check_repeat = (tid < kTok) ? (has_c || G.nc == 0) : (G.nc == 0);
        // ids whose ones are in the tiles of chunks c-3, c-2, c-1 (registers, rotated)
        int prevA[K], prevB[K], prevC[K];
        bool setA = false, setB = false, setC = false;
        // ids of the stage being built (cur) and of the next two (n1, n2): the
        // loads for stage c+2 are issued before stage c waits and builds
        int cur_v[K], n1_v[K], n2_v[K];
        auto fetch = [&](int c, int (&v)[K]) {
            const int t = t0 + c * kTok + u;
            if (writer && c < nchunks && t < t1) load_k<K>(ids + ((size_t)my_layer * T + t) * K, v);
        };
        fetch(0, cur_v);
        fetch(1, n1_v);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages, n = c / kStages;
            fetch(c + 2, n2_v);
            if (c >= kStages && !mbar_wait(&empty_bar[s], (n - 1) & 1)) { ok = false; break; }
            uint8_t *t_s = sm + s * per_stage + my_tile;
            if (writer) {
                if (setA) {                            // chunk c-3 used this stage
#pragma unroll
                    for (int j = 0; j < K; ++j) t_s[tile_byte(prevA[j], u)] = 0;
                }
#pragma unroll
                for (int j = 0; j < K; ++j) { prevA[j] = prevB[j]; prevB[j] = prevC[j]; }
                setA = setB;
                setB = setC;
                setC = false;
                const int t = t0 + c * kTok + u;
                if (t < t1) {
                    if (!ids_in_range<K>(cur_v, E)) {
                        record_error(err, MOE_DERR_ID_RANGE);
                    } else {
                        // a pick whose byte is already set repeats an earlier pick
                        uint32_t seen = 0;
#pragma unroll
                        for (int j = 0; j < K; ++j) {
                            uint8_t *b = t_s + tile_byte(cur_v[j], u);
                            if (check_repeat) seen |= *b;
                            *b = 1;
                        }
                        if (seen) {
#pragma unroll
                            for (int j = 0; j < K; ++j) t_s[tile_byte(cur_v[j], u)] = 0;
                            record_error(err, MOE_DERR_ID_REPEAT);
                        } else {
#pragma unroll
                            for (int j = 0; j < K; ++j) prevC[j] = cur_v[j];
                            setC = true;
                        }
                    }
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
        // ---- MMA warp: per full stage, one lane issues K / 32 x M tiles MMAs
        // into each accumulator and commits them to the stage's empty barrier
        const uint32_t idesc = (2u << 4) | ((uint32_t)(E >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
        const uint32_t idesc2 = (2u << 4) | ((uint32_t)((2 * rows) >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
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
                    const uint32_t koff = (uint32_t)(32 * ks);              // 32 tokens = 32 bytes of each row
                    const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
                    const uint64_t dA = smem_desc_sw128(a0 + koff);         // all E rows of A as the N operand
                    const uint64_t dB = smem_desc_sw128(b0 + koff);
                    for (int mi = 0; mi < G.mt; ++mi) {
                        const uint64_t da = smem_desc_sw128(a0 + koff + (uint32_t)(mi * 128 * 128));
                        if (stacked) {
                            mma_u8(tmem, da, dA, idesc2, acc);
                        } else {
                            if (has_c) mma_u8(tmem + (uint32_t)(mi * E), da, dA, idesc, acc);
                            if (has_m) mma_u8(tmem + m_off + (uint32_t)(mi * E), da, dB, idesc, acc);
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

    // epilogue: warp w (< 4) reads TMEM lanes 32w..32w+31 = rows of each M tile
    if (warp < 4) {
        bool ready = ok;
        if (nchunks > 0) ready = mbar_wait(&done_bar, 0) && ready;
        ready = __all_sync(0xffffffffu, ready);
        if (!ready && lane == 0) record_error(err, MOE_DERR_TIMEOUT);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        for (int q = 0; ready && q < 2; ++q) {
            if (q == 0 ? !has_c : !has_m) continue;
            const int prod = q == 0 ? la : G.nc + la;
            const uint32_t col0 = q == 0 ? 0u : m_off;
            uint32_t *dst = part + ((size_t)prod * G.S + slice) * E * E;
            for (int mi = 0; mi < G.mt; ++mi) {
                const int row = mi * 128 + warp * 32 + lane;
                for (int c0 = 0; c0 < E; c0 += 16) {
                    uint32_t r[16];
                    if (nchunks > 0) {
                        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + col0 + (uint32_t)(mi * E + c0);
                        asm volatile(
                            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                              "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                              "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                            : "r"(ta));
                        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    } else {
#pragma unroll
                        for (int x = 0; x < 16; ++x) r[x] = 0;
                    }
                    if (row < E) {
                        uint4 *o = reinterpret_cast<uint4 *>(dst + (size_t)row * E + c0);
                        o[0] = make_uint4(r[0], r[1], r[2], r[3]);
                        o[1] = make_uint4(r[4], r[5], r[6], r[7]);
                        o[2] = make_uint4(r[8], r[9], r[10], r[11]);
                        o[3] = make_uint4(r[12], r[13], r[14], r[15]);
                    }
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)G.cols)
                     : "memory");
}

// Sum of n partial words at base, base + stride, ... (8 loads in flight).
__device__ __forceinline__ uint32_t mma_sum(const uint32_t *__restrict__ part, size_t base, size_t stride, int n)
{
    uint32_t s = 0;
    int q = 0;
    for (; q + 8 <= n; q += 8) {
        uint32_t v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __ldg(part + base + (size_t)(q + i) * stride);
#pragma unroll
        for (int i = 0; i < 8; ++i) s += v[i];
    }
    for (; q < n; ++q) s += __ldg(part + base + (size_t)q * stride);
    return s;
}

// blockIdx.y = product: C of layer y (y < nc), M of layer y - nc otherwise.
__global__ void __launch_bounds__(kMmaReduceThreads)
coact_mma_reduce_kernel(MmaGeom G, const uint32_t *__restrict__ part, uint32_t *coact, float *ochiai, uint32_t *trans)
{
    extern __shared__ uint32_t mdiag[];
    const int E = G.E, p = blockIdx.y;
    const size_t EE = (size_t)E * E;
    const size_t c = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t pbase = (size_t)p * G.S * EE;
    if (p < G.nc) {
        if (ochiai) {
            for (int e = threadIdx.x; e < E; e += blockDim.x) mdiag[e] = mma_sum(part, pbase + (size_t)e * E + e, EE, G.S);
            __syncthreads();
        }
        if (c < EE) {
            const int i = (int)(c / E), j = (int)(c % E);
            const uint32_t v = mma_sum(part, pbase + c, EE, G.S);
            if (coact) coact[(size_t)p * EE + c] = v;
            if (ochiai) {
                const double den = __dmul_rn((double)mdiag[i], (double)mdiag[j]);
                const double s = den > 0.0 ? __ddiv_rn((double)v, __dsqrt_rn(den)) : 0.0;
                ochiai[(size_t)p * EE + c] = __double2float_rn(s);
            }
        }
    } else if (c < EE && trans) {
        trans[(size_t)(p - G.nc) * EE + c] = mma_sum(part, pbase + c, EE, G.S);
    }
}

template <int K>
moe_status launch_mma(const int32_t *ids, const MmaGeom &g, uint32_t *part, int32_t *err, cudaStream_t s)
{
    const size_t smem = mma_smem_bytes(g);
    if (allow_smem(coact_mma_kernel<K>, smem) != cudaSuccess) return MOE_ERR_CUDA;
    coact_mma_kernel<K><<<g.J * g.S, kMmaThreads, smem, s>>>(ids, g, part, err);
    return launch_status();
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
    g.paired = g.nc > 0 && nm > 0 && 2 * g.mt * E <= 512;
    g.J = g.paired ? L : g.P;
    // paired implies one 128-row tile (2 * mt * E <= 512); its C and M share one
    // N = 2 * rows accumulator
    const int acc_cols = g.paired ? 2 * g.rows : g.mt * E;
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
    return (size_t)kStages * (any_m ? 2 : 1) * g.rows * kTok;
}

size_t mma_partial_words(const MmaGeom &g)
{
    return (size_t)g.P * g.S * g.E * g.E;
}

moe_status coact_mma(const int32_t *ids, const MmaGeom &g, uint32_t *part, uint32_t *coact, float *ochiai,
                     uint32_t *trans, int32_t *err, cudaStream_t stream)
{
    moe_status st = MOE_ERR_ARG;
    switch (g.k) {
    case 1: st = launch_mma<1>(ids, g, part, err, stream); break;
    case 2: st = launch_mma<2>(ids, g, part, err, stream); break;
    case 3: st = launch_mma<3>(ids, g, part, err, stream); break;
    case 4: st = launch_mma<4>(ids, g, part, err, stream); break;
    case 5: st = launch_mma<5>(ids, g, part, err, stream); break;
    case 6: st = launch_mma<6>(ids, g, part, err, stream); break;
    case 7: st = launch_mma<7>(ids, g, part, err, stream); break;
    case 8: st = launch_mma<8>(ids, g, part, err, stream); break;
    }
    if (st != MOE_OK) return st;
    note_launches(1);
    const size_t EE = (size_t)g.E * g.E;
    dim3 grid((unsigned)((EE + kMmaReduceThreads - 1) / kMmaReduceThreads), (unsigned)g.P);
    coact_mma_reduce_kernel<<<grid, kMmaReduceThreads, sizeof(uint32_t) * g.E, stream>>>(g, part, coact, ochiai,
                                                                                          trans);
    st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}

}  // namespace moe

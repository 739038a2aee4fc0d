/*
 * moe_coact.h -- C ABI of libmoecoact.so: expert co-activation statistics and
 * deduplicated, rank-major expert-parallel dispatch and combine on one B200.
 *
 * What the library computes is defined on these pages (cited by title and
 * section):
 *   [EC]  "Expert Coupling in MoE Pretraining: Reducing All-to-All Overhead
 *          with Correlated Placement and Token Shuffling", abstract.
 *   [EPS] "Expert Parallelism > Expert Placement Strategies": the uniform
 *          placement listing; "Capacity-Aware Placement".
 *   [CB]  "Cobalt: Leveraging Expert Co-activation for Efficient Distributed
 *          MoE Training": "Key Observation (Expert Co-activation)" (Ochiai),
 *          "Problem Formulation" (cross-node cost V, node-level deduplication).
 *   [CE]  "Training Communication-Efficient Mixture-of-Experts Language Models
 *          with Layer Re-Configuration", footnote 3 (hidden states and routed
 *          probabilities are dispatched; combine is the inverse exchange).
 *
 * Notation: T tokens, E experts, k experts per token (k <= 8), L layers,
 * G expert-parallel ranks (G <= 64), rpn ranks per node, d hidden size.
 * D_t^l is the set of k distinct experts token t selects at layer l;
 * p(e) = expert_to_rank[e]; s_t is token t's source rank; N(r) = r / rpn.
 * EP ranks and nodes are logical partitions of one GPU's memory: "rank r's
 * receive buffer" is a segment of one device buffer (the moe_ep_* calls
 * spread the ranks over several devices instead).
 *
 * Conventions for every call:
 *  - Pointers marked "device" are device memory owned by the caller; "host"
 *    pointers are host memory owned by the caller.  The library never
 *    allocates or frees memory.
 *  - Device work is enqueued asynchronously on `stream`.  Argument errors are
 *    detected on the host before anything is enqueued and returned as
 *    MOE_ERR_ARG / MOE_ERR_WORKSPACE / MOE_ERR_UNSUPPORTED; nothing is
 *    enqueued then.  A CUDA launch failure returns MOE_ERR_CUDA.
 *  - Errors in the data (an expert id outside [0, E), a repeated id within a
 *    token, a rank outside [0, G), a row index outside the buffer) are found by
 *    the kernels, which skip the offending item and record a code in the
 *    caller's device word `err` (int32).  The first code recorded is kept
 *    (later ones do not overwrite a non-zero word) and no call clears it: the
 *    caller zeroes `err` and reads it after synchronising.  When it is
 *    non-zero the outputs of that call are unspecified.  Kernels never trap.
 *  - Calls keep no state between invocations except the global launch
 *    counter, the settings (moe_coact_stats_method,
 *    moe_plan_dispatch_method, moe_cooperative_blocks) and the static scratch of
 *    moe_plan_dispatch_static.  Workspace ("ws") is
 *    caller-provided device memory of at least the size the matching
 *    *_workspace query returns, 256-byte aligned.
 *  - The only kernels that wait on other blocks or on the tensor cores
 *    (moe_shuffle_balanced, moe_assign_replicas_capped, the single-launch
 *    method of the dispatch plan, the tensor-core method of moe_coact_stats)
 *    give every wait a 2 s limit and then report MOE_DERR_TIMEOUT in `err`.
 */
#ifndef MOE_COACT_H
#define MOE_COACT_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = 1,          /* invalid size, null pointer or misalignment   */
    MOE_ERR_DATA = 2,         /* host-visible data error (host placement calls) */
    MOE_ERR_WORKSPACE = 3,    /* ws too small or misaligned                   */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call failed                   */
    MOE_ERR_UNSUPPORTED = 5   /* shape outside what the kernels implement     */
} moe_status;

/* Codes written to the device error word. */
#define MOE_DERR_ID_RANGE   1   /* expert id outside [0, E)             */
#define MOE_DERR_ID_REPEAT  2   /* an expert id repeated within a token */
#define MOE_DERR_RANK_RANGE 3   /* expert_to_rank or src_rank outside [0, G) */
#define MOE_DERR_ROW_RANGE  4   /* a row index outside the row buffer   */
#define MOE_DERR_TIMEOUT    5   /* a bounded wait on an asynchronous copy ran out
                                   (the kernel stopped early; outputs incomplete) */

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

const char *moe_status_string(moe_status s);

/* Number of kernels this library has launched in this process (all devices,
 * all streams), for benchmark accounting.  Thread-safe. */
uint64_t moe_launch_count(void);

/* ------------------------------------------------------------------------
 * Co-activation statistics  ([EC]; [CB] "Key Observation")
 *
 *   coact[l][i][j]  = |{t : i in D_t^l and j in D_t^l}|   (C_ii = load n_i)
 *   ochiai[l][i][j] = C_ij / sqrt(C_ii * C_jj), evaluated in fp64 with IEEE
 *                     division and square root, rounded once to fp32; 0 when
 *                     C_ii * C_jj = 0
 *   trans[l][i][j]  = |{t : i in D_t^l and j in D_t^{l+1}}|, l < L-1
 *
 * ids     device int32 [L][T][k], row-major (token t's k picks contiguous)
 * coact   device uint32 [L][E][E] or NULL
 * ochiai  device float  [L][E][E] or NULL
 * trans   device uint32 [L-1][E][E] or NULL (ignored when L == 1)
 * err     device int32 [1]
 * ws      device workspace, moe_coact_stats_workspace(L, T, k, E, trans != NULL) bytes
 * Limits: 1 <= k <= 8, k <= E <= 1024, T >= 0, L >= 1, L*T*k < 2^31.
 * Data errors: MOE_DERR_ID_RANGE, MOE_DERR_ID_REPEAT.
 * ---------------------------------------------------------------------- */
size_t moe_coact_stats_workspace(int L, int T, int k, int E, int with_trans);
/* How moe_coact_stats counts (process-wide; returns the previous setting, or
 * -1 for an invalid argument): 0 = default: 2 for E >= 128 where the shape
 * allows, else 1 (measured on B200 with k = 8: the tensor cores are faster at
 * E = 128 and 256, the histograms at E = 64); 1 = shared-memory histograms
 * (per-token counter increments); 2 = tensor cores where the shape allows
 * (E % 16 == 0, 32 <= E <= 256, ids 16-byte aligned): C_l = X_l X_l^T and
 * M_l = X_l X_{l+1}^T for the one-hot X_l[e][t], tcgen05.mma kind::i8 with
 * exact int32 accumulation.  Both give identical results.  The setting affects
 * calls issued after it returns. */
int moe_coact_stats_method(int method);
/* Which method a moe_coact_stats call with these sizes (and C wanted) would use
 * under the current setting: 1 = histograms, 2 = tensor cores; 0 for sizes
 * the call rejects or for T = 0. */
int moe_coact_stats_path(int L, int T, int k, int E, int with_trans);
moe_status moe_coact_stats(const int32_t *ids, int L, int T, int k, int E,
                           uint32_t *coact, float *ochiai, uint32_t *trans,
                           int32_t *err, void *ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Deduplicated dispatch plan  ([EC]: each token travels to each GPU at most once;
 * [CB] "Problem Formulation": V with node-level deduplication, r_t^e = p(e))
 *
 * Rows are the pairs (t, r) with r in m_t = {p(e) : e in D_t}, i.e. one row
 * per token and destination rank however many of its experts live there.
 * Row order is (r, s_t, t) ascending: destination-major ("rank-major"), so
 * rank r's rows are the contiguous segment [offsets[r*G], offsets[r*G+G]),
 * split by source rank.
 *
 * All members are device pointers supplied by the caller:
 *   dest_mask [T]        uint64, bit r set iff r in m_t
 *   counts    [G][G]     int32, counts[s][r] = rows from source s to rank r
 *   offsets   [G*G+1]    int32, offsets[r*G+s] = first row of (r, s);
 *                        offsets[G*G] = R
 *   row_token [T*k]      int32, token of row i (entries [0, R) written)
 *   row_jmask [T*k]      uint8, bit j set iff p(e_tj) is row i's rank
 *   row_of    [T][k]     int32, the row that carries (t, e_tj)
 *   summary   [5]        int64: R, R_remote (rows with r != s_t),
 *                        local = #{(t,j) : p(e_tj) = s_t},
 *                        V = sum_t |{N(r) : r in m_t} \ {N(s_t)}|, T*k
 * ---------------------------------------------------------------------- */
typedef struct {
    uint64_t *dest_mask;
    int32_t *counts;
    int32_t *offsets;
    int32_t *row_token;
    uint8_t *row_jmask;
    int32_t *row_of;
    int64_t *summary;
} moe_plan;

/* ids            device int32 [T][k] (one layer)
 * expert_to_rank device int32 [E], values in [0, G)
 * src_rank       device int32 [T] or NULL; NULL means contiguous shards
 *                s_t = t / (T/G) and then requires G | T
 * Limits: 1 <= k <= 8, k <= E, 1 <= G <= 64, rpn >= 1, G % rpn == 0, T >= 0,
 * T*k < 2^31 (else MOE_ERR_ARG); E <= 12288 (else MOE_ERR_UNSUPPORTED).  The
 * plan's arrays need only their element alignment (row_of is written with
 * wider stores where it is 16- or 8-byte aligned).  Data errors:
 * MOE_DERR_ID_RANGE, MOE_DERR_ID_REPEAT, MOE_DERR_RANK_RANGE. */
size_t moe_plan_dispatch_workspace(int T, int k, int G, int with_src_rank);
/* The plan with source ranks in two calls.  moe_plan_sources computes its
 * first step alone -- the tokens' stable order by source rank, a counting
 * sort of src_rank -- into ws (moe_plan_dispatch_workspace(T, k, G, 1)
 * bytes); moe_plan_dispatch_presorted then takes the same arguments as
 * moe_plan_dispatch (src_rank not NULL) and the same workspace, and runs the
 * rest.  The result is moe_plan_dispatch's.  The source order depends only on
 * src_rank, so it can be computed as soon as the source ranks exist (the
 * previous layer's shuffle targets), on another stream, ahead of the layer's
 * routing; the caller orders the two calls (same stream, or an event) and
 * keeps the workspace for this plan in between.  moe_plan_sources: T >= 0,
 * 1 <= G <= 64, src_rank device int32 [T] (values outside [0, G) are
 * reported as MOE_DERR_RANK_RANGE in err and counted as rank 0, as by
 * moe_plan_dispatch).  moe_plan_dispatch_presorted does not re-read src_rank
 * and always launches separate kernels (moe_plan_dispatch_method does not
 * apply). */
moe_status moe_plan_sources(const int32_t *src_rank, int T, int G, int32_t *err, void *ws, size_t ws_bytes,
                            cudaStream_t stream);
moe_status moe_plan_dispatch_presorted(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                       const int32_t *expert_to_rank, const int32_t *src_rank,
                                       const moe_plan *plan, int32_t *err,
                                       void *ws, size_t ws_bytes, cudaStream_t stream);
/* How the plan is launched (process-wide; returns the previous setting, or -1
 * for an invalid argument): 0 = default: separate kernels (counting sort by
 * source, counts, scatter), each of which runs beside other work on the GPU
 * without waiting on it; 1 = one cooperative launch whose phases are
 * separated by grid barriers, when the plan has at most 512 chunks of 1024
 * tokens (else the separate kernels run).  A cooperative launch needs all its
 * blocks resident at once, so use 1 where the plan runs in line on its stream
 * rather than beside long kernels on another.  Results are identical; the
 * setting also applies to moe_plan_dispatch_ranks and
 * moe_plan_dispatch_static and affects calls issued after it returns. */
int moe_plan_dispatch_method(int method);

/* Blocks of the cooperative kernels' launches (moe_shuffle_balanced,
 * moe_assign_replicas_capped; process-wide; returns the previous setting, or
 * -1 for a negative argument): 0 = default, one block per SM; n > 0 = n
 * blocks (at most one per SM).  Results are identical for every setting.  A
 * smaller grid leaves the other SMs to kernels running beside the call on
 * other streams -- the row traffic, when these run on a second stream -- at
 * the cost of a longer call.  Affects calls issued after it returns. */
int moe_cooperative_blocks(int blocks);
moe_status moe_plan_dispatch(const int32_t *ids, int T, int k, int E, int G, int rpn,
                             const int32_t *expert_to_rank, const int32_t *src_rank,
                             const moe_plan *plan, int32_t *err,
                             void *ws, size_t ws_bytes, cudaStream_t stream);

/* The same plan when experts have several replicas ([CB] "Problem
 * Formulation": task (t, e) runs on a rank r_t^e holding e): pick_rank
 * device int32 [T][k] gives the serving rank of every pick (e.g. from
 * moe_assign_replicas), in place of p(e).  Rows, order, outputs, workspace
 * and errors as moe_plan_dispatch; a pick rank outside [0, G) is
 * MOE_DERR_RANK_RANGE. */
moe_status moe_plan_dispatch_ranks(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                   const int32_t *pick_rank, const int32_t *src_rank,
                                   const moe_plan *plan, int32_t *err,
                                   void *ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Communication-aware task assignment over replicas  ([CB] "Problem
 * Formulation": V counts the remote nodes a token's tasks reach; the
 * assignment sends each token to as few remote nodes as it can)
 *
 * For every token t (source rank s = src_rank[t], or t/(T/G) when NULL; node
 * ns = s / rpn): the smallest set S of nodes other than ns such that every
 * pick's expert has a replica on ns or on a node of S (exact; ties: smallest
 * S as a bit pattern); then, pick by pick in j order, among the ranks hosting
 * the expert on ns (or, if none, on the nodes of S): rank s if it is one of
 * them, else the lowest one an earlier pick of the token already uses (no new
 * row), else the lowest one.  n_remote[t] = |S|, the token's share of V.
 * replica_rank device int32 [E][1 + G/rpn] (ranks, unused slots -1) and
 * n_rep device int32 [E], e.g. from moe_place_replicas; pick_rank device
 * int32 [T][k] out; n_remote device int32 [T] out or NULL.
 * Limits: G/rpn <= 8 nodes.  Data errors: MOE_DERR_ID_RANGE (invalid ids or an
 * expert without replicas; the token's outputs are -1), MOE_DERR_RANK_RANGE.
 * ---------------------------------------------------------------------- */
moe_status moe_assign_replicas(const int32_t *ids, int T, int k, int E, int G, int rpn,
                               const int32_t *replica_rank, const int32_t *n_rep, const int32_t *src_rank,
                               int32_t *pick_rank, int32_t *n_remote, int32_t *err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Task assignment under a load tolerance  ([CB] "Problem Formulation": the
 * tasks a rank runs, sum_e w_r^e, at most (1 + eps) K T / G, beside the
 * fewest remote nodes per token)
 *
 * The page states the constraint, not how to meet it.  Reading taken: tokens
 * in id order; before token t every rank whose task count has reached
 * cap = floor((1 + eps) * (T k) / G) (fp64: one multiply, one divide; no cap
 * for eps = inf) is closed to t, and t is assigned exactly as by
 * moe_assign_replicas over the open replicas of its experts -- a pick whose
 * expert has no open replica may use all of them (the cap gives way, never
 * the task).  A token can take a rank past the cap by at most k - 1 tasks;
 * eps = inf gives moe_assign_replicas's result.  The call reaches the same
 * result with every token in flight at once: the uncapped assignment (the
 * first round's choices), then at most G + 1 rounds of one cooperative
 * launch (one grid barrier a round, with the library's 2 s bounded wait).
 * Arguments as moe_assign_replicas, plus: eps >= 0 (else MOE_ERR_ARG);
 * rank_load device int64 [G] out or NULL (tasks per rank after the batch);
 * ws device, moe_assign_replicas_capped_workspace(G) bytes, 256-byte aligned,
 * caller-owned, overwritten by each call (calls on one workspace must not
 * overlap).  Limits: T k < 2^31 (else MOE_ERR_ARG), G <= 64, G/rpn <= 8
 * nodes, E * (4 (G/rpn + 3) + 8) + 4 G (B | 1) bytes <= 200 KB for a grid of
 * B blocks (one per SM, or moe_cooperative_blocks; else
 * MOE_ERR_UNSUPPORTED).  When a block's share of the tokens fits, their
 * pick-rank sets (8 bytes a token) also live in its shared memory.  Data
 * errors as moe_assign_replicas; an invalid token counts for no rank.
 * ---------------------------------------------------------------------- */
size_t moe_assign_replicas_capped_workspace(int G);
moe_status moe_assign_replicas_capped(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                      const int32_t *replica_rank, const int32_t *n_rep, const int32_t *src_rank,
                                      double eps, int32_t *pick_rank, int32_t *n_remote, long long *rank_load,
                                      int32_t *err, void *ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * moe_coact_ema ([CB] "Key Observation": Ochiai on exponential moving averages
 *   of the co-selection counts and loads).  Per cell, in fp64 with IEEE
 *   rounding and no fused multiply-add:
 *     ema_out[l][i][j] = alpha * coact[l][i][j] + (1 - alpha) * ema_in[l][i][j]
 *   (ema_out = coact when ema_in is NULL: the first batch); the diagonal is the
 *   load EMA; ochiai[l][i][j] = ema_ij / sqrt(ema_ii * ema_jj) rounded once to
 *   fp32, 0 when the product is 0.
 *   coact device uint32 [L][E][E] (moe_coact_stats's output); ema_in device
 *   double [L][E][E] or NULL; ema_out device double [L][E][E], not ema_in
 *   (out of place; alternate two buffers); ochiai device float [L][E][E] or
 *   NULL.  MOE_ERR_ARG for alpha outside [0, 1], ema_in == ema_out, E > 4096.
 * ---------------------------------------------------------------------- */
moe_status moe_coact_ema(const uint32_t *coact, int L, int E, double alpha, const double *ema_in,
                         double *ema_out, float *ochiai, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Dispatch plan without caller-provided workspace.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory -- code running inside another framework's allocator or
 * memory-pool hook (a cudaMalloc there would re-enter the allocator),
 * processes that reserve their whole device-memory budget at start-up, and
 * latency-critical loops that cannot accept cudaMalloc's possible implicit
 * device synchronisation.
 *
 * Same arguments, outputs and errors as moe_plan_dispatch, without ws and
 * ws_bytes.  The scratch is a statically reserved device array of
 * MOE_PLAN_STATIC_SCRATCH_BYTES held by every GPU that loads the library until
 * the process exits.  Calls whose moe_plan_dispatch_workspace(T, k, G,
 * src_rank != NULL) exceeds it return MOE_ERR_WORKSPACE and enqueue nothing
 * (4 MiB covers, for example, T = 786432 tokens at G = 64 with source ranks).
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, which also loads the library's kernels on that
 * device); make that first call before any stream capture.  All calls on a
 * device share the array and each clears the part that must start at zero:
 * calls whose kernels overlap on the GPU (unordered streams) race on it.
 * ---------------------------------------------------------------------- */
#define MOE_PLAN_STATIC_SCRATCH_BYTES (4u << 20)
moe_status moe_plan_dispatch_static(const int32_t *ids, int T, int k, int E, int G, int rpn,
                                    const int32_t *expert_to_rank, const int32_t *src_rank,
                                    const moe_plan *plan, int32_t *err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Row permute into the rank-major send buffer  ([EC]; [CE] footnote 3)
 *   send[row_of[t][j]][:] = x[t][:]   for every t, j
 * which equals send[i] = x[row_token[i]] for every row i < R.  Each token's
 * row is read from x once and written to each of its distinct rows.
 *
 * x        device [T][d] elements of `dtype` (16-byte aligned)
 * row_of   device int32 [T][k] (from moe_plan_dispatch)
 * send     device [R_max][d] of `dtype` (16-byte aligned); rows >= R untouched
 * Requires d * sizeof(dtype) to be a multiple of 16 bytes.
 * Data errors: MOE_DERR_ROW_RANGE (row_of outside [0, R_max)).
 * ---------------------------------------------------------------------- */
moe_status moe_permute(const void *x, moe_dtype dtype, int T, int d, int k,
                       const int32_t *row_of, int64_t R_max, void *send,
                       int32_t *err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Weighted combine, the inverse of dispatch  ([EC]: "then combine the
 * results"; [CE] footnote 3)
 *   out[t][:] = sum_j w[t][j] * Y[idx[t][j]][:]
 * accumulated in fp32 with fused multiply-adds.  When several j of a token
 * name the same row (several of its experts on one rank), that row is read
 * once and its weights are first summed in j order; the distinct rows are
 * then accumulated in order of first appearance.  Worst-case error against
 * the exact sum is below (2k-1) * 2^-24 * sum_j |w_tj * Y_idx_tj|.
 * Output is fp32, or rounded to bf16 (nearest even) for out_dtype MOE_BF16.
 *
 * Y    device [R_max][d] of y_dtype (16-byte aligned)
 * idx  device int32 [T][k] row indices into Y (e.g. row_of)
 * w    device float [T][k]
 * out  device [T][d] of out_dtype (16-byte aligned)
 * Requires d * sizeof(y_dtype) to be a multiple of 16 bytes.
 * Data errors: MOE_DERR_ROW_RANGE (that term is skipped).
 * ---------------------------------------------------------------------- */
moe_status moe_combine(const void *Y, moe_dtype y_dtype, int64_t R_max, int d,
                       const int32_t *idx, const float *w, int T, int k,
                       void *out, moe_dtype out_dtype, int32_t *err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Receiver-side pre-reduced combine  ([CE] footnote 3: the dispatcher moves
 * hidden states and routed probabilities; [EC]: dispatch, then combine)
 *
 * With deduplicated dispatch a row reaches its rank once however many of the
 * token's experts live there.  The receiving rank can then apply those
 * experts, weight their outputs with the dispatched gates and return a single
 * row per (token, rank); the source only sums its rows.
 *
 * moe_dispatch_gates: for each row i < R (R = summary[0], read on the device):
 *   send_e[i][j] = e_tj and send_w[i][j] = w[t][j] for the picks j of token
 *   t = row_token[i] with bit j of row_jmask[i] set; -1 and 0 otherwise.
 *   ids device int32 [T][k]; w device float [T][k]; row_token, row_jmask,
 *   summary from moe_plan_dispatch; send_e device int32 [R_max][k]; send_w
 *   device float [R_max][k].  Data errors: MOE_DERR_ROW_RANGE.
 *
 * moe_expert_reduce: stand-in experts, expert e mapping a row x to scale[e]*x:
 *   y[i] = sum_j send_w[i][j] * scale[send_e[i][j]] * send[i]  (j with
 *   send_e >= 0), for i < R: g_j = send_w * scale rounded to fp32 once, then an
 *   fp32 FMA chain in j order; y fp32 or rounded to bf16 (nearest even).
 *   send device [R_max][d] of dtype; scale device float [E]; y device
 *   [R_max][d] of y_dtype (both 16-byte aligned; rows a multiple of 16 bytes).
 *   Data errors: MOE_DERR_ID_RANGE (send_e >= E; the row is not reduced).
 *
 * moe_combine_rows: out[t] = sum of the distinct rows {row_of[t][j]} of Y,
 *   each once (weight 1), fp32 accumulation in order of first appearance;
 *   Y device [R_max][d] of y_dtype, row_of device int32 [T][k], out device
 *   [T][d] of out_dtype.  Data errors: MOE_DERR_ROW_RANGE.
 * ---------------------------------------------------------------------- */
moe_status moe_dispatch_gates(const int32_t *ids, const float *w, int T, int k,
                              const int32_t *row_token, const uint8_t *row_jmask, const int64_t *summary,
                              int64_t R_max, int32_t *send_e, float *send_w, int32_t *err, cudaStream_t stream);
moe_status moe_expert_reduce(const void *send, moe_dtype dtype, int64_t R_max, int d,
                             const int64_t *summary, const int32_t *send_e, const float *send_w, int k,
                             const float *scale, int E, void *y, moe_dtype y_dtype, int32_t *err,
                             cudaStream_t stream);
moe_status moe_combine_rows(const void *Y, moe_dtype y_dtype, int64_t R_max, int d, const int32_t *row_of,
                            int T, int k, void *out, moe_dtype out_dtype, int32_t *err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Expert parallelism over several devices  ([EC]: each token is sent to each
 * GPU once and the results combined; [CE] footnote 3: hidden states and
 * routed probabilities are dispatched, the combine is the inverse exchange)
 *
 * The G ranks are spread over W devices, Gl = G/W consecutive ranks per
 * device: device h hosts ranks h*Gl .. h*Gl+Gl-1.  Each device plans its own
 * tokens with moe_plan_dispatch, every token's source rank in the device's
 * range (src_rank given).  Device h's receive buffer then holds the rows
 * addressed to its ranks in the order the one-device plan over all tokens
 * gives them -- destination rank, then source rank, then token -- i.e.
 * exactly rows [off(h*Gl, 0), off(h*Gl+Gl, 0)) of that plan's send buffer,
 * off(r, s) being its offsets[r*G+s].  Rows are stored to and loaded from
 * the other devices' buffers through peer pointers (plain loads and stores
 * over NVLink).  Synchronising the devices between the phases (all stores of
 * every device done before any receiver reads; all combines done before the
 * next dispatch overwrites a buffer) is the caller's, e.g. a small NCCL
 * all-reduce on the same stream.
 *
 * moe_ep_routes: counts_all device int32 [G][G], row s = the counts row of
 *   source rank s as planned by the device hosting s (gathered from all
 *   devices); offsets device int32 [G*G+1] of this device's plan; me = this
 *   device's index in [0, W).  Writes route device int64 [2*G*Gl + 2]:
 *   route[0] = rows this device receives; route[1+i], i <= P = G*Gl: the
 *   local row where segment i starts (segment i = destination rank i/Gl,
 *   source rank me*Gl + i%Gl; route[1+P] = this device's R); route[P+2+i]:
 *   the shift from a local row of segment i to its row in the receiving
 *   device's buffer.  Data errors: MOE_DERR_ROW_RANGE if a gathered count is
 *   negative or this device's row of counts_all disagrees with its plan.
 *
 * moe_ep_permute: recv[h][q][:] = x[t][:] for every local row (t, r) of this
 *   device's plan, h = r/Gl and q its row in h's buffer (from route); each
 *   token's row of x is read once.  x device [T][d] of dtype (16-byte
 *   aligned); row_of device int32 [T][k] of the local plan; recv_base device
 *   array of W addresses (this device's own buffer at index me; every buffer
 *   32-byte aligned, recv_cap rows of d elements).  Data errors:
 *   MOE_DERR_ROW_RANGE (a row outside the plan, a target row outside
 *   [0, recv_cap) or a misaligned or null base: that store is skipped).
 *
 * moe_ep_combine: the combine of moe_combine (w given) or of
 *   moe_combine_rows (w NULL: each distinct row once, weight 1) for this
 *   device's T tokens, with Y's row for a local row read from its receiving
 *   device's buffer: y_base device array of W addresses (32-byte aligned,
 *   y_cap rows of d elements of y_dtype each, in the receive-buffer order);
 *   idx device int32 [T][k] local rows (row_of), R_max the local row bound;
 *   out device [T][d] of out_dtype.  Results equal those of moe_combine /
 *   moe_combine_rows on the one-device send buffer bit for bit.  Data errors:
 *   MOE_DERR_ROW_RANGE (the term is skipped).
 *
 * moe_ep_scatter_rows: a record of row_bytes bytes per local row (e.g. the
 *   gates of moe_dispatch_gates: k int32 or k floats) stored to the receiving
 *   devices the same way: dst[h][q] = src[x] for the local rows x < R (R from
 *   route).  src device [R_max][row_bytes] (4-byte aligned); dst_base device
 *   array of W addresses (32-byte aligned, dst_cap records each); row_bytes a
 *   multiple of 4, at most 1024.
 *
 * Limits: 1 <= G <= 64, W | G, 0 <= me < W, 1 <= k <= 8, d*sizeof(dtype) a
 * multiple of 16 bytes.
 * ---------------------------------------------------------------------- */
moe_status moe_ep_routes(const int32_t *counts_all, const int32_t *offsets, int G, int W, int me,
                         int64_t *route, int32_t *err, cudaStream_t stream);
moe_status moe_ep_permute(const void *x, moe_dtype dtype, int T, int d, int k, const int32_t *row_of,
                          int64_t R_max, const int64_t *route, int G, int W, void *const *recv_base,
                          int64_t recv_cap, int32_t *err, cudaStream_t stream);
moe_status moe_ep_combine(void *const *y_base, moe_dtype y_dtype, int64_t y_cap, int d,
                          const int64_t *route, int G, int W, int64_t R_max, const int32_t *idx,
                          const float *w, int T, int k, void *out, moe_dtype out_dtype, int32_t *err,
                          cudaStream_t stream);
moe_status moe_ep_scatter_rows(const void *src, int64_t row_bytes, int64_t R_max, const int64_t *route,
                               int G, int W, void *const *dst_base, int64_t dst_cap, int32_t *err,
                               cudaStream_t stream);

/* moe_ep_exchange_rows ([EC] abstract: the method's gain is the rows that no
 *   longer cross GPUs): with the G ranks on W devices (Gl = G/W consecutive
 *   ranks each) and counts_all host int32 [G][G] (rows from source rank s to
 *   rank r, the gathered counts of every device's plan), sent[h] = rows whose
 *   source is on device h and whose rank is not, received[h] = rows whose rank
 *   is on device h and whose source is not.  Each such row crosses NVLink once
 *   in the dispatch and once back in the combine.  sent, received host int64
 *   [W] out.  MOE_ERR_ARG for a negative count or W not dividing G. */
moe_status moe_ep_exchange_rows(const int32_t *counts_all, int G, int W, long long *sent, long long *received);

/* ------------------------------------------------------------------------
 * Token shuffling  ([EC]: move each token to the GPU predicted to hold its
 * next-layer experts)
 *
 * moe_rank_score: rank_score[e][r] = sum over e' with p_{l+1}(e') = r of
 *   trans_l[e][e'] -- how often a token that picks e at layer l picks an
 *   expert hosted on rank r at layer l+1.
 *   trans_l device uint32 [E][E]; next_expert_to_rank device int32 [E];
 *   rank_score device uint32 [E][G].  Data errors: MOE_DERR_RANK_RANGE.
 *
 * moe_shuffle_targets: target[t] = argmax_r sum_j rank_score[e_tj][r]
 *   (sums in uint64; the lowest r among equal scores).
 *   ids device int32 [T][k]; rank_score device uint32 [E][G], E*G <= 16384;
 *   target device int32 [T].  Data errors: MOE_DERR_ID_RANGE.
 * ---------------------------------------------------------------------- */
moe_status moe_rank_score(const uint32_t *trans_l, const int32_t *next_expert_to_rank,
                          int E, int G, uint32_t *rank_score, int32_t *err, cudaStream_t stream);
moe_status moe_shuffle_targets(const int32_t *ids, int T, int k, int E, int G,
                               const uint32_t *rank_score, int32_t *target,
                               int32_t *err, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * moe_shuffle_balanced ([EC] abstract: the shuffle happens in the
 *   reduce-scatter after attention, and a reduce-scatter hands every rank an
 *   equal shard).  Shuffle targets with at most `capacity` tokens per rank:
 *   with S_t(r) = sum_j rank_score[e_tj][r] (uint64), the result is that of
 *   taking all (t, r) pairs in the order S desc, t asc, r asc and accepting a
 *   pair when t has no rank yet and r holds fewer than `capacity` tokens --
 *   the unique stable assignment of tokens to ranks under these orders.  With
 *   capacity >= T it equals moe_shuffle_targets.  Computed by deferred
 *   acceptance in one cooperative kernel (one block per SM, or as many as
 *   moe_cooperative_blocks sets; blocks own ranks in turn).
 *   ids device int32 [T][k]; rank_score device uint32 [E][G], E*G <= 16384,
 *   G <= 64, T < 2^27; requires G*capacity >= T (MOE_ERR_ARG otherwise);
 *   target device int32 [T] (out); info device int64 [6] (out, may be NULL):
 *   rounds taken, proposals made, then nanoseconds spent proposing (block
 *   0), gathering a rank's proposals and selecting (the slowest block's
 *   totals) and waiting at grid barriers (block 0).  ws: moe_shuffle_balanced_workspace(T, G,
 *   capacity) bytes, 256-byte aligned.  Data errors: MOE_DERR_ID_RANGE (the
 *   token's picks then score 0); MOE_DERR_TIMEOUT if a grid barrier waited
 *   more than 2 s (the kernel then returns with target incomplete).
 * ---------------------------------------------------------------------- */
size_t moe_shuffle_balanced_workspace(int T, int G, int capacity);
moe_status moe_shuffle_balanced(const int32_t *ids, int T, int k, int E, int G,
                                const uint32_t *rank_score, int capacity, int32_t *target,
                                long long *info, void *ws, size_t ws_bytes, int32_t *err,
                                cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Placement (host, synchronous)
 *
 * moe_place_uniform ([EPS] uniform listing): expert_to_rank[e] = e / (E/G);
 *   MOE_ERR_ARG unless G divides E.
 *
 * moe_place_capacity ([EPS] "Capacity-Aware Placement"): experts in
 *   descending load (equal loads: lower id first) each go to the rank with the
 *   least load so far (ties: lowest rank); loads summed in fp64.
 *   load host double [E]; rank_load host double [G] (out, may be NULL).
 *
 * moe_place_correlated ([EC]: experts often selected together share a GPU).
 *   The pages state the goal only; this is a greedy equal-size grouping.
 *   With nodes = G/rpn > 1, experts are first split into `nodes` groups of
 *   E/nodes, then each node's experts into rpn groups of E/G.  A group is
 *   seeded with the unassigned expert of largest C_ee and grown by the
 *   unassigned expert whose fp64 Ochiai summed over the group's members (in
 *   the order they joined) is largest; ties go to the lowest id.  Node group
 *   q, rank group u -> rank q*rpn + u.
 *   coact host uint32 [E][E] (one layer); requires G | E and rpn | G.
 *
 * expert_to_rank host int32 [E] (out) for all three.
 * ---------------------------------------------------------------------- */
moe_status moe_place_uniform(int E, int G, int32_t *expert_to_rank);
moe_status moe_place_capacity(const double *load, int E, int G, int32_t *expert_to_rank, double *rank_load);
moe_status moe_place_correlated(const uint32_t *coact, int E, int G, int rpn, int32_t *expert_to_rank);

/* moe_place_correlated_capped ([CB] "Problem Formulation": a load tolerance on
 *   every rank).  The correlated greedy above, where a node group only admits
 *   experts that keep its load (sum of C_ee) at most (1+eps) W / (G/rpn) and a
 *   rank group at most (1+eps) W / G, W = sum_e C_ee; when no unassigned
 *   expert fits, the lightest one joins (ties: lowest id), so a group exceeds
 *   its cap by less than one expert's load.  eps < 0: no cap (equals
 *   moe_place_correlated). */
moe_status moe_place_correlated_capped(const uint32_t *coact, int E, int G, int rpn, double eps,
                                       int32_t *expert_to_rank);

/* moe_place_replicas ([CB] "Problem Formulation": every expert has at least
 *   one replica, |P_r| <= (1+rho)E/G; "Two-Stage Expert Layout Planner":
 *   co-activated experts share nodes).  The page states the constraints, not
 *   an algorithm; this is a greedy.  Starting from expert_to_rank (one replica
 *   each), every rank gets room for `extra` more experts (extra = rho*E/G);
 *   candidate replicas (e, node q), e not on q, are taken in decreasing
 *   score(e, q) = sum of coact[e][e'] over the experts e' placed on q (ties:
 *   lower e, then lower q), each onto the rank of q with the most room left
 *   (ties: lowest rank), skipping nodes without room; zero scores are not added.
 *   replica_rank host int32 [E][1 + G/rpn] out (original rank first, then in
 *   the order added; -1 unused), n_rep host int32 [E] out. */
moe_status moe_place_replicas(const uint32_t *coact, int E, int G, int rpn, const int32_t *expert_to_rank,
                              int extra, int32_t *replica_rank, int32_t *n_rep);

/* moe_rank_loads ([EPS] "Capacity-Aware Placement": a device's load is the
 *   sum of its experts' loads).  rank_load[r] = sum of C_ee over the experts e
 *   with expert_to_rank[e] = r: the tasks rank r serves in the batch whose
 *   counts coact holds (only the diagonal is read).  coact host uint32 [E][E];
 *   expert_to_rank host int32 [E]; rank_load host int64 [G] out.  MOE_ERR_ARG
 *   for a rank outside [0, G). */
moe_status moe_rank_loads(const uint32_t *coact, int E, int G, const int32_t *expert_to_rank,
                          long long *rank_load);

/* ------------------------------------------------------------------------
 * moe_selftest_wait_timeout (no counterpart on the pages: a test of the error
 *   path of the bounded device waits).  kind 0: a cooperative launch of 4
 *   blocks meets at a grid barrier that block 1 never reaches; kind 1: one
 *   block waits on an mbarrier phase that nothing completes.  Either way the
 *   waits give up after about 2 s, err receives MOE_DERR_TIMEOUT and the
 *   kernel returns; nothing faults and the context stays usable.  ws:
 *   moe_selftest_workspace() bytes, 256-byte aligned (kind 0 only).
 * ---------------------------------------------------------------------- */
size_t moe_selftest_workspace(void);
moe_status moe_selftest_wait_timeout(int kind, int32_t *err, void *ws, size_t ws_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_COACT_H */

/*
 * ORACLE -- test infrastructure only.
 *
 * A plain, slow, single-threaded CPU statement of what the co-activation and
 * deduplicated-dispatch hot path computes, written from the pages' prose and
 * formulas.  Its only users are the tests, the smoke check of the build entry
 * and the CPU-baseline leg of the benchmark.  The product library never loads,
 * links or calls it, and it shares no code with the product's CUDA sources.
 *
 * Pages cited (by title and section):
 *   [EC]  "Expert Coupling in MoE Pretraining: Reducing All-to-All Overhead
 *          with Correlated Placement and Token Shuffling", abstract.
 *   [EPS] "Expert Parallelism > Expert Placement Strategies", the uniform
 *          placement listing and its printed example; "Capacity-Aware Placement".
 *   [CB]  "Cobalt: Leveraging Expert Co-activation for Efficient Distributed MoE
 *          Training", "Key Observation (Expert Co-activation)" (Ochiai formula)
 *          and "Problem Formulation" (cross-node cost V).
 *   [CE]  "Training Communication-Efficient Mixture-of-Experts Language Models
 *          with Layer Re-Configuration", footnote 3 (the dispatcher carries
 *          hidden states and routed probabilities; combine is the inverse).
 *
 * Precision: counts and plans are integers.  Ochiai is fp64 rounded once to
 * fp32.  The combine is evaluated in fp64 (the pages fix no precision for it).
 * Compile with -O2 -ffp-contract=off.
 *
 * Parity pins for every function live in the CPU tests; the correlated
 * placement's grouping quality is "parity unpinned" beyond its stated greedy
 * steps and the planted-cluster case.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_DATA 2

/* A token's D_t is a set of k distinct expert ids in [0, E) ([EC], abstract: each
 * token goes to k of the experts, so its picks are distinct).  Returns 1 when valid. */
static int token_valid(const int32_t *d, int k, int E)
{
    for (int a = 0; a < k; ++a) {
        if (d[a] < 0 || d[a] >= E) return 0;
        for (int b = 0; b < a; ++b)
            if (d[a] == d[b]) return 0;
    }
    return 1;
}

/* Co-activation counts, Ochiai similarity and cross-layer transitions.
 *
 * C_l[i][j] = |{t : i in D_t^l and j in D_t^l}|  ([EC]: pairs of experts
 *   a token picks at once; [CB] Problem/Stage 1: the number of tokens
 *   selecting both experts i and j).  C_l[i][i] = n_i, the expert's load.
 * S_l[i][j] = |A_i & A_j| / sqrt(|A_i| |A_j|) = C_ij / sqrt(C_ii C_jj)
 *   ([CB] "Key Observation": Ochiai over the token sets of two experts);
 *   0 where C_ii C_jj = 0; fp64, then rounded to fp32.
 * M_l[i][j] = |{t : i in D_t^l and j in D_t^{l+1}}|  ([EC]: the experts a
 *   token selects at one layer predict those it selects at the next).
 *
 * ids int32 [L][T][k]; coact uint32 [L][E][E]; ochiai float [L][E][E];
 * trans uint32 [L-1][E][E].  Any output may be NULL. */
int orc_coact(const int32_t *ids, int L, int T, int k, int E,
              uint32_t *coact, float *ochiai, uint32_t *trans)
{
    if (L < 1 || T < 0 || k < 1 || E < 1 || k > E) return ORC_ERR_ARG;
    for (int l = 0; l < L; ++l)
        for (int t = 0; t < T; ++t)
            if (!token_valid(ids + ((size_t)l * T + t) * k, k, E)) return ORC_ERR_DATA;

    const size_t EE = (size_t)E * E;
    uint32_t *C = NULL;
    if (coact || ochiai) {
        C = coact ? coact : (uint32_t *)malloc(sizeof(uint32_t) * EE * L);
        if (!C) return ORC_ERR_ARG;
        memset(C, 0, sizeof(uint32_t) * EE * L);
        for (int l = 0; l < L; ++l) {
            uint32_t *Cl = C + EE * l;
            for (int t = 0; t < T; ++t) {
                const int32_t *d = ids + ((size_t)l * T + t) * k;
                /* every ordered pair (a, b) of the token's picks, a == b included */
                for (int a = 0; a < k; ++a)
                    for (int b = 0; b < k; ++b)
                        Cl[(size_t)d[a] * E + d[b]] += 1;
            }
        }
    }
    if (ochiai) {
        for (int l = 0; l < L; ++l) {
            const uint32_t *Cl = C + EE * l;
            for (int i = 0; i < E; ++i)
                for (int j = 0; j < E; ++j) {
                    double den = (double)Cl[(size_t)i * E + i] * (double)Cl[(size_t)j * E + j];
                    double s = 0.0;
                    if (den > 0.0) s = (double)Cl[(size_t)i * E + j] / sqrt(den);
                    ochiai[EE * l + (size_t)i * E + j] = (float)s;
                }
        }
    }
    if (C && C != coact) free(C);
    if (trans && L > 1) {
        memset(trans, 0, sizeof(uint32_t) * EE * (L - 1));
        for (int l = 0; l + 1 < L; ++l) {
            uint32_t *Ml = trans + EE * l;
            for (int t = 0; t < T; ++t) {
                const int32_t *a = ids + ((size_t)l * T + t) * k;
                const int32_t *b = ids + ((size_t)(l + 1) * T + t) * k;
                for (int x = 0; x < k; ++x)
                    for (int y = 0; y < k; ++y)
                        Ml[(size_t)a[x] * E + b[y]] += 1;
            }
        }
    }
    return ORC_OK;
}

/* Uniform placement ([EPS], uniform listing): device = expert_id // (E/G),
 * defined only when G divides E. */
int orc_place_uniform(int E, int G, int32_t *expert_to_rank)
{
    if (E < 1 || G < 1 || E % G != 0) return ORC_ERR_ARG;
    int per = E / G;
    for (int e = 0; e < E; ++e) expert_to_rank[e] = e / per;
    return ORC_OK;
}

/* Capacity-aware placement ([EPS] "Capacity-Aware Placement"): experts in
 * descending order of load (equal loads: lower id first, a stable sort), each
 * onto the device with the least load so far (ties: the lowest device index).
 * Loads are summed in fp64 here. */
static const double *g_sort_load;
static int cmp_load_desc(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    if (g_sort_load[a] > g_sort_load[b]) return -1;
    if (g_sort_load[a] < g_sort_load[b]) return 1;
    return a < b ? -1 : (a > b);
}

int orc_place_capacity(const double *load, int E, int G, int32_t *expert_to_rank, double *device_load)
{
    if (E < 1 || G < 1) return ORC_ERR_ARG;
    int *order = (int *)malloc(sizeof(int) * E);
    if (!order) return ORC_ERR_ARG;
    for (int e = 0; e < E; ++e) order[e] = e;
    g_sort_load = load;
    qsort(order, E, sizeof(int), cmp_load_desc);
    for (int g = 0; g < G; ++g) device_load[g] = 0.0;
    for (int i = 0; i < E; ++i) {
        int e = order[i], best = 0;
        for (int g = 1; g < G; ++g)
            if (device_load[g] < device_load[best]) best = g;
        expert_to_rank[e] = best;
        device_load[best] += load[e];
    }
    free(order);
    return ORC_OK;
}

/* Ochiai in fp64 without the fp32 rounding, for the placement greedy. */
static double ochiai64(const uint32_t *C, int E, int i, int j)
{
    double den = (double)C[(size_t)i * E + i] * (double)C[(size_t)j * E + j];
    if (den > 0.0) return (double)C[(size_t)i * E + j] / sqrt(den);
    return 0.0;
}

/* Split the experts listed in pool[0..n) (ascending ids) into m groups of
 * n/m, one group at a time: seed with the unassigned expert of largest load
 * C_ee, then repeatedly add the unassigned expert whose summed fp64 Ochiai to
 * the group's members (summed in insertion order) is largest; ties go to the
 * lowest expert id.  group_of[pool index] receives the group number. */
/* Greedy equal-size grouping of pool[0..n) into m groups.  A group is seeded
 * with the unassigned expert of largest load n_e = C_ee and grown by the
 * unassigned expert whose Ochiai summed over the group's members (in joining
 * order) is largest; ties go to the lowest id.  With cap >= 0 (the load
 * tolerance of "Cobalt", "Problem Formulation"), only experts whose load keeps
 * the group's load n_e summed at most cap are candidates; when none is, the
 * lightest unassigned expert joins (ties: lowest id), so every group still
 * gets its n/m experts. */
static void greedy_groups(const uint32_t *C, int E, const int *pool, int n, int m, int *group_of, double cap)
{
    int size = n / m;
    int *taken = (int *)calloc(n, sizeof(int));
    int *members = (int *)malloc(sizeof(int) * size);
    for (int g = 0; g < m; ++g) {
        int best = -1;
        for (int x = 0; x < n; ++x) {
            if (taken[x]) continue;
            if (best < 0 || C[(size_t)pool[x] * E + pool[x]] > C[(size_t)pool[best] * E + pool[best]])
                best = x;
        }
        taken[best] = 1;
        group_of[best] = g;
        members[0] = pool[best];
        uint64_t load = C[(size_t)pool[best] * E + pool[best]];
        for (int cnt = 1; cnt < size; ++cnt) {
            int pick = -1;
            double pick_score = 0.0;
            for (int x = 0; x < n; ++x) {
                if (taken[x]) continue;
                uint64_t nx = C[(size_t)pool[x] * E + pool[x]];
                if (cap >= 0.0 && (double)(load + nx) > cap) continue;
                double s = 0.0;
                for (int q = 0; q < cnt; ++q) s += ochiai64(C, E, pool[x], members[q]);
                if (pick < 0 || s > pick_score) { pick = x; pick_score = s; }
            }
            if (pick < 0) {   /* nothing fits: the lightest */
                for (int x = 0; x < n; ++x) {
                    if (taken[x]) continue;
                    if (pick < 0 || C[(size_t)pool[x] * E + pool[x]] < C[(size_t)pool[pick] * E + pool[pick]])
                        pick = x;
                }
            }
            taken[pick] = 1;
            group_of[pick] = g;
            members[cnt] = pool[pick];
            load += C[(size_t)pool[pick] * E + pool[pick]];
        }
    }
    free(members);
    free(taken);
}

/* Correlated placement ([EC]: experts often selected together go on the same
 * GPU).  The pages give the goal, not an algorithm; this is the greedy reading:
 * with more than one node, first group the experts into G/rpn node groups of
 * E/(G/rpn), then each node's experts into rpn rank groups of E/G; node group
 * q and its rank group u map to rank q*rpn + u.  coact is one layer's
 * uint32 [E][E] count matrix.  With eps >= 0 every node group's load is kept
 * to at most (1+eps) W / (G/rpn) and every rank group's to (1+eps) W / G
 * where possible, W the total load; eps < 0: no load limit. */
int orc_place_correlated_capped(const uint32_t *coact, int E, int G, int rpn, double eps, int32_t *expert_to_rank)
{
    if (E < 1 || G < 1 || rpn < 1 || G % rpn != 0 || E % G != 0) return ORC_ERR_ARG;
    int nodes = G / rpn;
    double W = 0.0;
    for (int e = 0; e < E; ++e) W += (double)coact[(size_t)e * E + e];
    double cap_node = eps >= 0.0 ? (1.0 + eps) * W / nodes : -1.0;
    double cap_rank = eps >= 0.0 ? (1.0 + eps) * W / G : -1.0;
    int *all = (int *)malloc(sizeof(int) * E);
    int *node_of = (int *)malloc(sizeof(int) * E);
    int *pool = (int *)malloc(sizeof(int) * E);
    int *grp = (int *)malloc(sizeof(int) * E);
    for (int e = 0; e < E; ++e) all[e] = e;
    greedy_groups(coact, E, all, E, nodes, node_of, cap_node);
    for (int q = 0; q < nodes; ++q) {
        int n = 0;
        for (int e = 0; e < E; ++e)
            if (node_of[e] == q) pool[n++] = e;
        greedy_groups(coact, E, pool, n, rpn, grp, cap_rank);
        for (int x = 0; x < n; ++x) expert_to_rank[pool[x]] = q * rpn + grp[x];
    }
    free(all); free(node_of); free(pool); free(grp);
    return ORC_OK;
}

int orc_place_correlated(const uint32_t *coact, int E, int G, int rpn, int32_t *expert_to_rank)
{
    return orc_place_correlated_capped(coact, E, G, rpn, -1.0, expert_to_rank);
}

/* One dispatched row: token t sent to rank dst, from source rank src. */
typedef struct { int32_t dst, src, t; } orc_row;

static int cmp_row(const void *pa, const void *pb)
{
    const orc_row *a = (const orc_row *)pa, *b = (const orc_row *)pb;
    if (a->dst != b->dst) return a->dst < b->dst ? -1 : 1;
    if (a->src != b->src) return a->src < b->src ? -1 : 1;
    return a->t < b->t ? -1 : (a->t > b->t);
}

/* Deduplicated dispatch plan ([EC]: a dispatcher that sends each token to
 * each GPU once; [CB] "Problem Formulation": V counts each remote node a token
 * must reach once, given node-level deduplication).
 *
 * p(e) = expert_to_rank[e]; s_t = src_rank[t], or t / (T/G) when src_rank is
 * NULL; N(r) = r / rpn.  Rows are the pairs (t, r) with r in {p(e) : e in D_t},
 * ordered by (r, s_t, t).  Outputs:
 *   dest_mask[t]      bit r set when the token has a row for rank r (G <= 64)
 *   counts[s][r]      rows from source rank s to rank r
 *   offsets[r*G + s]  first row of the (r, s) segment; offsets[G*G] = R
 *   row_token[i], row_jmask[i] (bit j set when p(e_tj) is the row's rank)
 *   row_of[t][j]      the row that carries (t, e_tj)
 *   summary[5] = { R, R_remote (rows with r != s_t),
 *                  local = #{(t,j) : p(e_tj) = s_t},
 *                  V = sum_t |{N(p(e)) : e in D_t} \ {N(s_t)}|,  T*k }
 * row_token / row_jmask must hold T*k entries. */
/* The rank serving pick j of token t: pick_rank[t][j] when given (replicated
 * experts, see orc_assign_replicas), else p(e_tj). */
static int serving_rank(const int32_t *ids, const int32_t *expert_to_rank, const int32_t *pick_rank,
                        int k, int t, int j)
{
    return pick_rank ? pick_rank[(size_t)t * k + j] : expert_to_rank[ids[(size_t)t * k + j]];
}

static int plan_impl(const int32_t *ids, int T, int k, int E, int G, int rpn,
                     const int32_t *expert_to_rank, const int32_t *pick_rank, const int32_t *src_rank,
                     uint64_t *dest_mask, int32_t *counts, int32_t *offsets,
                     int32_t *row_token, uint8_t *row_jmask, int32_t *row_of, int64_t *summary)
{
    if (T < 0 || k < 1 || k > 8 || E < 1 || k > E || G < 1 || G > 64 || rpn < 1 || G % rpn != 0)
        return ORC_ERR_ARG;
    if (!src_rank && (T % G != 0)) return ORC_ERR_ARG;
    if (!pick_rank)
        for (int e = 0; e < E; ++e)
            if (expert_to_rank[e] < 0 || expert_to_rank[e] >= G) return ORC_ERR_DATA;
    for (int t = 0; t < T; ++t) {
        if (!token_valid(ids + (size_t)t * k, k, E)) return ORC_ERR_DATA;
        if (src_rank && (src_rank[t] < 0 || src_rank[t] >= G)) return ORC_ERR_DATA;
        if (pick_rank)
            for (int j = 0; j < k; ++j)
                if (pick_rank[(size_t)t * k + j] < 0 || pick_rank[(size_t)t * k + j] >= G) return ORC_ERR_DATA;
    }
    int nodes = G / rpn;
    orc_row *rows = (orc_row *)malloc(sizeof(orc_row) * ((size_t)T * k + 1));
    if (!rows) return ORC_ERR_ARG;
    size_t R = 0;
    int64_t local = 0, V = 0;
    for (int t = 0; t < T; ++t) {
        int s = src_rank ? src_rank[t] : t / (T / G);
        int want[64] = {0}, node_hit[64] = {0};
        for (int j = 0; j < k; ++j) {
            int r = serving_rank(ids, expert_to_rank, pick_rank, k, t, j);
            want[r] = 1;
            node_hit[r / rpn] = 1;
            if (r == s) local += 1;
        }
        uint64_t m = 0;
        for (int r = 0; r < G; ++r)
            if (want[r]) {
                m |= (uint64_t)1 << r;
                rows[R].dst = r; rows[R].src = s; rows[R].t = t;
                ++R;
            }
        dest_mask[t] = m;
        for (int q = 0; q < nodes; ++q)
            if (node_hit[q] && q != s / rpn) V += 1;
    }
    qsort(rows, R, sizeof(orc_row), cmp_row);
    memset(counts, 0, sizeof(int32_t) * G * G);
    int64_t remote = 0;
    for (size_t i = 0; i < R; ++i) {
        int t = rows[i].t, r = rows[i].dst;
        uint8_t jm = 0;
        for (int j = 0; j < k; ++j)
            if (serving_rank(ids, expert_to_rank, pick_rank, k, t, j) == r) {
                jm |= (uint8_t)(1u << j);
                row_of[(size_t)t * k + j] = (int32_t)i;
            }
        row_token[i] = t;
        row_jmask[i] = jm;
        counts[rows[i].src * G + r] += 1;
        if (r != rows[i].src) remote += 1;
    }
    int32_t run = 0;
    for (int r = 0; r < G; ++r)
        for (int s = 0; s < G; ++s) {
            offsets[r * G + s] = run;
            run += counts[s * G + r];
        }
    offsets[G * G] = run;
    summary[0] = (int64_t)R;
    summary[1] = remote;
    summary[2] = local;
    summary[3] = V;
    summary[4] = (int64_t)T * k;
    free(rows);
    return ORC_OK;
}

int orc_plan(const int32_t *ids, int T, int k, int E, int G, int rpn,
             const int32_t *expert_to_rank, const int32_t *src_rank,
             uint64_t *dest_mask, int32_t *counts, int32_t *offsets,
             int32_t *row_token, uint8_t *row_jmask, int32_t *row_of, int64_t *summary)
{
    return plan_impl(ids, T, k, E, G, rpn, expert_to_rank, NULL, src_rank, dest_mask, counts, offsets,
                     row_token, row_jmask, row_of, summary);
}

/* The same plan with the serving rank of every (token, pick) given. */
int orc_plan_ranks(const int32_t *ids, int T, int k, int E, int G, int rpn,
                   const int32_t *pick_rank, const int32_t *src_rank,
                   uint64_t *dest_mask, int32_t *counts, int32_t *offsets,
                   int32_t *row_token, uint8_t *row_jmask, int32_t *row_of, int64_t *summary)
{
    return plan_impl(ids, T, k, E, G, rpn, NULL, pick_rank, src_rank, dest_mask, counts, offsets,
                     row_token, row_jmask, row_of, summary);
}

/* Row permute into the rank-major send buffer: send[i] = x[row_token[i]]. */
int orc_permute(const void *x, int elem_bytes, int T, int d, const int32_t *row_token, int64_t R, void *send)
{
    size_t rowB = (size_t)elem_bytes * d;
    for (int64_t i = 0; i < R; ++i) {
        if (row_token[i] < 0 || row_token[i] >= T) return ORC_ERR_DATA;
        memcpy((char *)send + rowB * i, (const char *)x + rowB * row_token[i], rowB);
    }
    return ORC_OK;
}

static double load_elem(const void *Y, int y_is_bf16, size_t i)
{
    if (y_is_bf16) {
        uint32_t u = (uint32_t)((const uint16_t *)Y)[i] << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
    return (double)((const float *)Y)[i];
}

/* Weighted combine, the inverse of dispatch ([EC]: tokens are dispatched to
 * their experts and the results combined; [CE] footnote 3: the hidden-state
 * combine): out[t][c] = sum_j w[t][j] * Y[idx[t][j]][c], summed in fp64 in j
 * order. */
int orc_combine(const void *Y, int y_is_bf16, int64_t R_max, int d, const int32_t *idx,
                const float *w, int T, int k, double *out)
{
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j)
            if (idx[(size_t)t * k + j] < 0 || idx[(size_t)t * k + j] >= R_max) return ORC_ERR_DATA;
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                size_t row = (size_t)idx[(size_t)t * k + j];
                acc += (double)w[(size_t)t * k + j] * load_elem(Y, y_is_bf16, row * d + c);
            }
            out[(size_t)t * d + c] = acc;
        }
    return ORC_OK;
}

/* Rank scores for token shuffling ([EC]: move each token to the GPU
 * predicted to hold its next-layer experts):
 * rank_score[e][r] = sum over e' with p_{l+1}(e') = r of M_l[e][e']. */
int orc_rank_score(const uint32_t *trans, const int32_t *next_expert_to_rank, int E, int G, uint32_t *rank_score)
{
    for (int e = 0; e < E; ++e)
        if (next_expert_to_rank[e] < 0 || next_expert_to_rank[e] >= G) return ORC_ERR_DATA;
    for (int e = 0; e < E; ++e) {
        for (int r = 0; r < G; ++r) {
            uint64_t s = 0;
            for (int f = 0; f < E; ++f)
                if (next_expert_to_rank[f] == r) s += trans[(size_t)e * E + f];
            if (s > 0xFFFFFFFFull) return ORC_ERR_DATA;
            rank_score[(size_t)e * G + r] = (uint32_t)s;
        }
    }
    return ORC_OK;
}

/* Shuffle target: target[t] = argmax_r sum_j rank_score[e_tj][r], the lowest
 * r among equal scores. */
int orc_shuffle_targets(const int32_t *ids, int T, int k, int E, int G, const uint32_t *rank_score, int32_t *target)
{
    for (int t = 0; t < T; ++t) {
        const int32_t *d = ids + (size_t)t * k;
        if (!token_valid(d, k, E)) return ORC_ERR_DATA;
        int best = 0;
        uint64_t best_s = 0;
        for (int r = 0; r < G; ++r) {
            uint64_t s = 0;
            for (int j = 0; j < k; ++j) s += rank_score[(size_t)d[j] * G + r];
            if (r == 0 || s > best_s) { best = r; best_s = s; }
        }
        target[t] = best;
    }
    return ORC_OK;
}

/* Capacity-balanced shuffle target.  [EC] moves each token to the GPU
 * predicted to hold its next-layer experts during the reduce-scatter that
 * follows attention; a reduce-scatter hands every rank an equal shard, so here
 * every rank receives at most `capacity` tokens (exactly T/G when T =
 * G*capacity).  Reading taken: score S_t(r) = sum_j rank_score[e_tj][r] as in
 * the unconstrained target; all (t, r) pairs are taken in the order S desc,
 * then t asc, then r asc, and a pair is accepted when t has no rank yet and r
 * holds fewer than `capacity` tokens.  With capacity >= T this is the
 * unconstrained argmax. */
typedef struct { uint64_t s; int32_t t, r; } orc_pair;

static int cmp_pair(const void *pa, const void *pb)
{
    const orc_pair *a = (const orc_pair *)pa, *b = (const orc_pair *)pb;
    if (a->s != b->s) return a->s > b->s ? -1 : 1;
    if (a->t != b->t) return a->t < b->t ? -1 : 1;
    if (a->r != b->r) return a->r < b->r ? -1 : 1;
    return 0;
}

int orc_shuffle_balanced(const int32_t *ids, int T, int k, int E, int G, const uint32_t *rank_score,
                         int capacity, int32_t *target)
{
    if (T < 0 || k < 1 || G < 1 || capacity < 0 || (int64_t)G * capacity < T) return ORC_ERR_ARG;
    for (int t = 0; t < T; ++t)
        if (!token_valid(ids + (size_t)t * k, k, E)) return ORC_ERR_DATA;
    size_t n = (size_t)T * G;
    orc_pair *pairs = (orc_pair *)malloc((n ? n : 1) * sizeof(orc_pair));
    int32_t *held = (int32_t *)calloc((size_t)G, sizeof(int32_t));
    if (!pairs || !held) { free(pairs); free(held); return ORC_ERR_ARG; }
    for (int t = 0; t < T; ++t) {
        const int32_t *d = ids + (size_t)t * k;
        for (int r = 0; r < G; ++r) {
            uint64_t s = 0;
            for (int j = 0; j < k; ++j) s += rank_score[(size_t)d[j] * G + r];
            orc_pair *p = &pairs[(size_t)t * G + r];
            p->s = s; p->t = t; p->r = r;
        }
        target[t] = -1;
    }
    qsort(pairs, n, sizeof(orc_pair), cmp_pair);
    for (size_t i = 0; i < n; ++i) {
        const orc_pair *p = &pairs[i];
        if (target[p->t] < 0 && held[p->r] < capacity) {
            target[p->t] = p->r;
            held[p->r] += 1;
        }
    }
    free(pairs);
    free(held);
    return ORC_OK;
}

/* Exponential moving averages of the co-activation counts ("Cobalt", "Key
 * Observation": the planner keeps an EMA of the tokens selecting both experts
 * i and j, and of each expert's load, and evaluates Ochiai on them).  Per cell,
 * in fp64: ema_out = alpha * C + (1 - alpha) * ema_in, or C when ema_in is
 * NULL (the first batch); the load EMA is the diagonal.  Ochiai on the
 * averages: ema_ij / sqrt(ema_ii * ema_jj), rounded once to fp32, 0 when the
 * product is 0. */
int orc_coact_ema(const uint32_t *coact, int L, int E, double alpha, const double *ema_in, double *ema_out,
                  float *ochiai)
{
    if (L < 1 || E < 1 || !(alpha >= 0.0 && alpha <= 1.0)) return ORC_ERR_ARG;
    size_t EE = (size_t)E * E;
    for (size_t c = 0; c < (size_t)L * EE; ++c) {
        double x = (double)coact[c];
        if (ema_in) {
            double a = alpha * x;
            double b = (1.0 - alpha) * ema_in[c];
            ema_out[c] = a + b;
        } else {
            ema_out[c] = x;
        }
    }
    if (ochiai) {
        for (int l = 0; l < L; ++l) {
            const double *m = ema_out + (size_t)l * EE;
            for (int i = 0; i < E; ++i)
                for (int j = 0; j < E; ++j) {
                    double den = m[(size_t)i * E + i] * m[(size_t)j * E + j];
                    ochiai[(size_t)l * EE + (size_t)i * E + j] = den > 0.0 ? (float)(m[(size_t)i * E + j] / sqrt(den)) : 0.0f;
                }
        }
    }
    return ORC_OK;
}

/* ---- receiver-side pre-reduced combine (a NEXT row of the path) ----------- */

/* Gate dispatch ([CE] footnote 3: the routed probabilities are dispatched with
 * the hidden states).  Row i carries token t = row_token[i]; for each pick j
 * of t whose expert lives on the row's rank (bit j of row_jmask[i]) the row
 * carries (e_tj, w_tj), else (-1, 0). */
int orc_dispatch_gates(const int32_t *ids, const float *w, int T, int k, const int32_t *row_token,
                       const uint8_t *row_jmask, int64_t R, int32_t *send_e, float *send_w)
{
    for (int64_t i = 0; i < R; ++i) {
        int t = row_token[i];
        if (t < 0 || t >= T) return ORC_ERR_DATA;
        for (int j = 0; j < k; ++j) {
            int on = (row_jmask[i] >> j) & 1;
            send_e[i * k + j] = on ? ids[(size_t)t * k + j] : -1;
            send_w[i * k + j] = on ? w[(size_t)t * k + j] : 0.0f;
        }
    }
    return ORC_OK;
}

/* The receiving rank applies each of the row's experts and sums their
 * outputs weighted by the dispatched gates, returning one row per (token,
 * rank) ([EC]: dispatch, then combine; here the weighting moves to the
 * receiver).  Stand-in experts: expert e maps a row x to scale[e] * x.
 *   y[i][c] = sum_j send_w[i][j] * scale[send_e[i][j]] * send[i][c]
 * over the j with send_e[i][j] >= 0, in fp64. */
int orc_expert_reduce(const void *send, int is_bf16, int64_t R, int d, const int32_t *send_e,
                      const float *send_w, int k, const float *scale, int E, double *y)
{
    for (int64_t i = 0; i < R; ++i)
        for (int j = 0; j < k; ++j)
            if (send_e[i * k + j] >= E) return ORC_ERR_DATA;
    for (int64_t i = 0; i < R; ++i)
        for (int c = 0; c < d; ++c) {
            double x = load_elem(send, is_bf16, (size_t)i * d + c), acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = send_e[i * k + j];
                if (e >= 0) acc += (double)send_w[i * k + j] * (double)scale[e] * x;
            }
            y[(size_t)i * d + c] = acc;
        }
    return ORC_OK;
}

/* The source sums the pre-reduced rows of each token once each:
 * out[t][c] = sum over the distinct rows r in {row_of[t][j]} of y[r][c] (fp64,
 * y given as float32 or bf16 bits). */
int orc_combine_rows(const void *y, int is_bf16, int64_t R_max, int d, const int32_t *row_of, int T, int k,
                     double *out)
{
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j)
            if (row_of[(size_t)t * k + j] < 0 || row_of[(size_t)t * k + j] >= R_max) return ORC_ERR_DATA;
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int r = row_of[(size_t)t * k + j], seen = 0;
                for (int q = 0; q < j; ++q) seen |= row_of[(size_t)t * k + q] == r;
                if (!seen) acc += load_elem(y, is_bf16, (size_t)r * d + c);
            }
            out[(size_t)t * d + c] = acc;
        }
    return ORC_OK;
}

/* ---- expert replicas and communication-aware task assignment ([CB]) ------- */

/* Replica layout.  [CB] "Problem Formulation": P_r is the set of experts with
 * a replica on rank r, every expert has at least one, |P_r| <= (1+rho)E/G;
 * "Two-Stage Expert Layout Planner" maximises co-activation within nodes.  The
 * page gives no algorithm; this is the greedy reading: start from a placement
 * with one replica per expert (expert_to_rank), give every rank room for
 * `extra` more experts, and repeatedly add the replica (e, node q) of largest
 * score(e, q) = sum over the experts e' placed on q of C[e][e'] (e not yet on
 * q; ties: lower e, then lower q) on the rank of q with the most free room
 * (ties: lowest rank), until no rank has room or no candidate scores above 0.
 * Output: replica_rank[e][0..n_rep[e]) (the original rank first, then in the
 * order added), unused slots -1; max_rep = 1 + G/rpn slots per expert. */
int orc_place_replicas(const uint32_t *coact, int E, int G, int rpn, const int32_t *expert_to_rank, int extra,
                       int32_t *replica_rank, int32_t *n_rep)
{
    if (E < 1 || G < 1 || rpn < 1 || G % rpn != 0 || extra < 0) return ORC_ERR_ARG;
    const int nodes = G / rpn, max_rep = 1 + nodes;
    int *room = (int *)malloc(sizeof(int) * G);
    int *on_node = (int *)calloc((size_t)E * nodes, sizeof(int));
    uint64_t *score = (uint64_t *)calloc((size_t)E * nodes, sizeof(uint64_t));
    int *used = (int *)calloc((size_t)E * nodes, sizeof(int));
    for (int r = 0; r < G; ++r) room[r] = extra;
    for (int e = 0; e < E; ++e) {
        if (expert_to_rank[e] < 0 || expert_to_rank[e] >= G) { free(room); free(on_node); free(score); free(used); return ORC_ERR_DATA; }
        for (int q = 0; q < max_rep; ++q) replica_rank[(size_t)e * max_rep + q] = -1;
        replica_rank[(size_t)e * max_rep] = expert_to_rank[e];
        n_rep[e] = 1;
        on_node[(size_t)e * nodes + expert_to_rank[e] / rpn] = 1;
    }
    for (int e = 0; e < E; ++e)
        for (int f = 0; f < E; ++f)
            if (f != e) score[(size_t)e * nodes + expert_to_rank[f] / rpn] += coact[(size_t)e * E + f];
    for (;;) {
        int be = -1, bq = -1;
        uint64_t bs = 0;
        for (int e = 0; e < E; ++e)
            for (int q = 0; q < nodes; ++q) {
                if (on_node[(size_t)e * nodes + q] || used[(size_t)e * nodes + q]) continue;
                uint64_t sc = score[(size_t)e * nodes + q];
                if (sc == 0) continue;
                int has_room = 0;
                for (int r = q * rpn; r < (q + 1) * rpn; ++r) has_room |= room[r] > 0;
                if (!has_room) continue;
                if (be < 0 || sc > bs) { be = e; bq = q; bs = sc; }
            }
        if (be < 0) break;
        int br = -1;
        for (int r = bq * rpn; r < (bq + 1) * rpn; ++r)
            if (room[r] > 0 && (br < 0 || room[r] > room[br])) br = r;
        room[br] -= 1;
        used[(size_t)be * nodes + bq] = 1;
        on_node[(size_t)be * nodes + bq] = 1;
        replica_rank[(size_t)be * max_rep + n_rep[be]] = br;
        n_rep[be] += 1;
    }
    free(room); free(on_node); free(score); free(used);
    return ORC_OK;
}

/* Communication-aware task assignment of one token ([CB]: each token goes to as
 * few remote nodes as it can; V counts, per token, the remote
 * nodes its tasks reach).  Token with picks d[0..k) and source rank s (node
 * ns = s / rpn).  A replica of a pick's expert may serve it when its rank is
 * open (bit r of open_ranks), or when none of that expert's replicas is open.
 * Among all choices of one such replica per pick, the fewest distinct nodes
 * other than ns -- found as the smallest node set S (ties: smallest as a bit
 * pattern) such that every pick's expert has a usable replica on ns or in S.
 * Then, pick by pick in j order, among the usable ranks hosting the expert on
 * ns (or, if none, on the nodes of S): rank s if it is one of them; else the
 * lowest of them that an earlier pick of the token already uses (no new row);
 * else the lowest of them.  Writes pick_rank[0..k); returns |S|, or -1 when
 * an expert has no replica at all. */
static int assign_token(const int32_t *d, int k, int s, int rpn, int nodes, const int32_t *replica_rank,
                        const int32_t *n_rep, uint64_t open_ranks, int32_t *pick_rank)
{
    const int max_rep = 1 + nodes, ns = s / rpn;
    int any_open[8];
    for (int j = 0; j < k; ++j) {
        any_open[j] = 0;
        for (int q = 0; q < n_rep[d[j]]; ++q)
            if ((open_ranks >> replica_rank[(size_t)d[j] * max_rep + q]) & 1) any_open[j] = 1;
    }
#define USABLE(j, r) (!any_open[j] || ((open_ranks >> (r)) & 1))
    int best_size = nodes + 1, best_set = 0;
    for (int set = 0; set < (1 << nodes); ++set) {
        if ((set >> ns) & 1) continue;
        int ok = 1;
        for (int j = 0; j < k && ok; ++j) {
            int covered = 0;
            for (int q = 0; q < n_rep[d[j]]; ++q) {
                int r = replica_rank[(size_t)d[j] * max_rep + q], node = r / rpn;
                if (USABLE(j, r) && (node == ns || ((set >> node) & 1))) covered = 1;
            }
            ok = covered;
        }
        if (!ok) continue;
        int size = 0;
        for (int q = 0; q < nodes; ++q) size += (set >> q) & 1;
        if (size < best_size) { best_size = size; best_set = set; }
    }
    if (best_size > nodes) return -1;   /* an expert without replicas */
    for (int j = 0; j < k; ++j) {
        int any_ns = 0;
        for (int q = 0; q < n_rep[d[j]]; ++q) {
            int r = replica_rank[(size_t)d[j] * max_rep + q];
            if (USABLE(j, r) && r / rpn == ns) any_ns = 1;
        }
        int pick = -1, used_pick = -1, low = -1;
        for (int q = 0; q < n_rep[d[j]]; ++q) {
            int r = replica_rank[(size_t)d[j] * max_rep + q];
            if (!USABLE(j, r)) continue;
            int allowed = any_ns ? (r / rpn == ns) : ((best_set >> (r / rpn)) & 1);
            if (!allowed) continue;
            if (r == s) pick = r;
            int used = 0;
            for (int q2 = 0; q2 < j; ++q2) used |= pick_rank[q2] == r;
            if (used && (used_pick < 0 || r < used_pick)) used_pick = r;
            if (low < 0 || r < low) low = r;
        }
        if (pick < 0) pick = used_pick >= 0 ? used_pick : low;
        pick_rank[j] = pick;
    }
#undef USABLE
    return best_size;
}

static int check_replica_table(int E, int G, int max_rep, const int32_t *replica_rank, const int32_t *n_rep)
{
    for (int e = 0; e < E; ++e) {
        if (n_rep[e] < 0 || n_rep[e] > max_rep) return ORC_ERR_DATA;
        for (int q = 0; q < n_rep[e]; ++q)
            if (replica_rank[(size_t)e * max_rep + q] < 0 || replica_rank[(size_t)e * max_rep + q] >= G)
                return ORC_ERR_DATA;
    }
    return ORC_OK;
}

/* Every rank open: the assignment of [CB]'s fewest-remote-nodes rule
 * alone.  Requires G/rpn <= 8.  pick_rank [T][k] out; n_remote [T] out (|S|,
 * may be NULL). */
int orc_assign_replicas(const int32_t *ids, int T, int k, int E, int G, int rpn, const int32_t *replica_rank,
                        const int32_t *n_rep, const int32_t *src_rank, int32_t *pick_rank, int32_t *n_remote)
{
    if (T < 0 || k < 1 || k > 8 || G < 1 || G > 64 || rpn < 1 || G % rpn != 0 || G / rpn > 8) return ORC_ERR_ARG;
    if (!src_rank && T % G != 0) return ORC_ERR_ARG;
    const int nodes = G / rpn;
    if (check_replica_table(E, G, 1 + nodes, replica_rank, n_rep) != ORC_OK) return ORC_ERR_DATA;
    for (int t = 0; t < T; ++t) {
        const int32_t *d = ids + (size_t)t * k;
        if (!token_valid(d, k, E)) return ORC_ERR_DATA;
        const int s = src_rank ? src_rank[t] : t / (T / G);
        if (s < 0 || s >= G) return ORC_ERR_DATA;
        const int size = assign_token(d, k, s, rpn, nodes, replica_rank, n_rep, ~(uint64_t)0, pick_rank + (size_t)t * k);
        if (size < 0) return ORC_ERR_DATA;
        if (n_remote) n_remote[t] = size;
    }
    return ORC_OK;
}

/* The per-rank workload cap of [CB] "Problem Formulation": the tasks rank r
 * runs, sum_e w_r^e, at most (1 + eps) K T / G.  cap = floor((1 + eps) * (T k)
 * / G) in fp64 (one multiply, one divide, IEEE rounding); INT64_MAX when that
 * is 9e18 or more (eps = inf: no cap). */
int64_t orc_load_cap(int T, int k, int G, double eps)
{
    const double c = floor((1.0 + eps) * (double)((int64_t)T * k) / (double)G);
    return c >= 9.0e18 ? INT64_MAX : (int64_t)c;
}

/* Assignment under the load tolerance eps ([CB] "Problem Formulation": the
 * fewest remote nodes per token, and sum_e w_r^e <= (1 + eps) K T / G per
 * rank).  The page states the constraint, not how to meet it; the reading
 * taken: tokens in id order; before token t a rank whose load (tasks already
 * assigned to it) has reached cap = orc_load_cap(T, k, G, eps) is closed, and
 * t is assigned as in assign_token over the open ranks.  A pick whose expert
 * has no open replica may use all of its replicas (the cap gives way, not the
 * task), and a token may take a rank past the cap by at most k - 1 tasks.
 * pick_rank [T][k] out; n_remote [T] out or NULL; rank_load [G] out or NULL
 * (tasks per rank). */
int orc_assign_replicas_capped(const int32_t *ids, int T, int k, int E, int G, int rpn,
                               const int32_t *replica_rank, const int32_t *n_rep, const int32_t *src_rank,
                               double eps, int32_t *pick_rank, int32_t *n_remote, int64_t *rank_load)
{
    if (T < 0 || k < 1 || k > 8 || G < 1 || G > 64 || rpn < 1 || G % rpn != 0 || G / rpn > 8) return ORC_ERR_ARG;
    if (!(eps >= 0.0)) return ORC_ERR_ARG;
    if (!src_rank && T % G != 0) return ORC_ERR_ARG;
    const int nodes = G / rpn;
    if (check_replica_table(E, G, 1 + nodes, replica_rank, n_rep) != ORC_OK) return ORC_ERR_DATA;
    const int64_t cap = orc_load_cap(T, k, G, eps);
    int64_t load[64] = {0};
    for (int t = 0; t < T; ++t) {
        const int32_t *d = ids + (size_t)t * k;
        if (!token_valid(d, k, E)) return ORC_ERR_DATA;
        const int s = src_rank ? src_rank[t] : t / (T / G);
        if (s < 0 || s >= G) return ORC_ERR_DATA;
        uint64_t open_ranks = 0;
        for (int r = 0; r < G; ++r)
            if (load[r] < cap) open_ranks |= (uint64_t)1 << r;
        const int size = assign_token(d, k, s, rpn, nodes, replica_rank, n_rep, open_ranks, pick_rank + (size_t)t * k);
        if (size < 0) return ORC_ERR_DATA;
        for (int j = 0; j < k; ++j) load[pick_rank[(size_t)t * k + j]] += 1;
        if (n_remote) n_remote[t] = size;
    }
    if (rank_load)
        for (int r = 0; r < G; ++r) rank_load[r] = load[r];
    return ORC_OK;
}

/* Tasks each rank serves under a one-replica placement: load[r] = sum of n_e
 * over the experts e with expert_to_rank[e] = r, n_e = C_ee the tokens that
 * pick e ([EPS] "Capacity-Aware Placement": a device's load is the sum of its
 * experts' loads).  coact [E][E] (only the diagonal is read); load [G] out. */
int orc_rank_loads(const uint32_t *coact, int E, int G, const int32_t *expert_to_rank, int64_t *load)
{
    if (E < 1 || G < 1) return ORC_ERR_ARG;
    for (int r = 0; r < G; ++r) load[r] = 0;
    for (int e = 0; e < E; ++e) {
        if (expert_to_rank[e] < 0 || expert_to_rank[e] >= G) return ORC_ERR_DATA;
        load[expert_to_rank[e]] += coact[(size_t)e * E + e];
    }
    return ORC_OK;
}

/* Expert parallelism over W devices ([EC] abstract: each token is sent to each
 * GPU once; reading taken: device h hosts ranks h*Gl .. h*Gl+Gl-1, Gl = G/W,
 * and its receive buffer holds its ranks' rows in the one-device order --
 * destination rank, source rank, token).  From every source rank's row counts
 * counts_all[s][r] and device me's own plan offsets (its tokens only), the
 * route of each of me's segments (r, s), s among me's ranks:
 *   route[0]       rows device me receives,
 *   route[1+i]     first local row of segment i = r*Gl + (s - me*Gl),
 *   route[1+P]     me's row count R (P = G*Gl segments),
 *   route[P+2+i]   row of the segment's first row in device r/Gl's buffer
 *                  minus its local row.
 * Written as the definition: the one-device offsets are the running sum of
 * the counts in (r, s) order; a device's buffer starts at the offset of its
 * first rank. */
int orc_ep_routes(const int32_t *counts_all, const int32_t *offsets, int G, int W, int me, int64_t *route)
{
    if (G < 1 || G > 64 || W < 1 || G % W || me < 0 || me >= W) return ORC_ERR_ARG;
    const int Gl = G / W, P = G * Gl;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(G * G + 1));
    if (!off) return ORC_ERR_ARG;
    int64_t run = 0;
    for (int r = 0; r < G; ++r)
        for (int s = 0; s < G; ++s) {
            off[r * G + s] = run;
            run += counts_all[s * G + r];
        }
    off[G * G] = run;
    route[0] = off[(me + 1) * Gl * G] - off[me * Gl * G];
    for (int i = 0; i < P; ++i) {
        const int r = i / Gl, s = me * Gl + i % Gl;
        const int64_t first_local = offsets[r * G + s];
        const int64_t first_global = off[r * G + s] - off[(r / Gl) * Gl * G];
        route[1 + i] = first_local;
        route[P + 2 + i] = first_global - first_local;
    }
    route[1 + P] = offsets[G * G];
    free(off);
    return ORC_OK;
}

/* Rows crossing devices in the exchange, as the definition: with the G ranks
 * on W devices (G/W consecutive ranks each), a row from source rank s to rank
 * r crosses when s and r are on different devices.  sent[h]: rows whose
 * source is on device h and rank elsewhere; received[h]: the reverse. */
int orc_ep_exchange_rows(const int32_t *counts_all, int G, int W, int64_t *sent, int64_t *received)
{
    if (G < 1 || G > 64 || W < 1 || G % W) return ORC_ERR_ARG;
    const int Gl = G / W;
    for (int h = 0; h < W; ++h) { sent[h] = 0; received[h] = 0; }
    for (int s = 0; s < G; ++s)
        for (int r = 0; r < G; ++r) {
            if (counts_all[s * G + r] < 0) return ORC_ERR_DATA;
            if (s / Gl == r / Gl) continue;
            sent[s / Gl] += counts_all[s * G + r];
            received[r / Gl] += counts_all[s * G + r];
        }
    return ORC_OK;
}

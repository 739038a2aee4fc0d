// Expert placement on the host (run once per re-layout, not per step).
//
// Uniform: "Expert Parallelism > Expert Placement Strategies", the uniform
// listing (device = expert_id // (E/G)).  Capacity-aware: same page,
// "Capacity-Aware Placement" (largest expected load first, onto the least
// loaded device).  Correlated: "Expert Coupling in MoE Pretraining", abstract
// (experts often selected together share a GPU) -- the page gives the goal;
// this is a greedy equal-size grouping by fp64 Ochiai, node level first when
// ranks span several nodes ("Cobalt": a token crosses to a remote node once,
// so co-activated experts should share nodes as well as ranks).
//
// The greedy keeps, for every unassigned expert, its running sum of Ochiai to
// the current group's members; each new member adds its column once, so the
// sum is accumulated in the order members joined (O(E^2) per level).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

#include "moe_coact.h"

namespace {

double ochiai64(const uint32_t *C, int E, int i, int j)
{
    const double den = (double)C[(size_t)i * E + i] * (double)C[(size_t)j * E + j];
    if (den > 0.0) return (double)C[(size_t)i * E + j] / std::sqrt(den);
    return 0.0;
}

// Split `pool` (ascending expert ids) into m groups of pool.size()/m.  With
// cap >= 0 a group only admits experts that keep its load (sum of C_ee) at
// most cap; when none does, the lightest unassigned expert joins (ties: lowest
// id).  Running Ochiai sums per candidate, in the members' joining order.
std::vector<int> greedy_split(const uint32_t *C, int E, const std::vector<int> &pool, int m, double cap)
{
    const int n = (int)pool.size();
    const int size = n / m;
    std::vector<int> group(n, -1);
    std::vector<double> score(n);
    auto load_of = [&](int x) { return (uint64_t)C[(size_t)pool[x] * E + pool[x]]; };
    for (int g = 0; g < m; ++g) {
        int seed = -1;
        for (int x = 0; x < n; ++x) {
            if (group[x] >= 0) continue;
            if (seed < 0 || load_of(x) > load_of(seed)) seed = x;
        }
        group[seed] = g;
        uint64_t load = load_of(seed);
        for (int x = 0; x < n; ++x) score[x] = 0.0;
        int last = seed;
        for (int cnt = 1; cnt < size; ++cnt) {
            int pick = -1;
            for (int x = 0; x < n; ++x) {
                if (group[x] >= 0) continue;
                score[x] += ochiai64(C, E, pool[x], pool[last]);
                if (cap >= 0.0 && (double)(load + load_of(x)) > cap) continue;
                if (pick < 0 || score[x] > score[pick]) pick = x;
            }
            if (pick < 0)
                for (int x = 0; x < n; ++x)
                    if (group[x] < 0 && (pick < 0 || load_of(x) < load_of(pick))) pick = x;
            group[pick] = g;
            load += load_of(pick);
            last = pick;
        }
    }
    return group;
}

moe_status place_correlated(const uint32_t *coact, int E, int G, int rpn, double eps, int32_t *expert_to_rank)
{
    if (E < 1 || G < 1 || rpn < 1 || G % rpn != 0 || E % G != 0 || !coact || !expert_to_rank) return MOE_ERR_ARG;
    const int nodes = G / rpn;
    double W = 0.0;
    for (int e = 0; e < E; ++e) W += (double)coact[(size_t)e * E + e];
    const double cap_node = eps >= 0.0 ? (1.0 + eps) * W / nodes : -1.0;
    const double cap_rank = eps >= 0.0 ? (1.0 + eps) * W / G : -1.0;
    std::vector<int> all(E);
    for (int e = 0; e < E; ++e) all[e] = e;
    const std::vector<int> node_of = greedy_split(coact, E, all, nodes, cap_node);
    for (int q = 0; q < nodes; ++q) {
        std::vector<int> pool;
        for (int e = 0; e < E; ++e)
            if (node_of[e] == q) pool.push_back(e);
        const std::vector<int> grp = greedy_split(coact, E, pool, rpn, cap_rank);
        for (size_t x = 0; x < pool.size(); ++x) expert_to_rank[pool[x]] = q * rpn + grp[x];
    }
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_place_uniform(int E, int G, int32_t *expert_to_rank)
{
    if (E < 1 || G < 1 || E % G != 0 || !expert_to_rank) return MOE_ERR_ARG;
    const int per = E / G;
    for (int e = 0; e < E; ++e) expert_to_rank[e] = e / per;
    return MOE_OK;
}

extern "C" moe_status moe_place_capacity(const double *load, int E, int G, int32_t *expert_to_rank, double *rank_load)
{
    if (E < 1 || G < 1 || !load || !expert_to_rank) return MOE_ERR_ARG;
    std::vector<int> order(E);
    for (int e = 0; e < E; ++e) order[e] = e;
    // stable insertion by descending load (lower id first among equals)
    for (int i = 1; i < E; ++i) {
        const int e = order[i];
        int j = i;
        while (j > 0 && load[order[j - 1]] < load[e]) {
            order[j] = order[j - 1];
            --j;
        }
        order[j] = e;
    }
    std::vector<double> dev(G, 0.0);
    for (int i = 0; i < E; ++i) {
        const int e = order[i];
        int best = 0;
        for (int g = 1; g < G; ++g)
            if (dev[g] < dev[best]) best = g;
        expert_to_rank[e] = best;
        dev[best] += load[e];
    }
    if (rank_load)
        for (int g = 0; g < G; ++g) rank_load[g] = dev[g];
    return MOE_OK;
}

extern "C" moe_status moe_place_correlated(const uint32_t *coact, int E, int G, int rpn, int32_t *expert_to_rank)
{
    return place_correlated(coact, E, G, rpn, -1.0, expert_to_rank);
}

extern "C" moe_status moe_place_correlated_capped(const uint32_t *coact, int E, int G, int rpn, double eps,
                                                  int32_t *expert_to_rank)
{
    return place_correlated(coact, E, G, rpn, eps, expert_to_rank);
}

// Replica layout ("Cobalt", "Problem Formulation": every expert on at least one
// rank, at most (1+rho)E/G experts per rank; "Two-Stage Expert Layout
// Planner": co-activated experts share nodes).  Greedy, from a placement with
// one replica per expert: every rank gets room for `extra` more experts; the
// candidate replicas (e, node q), e not already on q, are taken in decreasing
// order of score(e, q) = sum of C[e][e'] over the experts e' placed on q (ties:
// lower e, then lower q); a candidate whose node has no room left is skipped
// for good (room only shrinks), the others go on the rank of q with the most
// room (ties: lowest rank).  Candidates scoring 0 are never added.
extern "C" moe_status moe_place_replicas(const uint32_t *coact, int E, int G, int rpn, const int32_t *expert_to_rank,
                                         int extra, int32_t *replica_rank, int32_t *n_rep)
{
    if (E < 1 || G < 1 || rpn < 1 || G % rpn != 0 || extra < 0 || !coact || !expert_to_rank || !replica_rank || !n_rep)
        return MOE_ERR_ARG;
    const int nodes = G / rpn, max_rep = 1 + nodes;
    for (int e = 0; e < E; ++e)
        if (expert_to_rank[e] < 0 || expert_to_rank[e] >= G) return MOE_ERR_DATA;
    std::vector<uint64_t> score((size_t)E * nodes, 0);
    for (int e = 0; e < E; ++e)
        for (int f = 0; f < E; ++f)
            if (f != e) score[(size_t)e * nodes + expert_to_rank[f] / rpn] += coact[(size_t)e * E + f];
    struct Cand { uint64_t s; int e, q; };
    std::vector<Cand> cands;
    for (int e = 0; e < E; ++e) {
        for (int q = 0; q < max_rep; ++q) replica_rank[(size_t)e * max_rep + q] = -1;
        replica_rank[(size_t)e * max_rep] = expert_to_rank[e];
        n_rep[e] = 1;
        for (int q = 0; q < nodes; ++q)
            if (q != expert_to_rank[e] / rpn && score[(size_t)e * nodes + q] > 0)
                cands.push_back({score[(size_t)e * nodes + q], e, q});
    }
    std::stable_sort(cands.begin(), cands.end(), [](const Cand &a, const Cand &b) { return a.s > b.s; });
    std::vector<int> room(G, extra);
    for (const Cand &c : cands) {
        int br = -1;
        for (int r = c.q * rpn; r < (c.q + 1) * rpn; ++r)
            if (room[r] > 0 && (br < 0 || room[r] > room[br])) br = r;
        if (br < 0) continue;
        room[br] -= 1;
        replica_rank[(size_t)c.e * max_rep + n_rep[c.e]] = br;
        n_rep[c.e] += 1;
    }
    return MOE_OK;
}

// Tasks each rank serves under a one-replica placement: the sum of n_e = C_ee
// over the experts it holds ("Expert Placement Strategies", "Capacity-Aware
// Placement": a device's load is its experts' loads together).
extern "C" moe_status moe_rank_loads(const uint32_t *coact, int E, int G, const int32_t *expert_to_rank,
                                     long long *rank_load)
{
    if (!coact || !expert_to_rank || !rank_load || E < 1 || G < 1) return MOE_ERR_ARG;
    for (int e = 0; e < E; ++e)
        if (expert_to_rank[e] < 0 || expert_to_rank[e] >= G) return MOE_ERR_ARG;
    for (int r = 0; r < G; ++r) rank_load[r] = 0;
    for (int e = 0; e < E; ++e) rank_load[expert_to_rank[e]] += coact[(size_t)e * E + e];
    return MOE_OK;
}

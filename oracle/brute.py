"""ORACLE -- test infrastructure only.

Brute force in pure Python (sets, dicts, exact rationals) for inputs of a few
dozen tokens.  It restates the same definitions as oracle.c in a different
form -- token sets per expert instead of pair loops, a dict of rows per rank
instead of a sorted row array -- so that the two pin each other.
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction


def token_sets(ids_l, E):
    """A_e = set of tokens that selected expert e (the Ochiai operands on the
    Cobalt page, "Key Observation")."""
    A = [set() for _ in range(E)]
    for t, d in enumerate(ids_l):
        for e in d:
            A[int(e)].add(t)
    return A


def coact(ids, E):
    """C[l][i][j] = |A_i & A_j| at layer l."""
    out = []
    for ids_l in ids:
        A = token_sets(ids_l, E)
        out.append([[len(A[i] & A[j]) for j in range(E)] for i in range(E)])
    return out


def f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def ochiai(ids, E):
    """|A & B| / sqrt(|A| |B|), 0 for an empty operand; fp64 then fp32."""
    out = []
    for ids_l in ids:
        A = token_sets(ids_l, E)
        S = []
        for i in range(E):
            row = []
            for j in range(E):
                den = len(A[i]) * len(A[j])
                row.append(f32(len(A[i] & A[j]) / math.sqrt(den)) if den else 0.0)
            S.append(row)
        out.append(S)
    return out


def trans(ids, E):
    """M[l][i][j] = |A_i^l & A_j^{l+1}|."""
    out = []
    for l in range(len(ids) - 1):
        A = token_sets(ids[l], E)
        B = token_sets(ids[l + 1], E)
        out.append([[len(A[i] & B[j]) for j in range(E)] for i in range(E)])
    return out


def plan(ids_l, E, G, rpn, e2r, src_rank=None):
    """Rows per destination rank, each rank's list ordered by (source, token)."""
    T = len(ids_l)
    src = [int(src_rank[t]) if src_rank is not None else t // (T // G) for t in range(T)]
    per_dst = {r: [] for r in range(G)}
    dest = []
    for t, d in enumerate(ids_l):
        ranks = {int(e2r[int(e)]) for e in d}
        dest.append(ranks)
        for r in ranks:
            per_dst[r].append((src[t], t))
    rows = []
    for r in range(G):
        for s, t in sorted(per_dst[r]):
            rows.append((r, s, t))
    where = {(t, r): i for i, (r, s, t) in enumerate(rows)}
    row_of = [[where[(t, int(e2r[int(e)]))] for e in d] for t, d in enumerate(ids_l)]
    row_jmask = [sum(1 << j for j, e in enumerate(ids_l[t]) if int(e2r[int(e)]) == r) for (r, s, t) in rows]
    counts = [[0] * G for _ in range(G)]
    for r, s, t in rows:
        counts[s][r] += 1
    offsets = []
    run = 0
    for r in range(G):
        for s in range(G):
            offsets.append(run)
            run += counts[s][r]
    offsets.append(run)
    local = sum(1 for t, d in enumerate(ids_l) for e in d if int(e2r[int(e)]) == src[t])
    V = sum(len({int(e2r[int(e)]) // rpn for e in d} - {src[t] // rpn}) for t, d in enumerate(ids_l))
    remote = sum(1 for (r, s, t) in rows if r != s)
    return dict(row_token=[t for (r, s, t) in rows], row_jmask=row_jmask, row_of=row_of,
                counts=counts, offsets=offsets, dest=dest,
                R=len(rows), R_remote=remote, local=local, V=V)


def combine_exact(Y, idx, w):
    """Exact rational sum_j w[t][j] * Y[idx[t][j]][c] (Y, w given as Python floats)."""
    out = []
    for t in range(len(idx)):
        row = []
        for c in range(len(Y[0])):
            acc = Fraction(0)
            for j in range(len(idx[t])):
                acc += Fraction(float(w[t][j])) * Fraction(float(Y[idx[t][j]][c]))
            row.append(acc)
        out.append(row)
    return out


def shuffle_targets(ids_l, G, rank_score):
    tg = []
    for d in ids_l:
        scores = [sum(int(rank_score[int(e)][r]) for e in d) for r in range(G)]
        best = max(scores)
        tg.append(scores.index(best))
    return tg


def shuffle_balanced_da(ids_l, G, rank_score, capacity):
    """Capacity-balanced shuffle by token-proposing deferred acceptance
    (Gale-Shapley): each free token proposes to its next rank in the order
    score desc, rank asc; a rank keeps its `capacity` best proposers in the
    order score desc, token asc and rejects the rest.  Preferences that come
    from one common ordering of the (t, r) pairs have exactly one stable
    assignment, so this must agree with the greedy over that ordering."""
    T = len(ids_l)
    S = [[sum(int(rank_score[int(e)][r]) for e in d) for r in range(G)] for d in ids_l]
    pref = [sorted(range(G), key=lambda r: (-S[t][r], r)) for t in range(T)]
    nxt = [0] * T
    held = [[] for _ in range(G)]
    free = list(range(T))
    while free:
        t = free.pop()
        r = pref[t][nxt[t]]
        nxt[t] += 1
        held[r].append(t)
        if len(held[r]) > capacity:
            held[r].sort(key=lambda u: (-S[u][r], u))
            free.append(held[r].pop())
    tgt = [None] * T
    for r in range(G):
        for t in held[r]:
            tgt[t] = r
    return tgt


def blocking_pairs(ids_l, G, rank_score, capacity, tgt):
    """(t, r) pairs that would both rather be matched to each other: t ranks r
    above its own rank (score desc, rank asc) and r has room or holds a token
    it ranks below t (score desc, token asc)."""
    T = len(ids_l)
    S = [[sum(int(rank_score[int(e)][r]) for e in d) for r in range(G)] for d in ids_l]
    held = [[t for t in range(T) if tgt[t] == r] for r in range(G)]
    out = []
    for t in range(T):
        mine = (-S[t][tgt[t]], tgt[t])
        for r in range(G):
            if (-S[t][r], r) >= mine:
                continue
            worst = max(held[r], key=lambda u: (-S[u][r], u)) if held[r] else None
            if len(held[r]) < capacity or (-S[worst][r], worst) > (-S[t][r], t):
                out.append((t, r))
    return out


def place_correlated(C, G, rpn, eps=-1.0):
    """Restatement of the greedy grouping with Python lists and Fraction-free
    fp64 (same summation order as the specification: insertion order); with
    eps >= 0 a group only admits experts that keep its load within the cap,
    else the lightest expert left."""
    E = len(C)
    W = float(sum(int(C[e][e]) for e in range(E)))

    def s64(i, j):
        den = float(C[i][i]) * float(C[j][j])
        return C[i][j] / math.sqrt(den) if den > 0 else 0.0

    def groups(pool, m, cap):
        size = len(pool) // m
        left = sorted(pool)
        res = []
        for _ in range(m):
            seed = max(left, key=lambda e: (C[e][e], -e))
            grp = [seed]
            load = int(C[seed][seed])
            left.remove(seed)
            while len(grp) < size:
                def score(e):
                    s = 0.0
                    for g in grp:
                        s += s64(e, g)
                    return s
                fits = [e for e in left if cap < 0 or float(load + int(C[e][e])) <= cap]
                if fits:
                    best = max(fits, key=lambda e: (score(e), -e))
                else:
                    best = min(left, key=lambda e: (int(C[e][e]), e))
                grp.append(best)
                load += int(C[best][best])
                left.remove(best)
            res.append(grp)
        return res

    nodes = G // rpn
    cap_node = (1 + eps) * W / nodes if eps >= 0 else -1.0
    cap_rank = (1 + eps) * W / G if eps >= 0 else -1.0
    e2r = [0] * E
    for q, ng in enumerate(groups(list(range(E)), nodes, cap_node)):
        for u, rg in enumerate(groups(ng, rpn, cap_rank)):
            for e in rg:
                e2r[e] = q * rpn + u
    return e2r


def assign_replicas_capped(ids_l, G, rpn, replica_rank, n_rep, eps, src_rank=None):
    """Restatement of the load-capped assignment with Python sets: tokens in
    id order; ranks whose task count has reached floor((1 + eps) T k / G) are
    closed to the next token; a pick uses its expert's open replicas, or all
    of them when none is open; the remote node set is the smallest covering
    one (ties: smallest bit pattern), found by listing every node set; picks
    in j order prefer the source rank, then a rank the token already uses,
    then the lowest rank, among the usable ranks on the source node or, if
    none, on the chosen set.  Returns (picks, n_remote, loads) as lists."""
    T, k = len(ids_l), len(ids_l[0]) if len(ids_l) else 0
    nodes = G // rpn
    cap = math.floor((1.0 + eps) * float(T * k) / G) if math.isfinite(eps) else math.inf
    load = [0] * G
    picks, nrem = [], []
    for t in range(T):
        s = int(src_rank[t]) if src_rank is not None else t // (T // G)
        ns = s // rpn
        open_r = {r for r in range(G) if load[r] < cap}
        usable = []
        for e in ids_l[t]:
            reps = [int(r) for r in replica_rank[e][: n_rep[e]]]
            opn = [r for r in reps if r in open_r]
            usable.append(opn if opn else reps)
        best = None
        for bits in range(1 << nodes):
            S = {q for q in range(nodes) if (bits >> q) & 1}
            if ns in S:
                continue
            if all(any(r // rpn == ns or r // rpn in S for r in u) for u in usable):
                key = (len(S), bits)
                if best is None or key < best[0]:
                    best = (key, S)
        S = best[1]
        mine = []
        for u in usable:
            home = [r for r in u if r // rpn == ns]
            allowed = home if home else [r for r in u if r // rpn in S]
            if s in allowed:
                p = s
            elif any(r in mine for r in allowed):
                p = min(r for r in allowed if r in mine)
            else:
                p = min(allowed)
            mine.append(p)
        for p in mine:
            load[p] += 1
        picks.append(mine)
        nrem.append(len(S))
    return picks, nrem, load

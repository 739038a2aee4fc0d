"""Pins for the oracle of the load-capped task assignment ("Cobalt ...",
"Problem Formulation": a task runs on a rank holding its expert, the remote
nodes per token are to be few, and the tasks of a rank, sum_e w_r^e, stay
within (1 + eps) K T / G).

Reading pinned here: tokens in id order; a rank whose task count has
reached floor((1 + eps) T k / G) before token t is closed to t; t's picks use
their experts' open replicas (all replicas when none is open) under the
fewest-remote-nodes rule.  Checked against a hand-worked case, the eps = inf
limit (the uncapped assignment), a pure-Python restatement, and brute force
over every replica choice of each token given the ranks open to it."""
import itertools
import math

import numpy as np
import pytest

from oracle import brute


def _layout(orc, seed, T=64, E=16, k=3, G=8, rpn=2, extra=2, hot_frac=0.6):
    rng = np.random.default_rng(seed)
    hot = rng.permutation(E)[: k + 2]
    ids = np.where((rng.random(T) < hot_frac)[:, None],
                   hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                   np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    rr, nr = orc.place_replicas(C, G, rpn, e2r, extra)
    return rng, ids, e2r, rr, nr


def test_cap_value(orc):
    # floor((1 + eps) T k / G) in fp64; eps = inf: no cap
    assert orc.load_cap(100, 2, 8, 0.0) == 25
    assert orc.load_cap(100, 2, 8, 0.1) == 27          # 27.5
    assert orc.load_cap(96, 3, 8, 0.05) == 37          # 37.8
    assert orc.load_cap(5, 1, 4, 0.0) == 1             # 1.25
    assert orc.load_cap(64, 8, 64, 0.0) == 8
    assert orc.load_cap(64, 8, 64, math.inf) == 2 ** 63 - 1


def test_hand_worked(orc):
    # 2 nodes of one rank.  Expert 0 on ranks 0 and 1, expert 1 only on rank
    # 0.  Six one-pick tokens from rank 0: cap = floor(6 / 2) = 3.
    rr = np.array([[0, 1, -1], [0, -1, -1]], np.int32)
    nr = np.array([2, 1], np.int32)
    ids = np.array([[0], [0], [0], [0], [1], [1]], np.int32)
    src = np.zeros(6, np.int32)
    pr, nrem, load = orc.assign_replicas_capped(ids, 2, 2, 1, rr, nr, 0.0, src_rank=src)
    # tokens 0-2 stay on the source rank until it holds 3 tasks; token 3 goes
    # to rank 1 (one remote node); tokens 4 and 5 have no open replica of
    # expert 1 and keep rank 0 (the cap gives way)
    assert pr[:, 0].tolist() == [0, 0, 0, 1, 0, 0]
    assert nrem.tolist() == [0, 0, 0, 1, 0, 0]
    assert load.tolist() == [5, 1]
    # uncapped: everything on the source rank
    pr0, nrem0 = orc.assign_replicas(ids, 2, 2, 1, rr, nr, src_rank=src)
    assert pr0[:, 0].tolist() == [0] * 6 and nrem0.tolist() == [0] * 6


def test_hand_worked_two_picks(orc):
    # experts 0 and 1 each on ranks 0 and 1 (2 nodes of one rank); two
    # two-pick tokens from rank 0: cap = floor(4 / 2) = 2.  Token 0 puts both
    # tasks on rank 0 (no remote node); rank 0 is then closed, so token 1
    # sends both to rank 1 (one remote node, one row).
    rr = np.array([[0, 1, -1], [1, 0, -1]], np.int32)
    nr = np.array([2, 2], np.int32)
    ids = np.array([[0, 1], [1, 0]], np.int32)
    pr, nrem, load = orc.assign_replicas_capped(ids, 2, 2, 1, rr, nr, 0.0, src_rank=np.zeros(2, np.int32))
    assert pr.tolist() == [[0, 0], [1, 1]] and nrem.tolist() == [0, 1] and load.tolist() == [2, 2]
    # a token may take a rank past the cap by k - 1: 4 ranks, cap = floor(4/4) = 1
    pr, _, load = orc.assign_replicas_capped(ids, 2, 4, 1, np.array([[0, 1, -1, -1, -1], [1, 0, -1, -1, -1]], np.int32),
                                             nr, 0.0, src_rank=np.zeros(2, np.int32))
    assert pr.tolist() == [[0, 0], [1, 1]] and load.tolist() == [2, 2, 0, 0]


@pytest.mark.parametrize("seed,G,rpn", [(0, 8, 2), (1, 8, 4), (2, 4, 1)])
def test_no_cap_is_the_uncapped_assignment(orc, seed, G, rpn):
    rng, ids, e2r, rr, nr = _layout(orc, seed, G=G, rpn=rpn)
    pr0, nrem0 = orc.assign_replicas(ids, 16, G, rpn, rr, nr)
    for eps in (math.inf, 1e6):
        pr, nrem, load = orc.assign_replicas_capped(ids, 16, G, rpn, rr, nr, eps)
        assert np.array_equal(pr, pr0) and np.array_equal(nrem, nrem0)
        assert load.tolist() == np.bincount(pr.ravel(), minlength=G).tolist()


def test_one_replica_each_has_no_choice(orc):
    rng, ids, e2r, rr, nr = _layout(orc, 3, extra=0)
    assert (nr == 1).all()
    for eps in (0.0, 0.1):
        pr, nrem, load = orc.assign_replicas_capped(ids, 16, 8, 2, rr, nr, eps)
        assert (pr == e2r[ids]).all()


CASES = [(4, 8, 2, 0.0, False), (5, 8, 2, 0.05, True), (6, 8, 4, 0.2, False), (7, 4, 1, 0.1, True),
         (8, 8, 1, 0.0, True), (9, 8, 2, 1.0, False), (10, 16, 2, 0.03, True)]


@pytest.mark.parametrize("seed,G,rpn,eps,with_src", CASES)
def test_matches_restatement(orc, seed, G, rpn, eps, with_src):
    rng, ids, e2r, rr, nr = _layout(orc, seed, T=96, G=G, rpn=rpn, extra=2)
    T = ids.shape[0]
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    pr, nrem, load = orc.assign_replicas_capped(ids, 16, G, rpn, rr, nr, eps, src_rank=src)
    bp, bn, bl = brute.assign_replicas_capped(ids.tolist(), G, rpn, rr.tolist(), nr.tolist(), eps,
                                              None if src is None else src.tolist())
    assert pr.tolist() == bp and nrem.tolist() == bn and load.tolist() == bl


@pytest.mark.parametrize("seed,G,rpn,eps,with_src", CASES)
def test_each_token_minimal_over_its_open_ranks(orc, seed, G, rpn, eps, with_src):
    """Replaying the loads token by token gives each token's open ranks; over
    every choice of one usable replica per pick, none reaches fewer remote
    nodes than the oracle's; picks host their experts; a rank passes the cap
    by more than k - 1 only through picks with no open replica."""
    rng, ids, e2r, rr, nr = _layout(orc, seed, T=96, G=G, rpn=rpn, extra=2)
    T, k = ids.shape
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    pr, nrem, load = orc.assign_replicas_capped(ids, 16, G, rpn, rr, nr, eps, src_rank=src)
    cap = orc.load_cap(T, k, G, eps)
    s_of = src if with_src else np.arange(T) // (T // G)
    run = np.zeros(G, np.int64)
    forced = np.zeros(G, np.int64)
    for t in range(T):
        ns = s_of[t] // rpn
        usable = []
        for j, e in enumerate(ids[t]):
            reps = rr[e, : nr[e]].tolist()
            opn = [r for r in reps if run[r] < cap]
            usable.append(opn if opn else reps)
            assert pr[t, j] in usable[-1]
            if not opn:
                forced[pr[t, j]] += 1
        best = min(len({r // rpn for r in combo} - {ns}) for combo in itertools.product(*usable))
        assert nrem[t] == best == len({int(r) // rpn for r in pr[t]} - {ns})
        for r in pr[t]:
            run[r] += 1
    assert run.tolist() == load.tolist() and load.sum() == T * k
    assert (load <= cap + k - 1 + forced).all()
    p = orc.plan(ids, 16, G, rpn, None, src_rank=src, pick_rank=pr)
    assert p["V"] == int(nrem.sum())


def test_tighter_cap_lowers_the_busiest_rank(orc):
    rng, ids, e2r, rr, nr = _layout(orc, 11, T=256, E=16, k=3, G=8, rpn=2, extra=2, hot_frac=0.9)
    _, _, free = orc.assign_replicas_capped(ids, 16, 8, 2, rr, nr, math.inf)
    _, _, tight = orc.assign_replicas_capped(ids, 16, 8, 2, rr, nr, 0.0)
    assert tight.max() < free.max()


def test_rank_loads(orc):
    C = np.diag(np.array([5, 0, 7, 2], np.uint32))
    assert orc.rank_loads(C, np.array([1, 0, 1, 2], np.int32), 3).tolist() == [0, 12, 2]
    rng, ids, e2r, rr, nr = _layout(orc, 12, extra=0)
    C = orc.coact(ids[None], 16, want=("coact",))["coact"][0]
    assert orc.rank_loads(C, e2r, 8).tolist() == np.bincount(e2r[ids].ravel(), minlength=8).tolist()


def test_rejects_bad_arguments(orc):
    rng, ids, e2r, rr, nr = _layout(orc, 13)
    for eps in (-0.1, float("nan")):
        with pytest.raises(orc.OracleError):
            orc.assign_replicas_capped(ids, 16, 8, 2, rr, nr, eps)

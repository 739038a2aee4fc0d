"""Pins for the oracle of expert replicas and communication-aware task
assignment ("Cobalt ...", "Problem Formulation": every expert has at least
one replica, |P_r| <= (1+rho)E/G, a task runs on a rank holding its expert,
and V counts the remote nodes each token reaches; "communication-aware task
assignment routes tokens to the fewest remote nodes possible").

The assignment is checked against brute force over every choice of one
replica per pick: its remote-node count must be the minimum."""
import itertools

import numpy as np
import pytest


def _routing(rng, T, E, k, hot_frac=0.6):
    hot = rng.permutation(E)[: k + 2]
    return np.where((rng.random(T) < hot_frac)[:, None],
                    hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                    np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)


def _setup(orc, seed, T=96, E=16, k=3, G=8, rpn=2, extra=1):
    rng = np.random.default_rng(seed)
    ids = _routing(rng, T, E, k)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    rr, nr = orc.place_replicas(C, G, rpn, e2r, extra)
    return rng, ids, C, e2r, rr, nr


@pytest.mark.parametrize("seed,G,rpn,extra", [(0, 8, 2, 1), (1, 8, 4, 2), (2, 4, 1, 1), (3, 16, 2, 1)])
def test_replica_layout_invariants(orc, seed, G, rpn, extra):
    rng, ids, C, e2r, rr, nr = _setup(orc, seed, E=16, G=G, rpn=rpn, extra=extra)
    E = 16
    assert (rr[:, 0] == e2r).all() and (nr >= 1).all()
    per_rank = np.zeros(G, int)
    for e in range(E):
        ranks = rr[e, : nr[e]]
        assert (rr[e, nr[e]:] == -1).all()
        assert len(set((ranks // rpn).tolist())) == nr[e]        # at most one replica per node
        np.add.at(per_rank, ranks, 1)
    assert (per_rank <= E // G + extra).all()


def test_no_room_means_no_replicas(orc):
    rng, ids, C, e2r, rr, nr = _setup(orc, 4, extra=0)
    assert (nr == 1).all()
    pr, nrem = orc.assign_replicas(ids, 16, 8, 2, rr, nr)
    assert (pr == e2r[ids]).all()
    a = orc.plan(ids, 16, 8, 2, e2r)
    b = orc.plan(ids, 16, 8, 2, None, pick_rank=pr)
    for key in ("row_token", "row_jmask", "row_of", "counts", "offsets", "summary"):
        assert np.array_equal(a[key], b[key])
    assert a["V"] == int(nrem.sum())


@pytest.mark.parametrize("seed,G,rpn,with_src", [(5, 8, 2, False), (6, 8, 4, True), (7, 4, 1, True), (8, 8, 1, False)])
def test_assignment_is_minimal_by_brute_force(orc, seed, G, rpn, with_src):
    rng, ids, C, e2r, rr, nr = _setup(orc, seed, T=64, E=16, k=3, G=G, rpn=rpn, extra=2)
    T, k = ids.shape
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    pr, nrem = orc.assign_replicas(ids, 16, G, rpn, rr, nr, src_rank=src)
    s_of = src if with_src else np.arange(T) // (T // G)
    for t in range(T):
        ns = s_of[t] // rpn
        choices = [rr[e, : nr[e]].tolist() for e in ids[t]]
        best = min(len({r // rpn for r in combo} - {ns}) for combo in itertools.product(*choices))
        assert nrem[t] == best
        for j, e in enumerate(ids[t]):
            assert pr[t, j] in rr[e, : nr[e]]
        assert len({int(r) // rpn for r in pr[t]} - {ns}) == best
    p = orc.plan(ids, 16, G, rpn, None, src_rank=src, pick_rank=pr)
    assert p["V"] == int(nrem.sum())


def test_replicas_never_add_remote_nodes(orc):
    rng, ids, C, e2r, rr, nr = _setup(orc, 9, T=128, E=32, k=4, G=8, rpn=2, extra=2)
    rr0, nr0 = orc.place_replicas(C, 8, 2, e2r, 0)
    _, with_rep = orc.assign_replicas(ids, 32, 8, 2, rr, nr)
    _, without = orc.assign_replicas(ids, 32, 8, 2, rr0, nr0)
    assert (with_rep <= without).all() and with_rep.sum() < without.sum()


def test_pick_rule_prefers_source_then_source_node(orc):
    # expert 0 on ranks {0 (node 0), 3 (node 1)}; expert 1 only on rank 2 (node 1)
    rr = np.array([[0, 3, -1], [2, -1, -1], [1, -1, -1], [3, -1, -1]], np.int32)
    nr = np.array([2, 1, 1, 1], np.int32)
    ids = np.array([[0, 1], [0, 2], [1, 3]], np.int32)
    src = np.array([0, 2, 0], np.int32)
    pr, nrem = orc.assign_replicas(ids, 4, 4, 2, rr, nr, src_rank=src)
    # token 0 from rank 0: expert 0 on its own rank, expert 1 needs node 1
    assert pr[0].tolist() == [0, 2] and nrem[0] == 1
    # token 1 from rank 2 (node 1): expert 0's replica on node 1 (rank 3); expert 2 only on rank 1 (node 0)
    assert pr[1].tolist() == [3, 1] and nrem[1] == 1
    # token 2 from rank 0: experts 1 and 3 both live on node 1
    assert pr[2].tolist() == [2, 3] and nrem[2] == 1


def test_assignment_rejects_many_nodes(orc):
    rng, ids, C, e2r, rr, nr = _setup(orc, 10, E=16, G=16, rpn=1, extra=0)
    with pytest.raises(orc.OracleError):
        orc.assign_replicas(ids, 16, 16, 1, rr, nr)


def test_replica_room_ties_go_to_lowest_rank(orc):
    # 2 nodes of 2 ranks, 4 experts one per rank; expert 0 (rank 0) is
    # co-activated with experts 2 and 3 (node 1) -> a replica on node 1, whose
    # ranks 2 and 3 have equal room: it goes to rank 2
    C = np.zeros((4, 4), np.uint32)
    C[0, 2] = C[2, 0] = 5
    C[0, 3] = C[3, 0] = 4
    rr, nr = orc.place_replicas(C, 4, 2, np.array([0, 1, 2, 3], np.int32), 1)
    assert nr.tolist() == [2, 1, 2, 2]
    assert rr[0].tolist() == [0, 2, -1]
    # expert 2 and 3 (node 1) are co-activated with expert 0 (node 0): replicas
    # on node 0, in score order (expert 2 first), each onto the rank with the
    # most room left: rank 0 and 1 start equal -> rank 0, then rank 1
    assert rr[2].tolist() == [2, 0, -1] and rr[3].tolist() == [3, 1, -1]


def test_replica_minimal_set_ties_go_to_smallest_pattern(orc):
    # 3 nodes of 1 rank; expert 0 on rank 0, expert 1 on ranks 1 and 2: from
    # rank 0, node 1 and node 2 both cover expert 1 with one remote node ->
    # the smaller bit pattern, node 1
    rr = np.array([[0, -1, -1, -1], [1, 2, -1, -1]], np.int32)
    nr = np.array([1, 2], np.int32)
    ids = np.array([[0, 1]] * 3, np.int32)
    pr, nrem = orc.assign_replicas(ids, 2, 3, 1, rr, nr, src_rank=np.array([0, 0, 0], np.int32))
    assert pr.tolist() == [[0, 1]] * 3 and nrem.tolist() == [1, 1, 1]
    # listed in the other order the choice is the same
    rr2 = np.array([[0, -1, -1, -1], [2, 1, -1, -1]], np.int32)
    pr2, _ = orc.assign_replicas(ids, 2, 3, 1, rr2, nr, src_rank=np.array([0, 0, 0], np.int32))
    assert pr2.tolist() == [[0, 1]] * 3


def test_replica_pick_reuses_a_rank_already_serving_the_token(orc):
    # 2 nodes of 2 ranks; expert 0 only on rank 3, expert 1 on ranks 2 and 3
    # (both node 1).  From rank 0 both picks need node 1.
    rr = np.array([[3, -1, -1], [2, 3, -1]], np.int32)
    nr = np.array([1, 2], np.int32)
    ids = np.array([[0, 1], [1, 0]], np.int32)
    pr, nrem = orc.assign_replicas(ids, 2, 4, 2, rr, nr, src_rank=np.array([0, 0], np.int32))
    # [0, 1]: expert 0 -> rank 3; expert 1 could use rank 2 or 3, rank 3 already
    # carries the token's row -> 3 (one row).  [1, 0]: expert 1 first -> the
    # lowest, rank 2; expert 0 only on rank 3.
    assert pr.tolist() == [[3, 3], [2, 3]] and nrem.tolist() == [1, 1]

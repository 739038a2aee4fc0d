"""Pins for the oracle of the capacity-balanced token shuffle.

"Expert Coupling in MoE Pretraining ...", abstract: token shuffling moves each
token to the GPU predicted to hold its next-layer experts during the
reduce-scatter after attention; a reduce-scatter gives every rank an equal
shard.  The oracle takes the (t, r) pairs greedily in the order score desc,
t asc, r asc under a per-rank capacity.  Pinned by: the unconstrained argmax
(capacity >= T), token-proposing deferred acceptance (a different algorithm
that reaches the same unique stable assignment), the absence of blocking
pairs, exact shard sizes, and a hand-worked example."""
import numpy as np
import pytest

from oracle import brute


def _case(rng, T, E, k, G, hi):
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    rs = rng.integers(0, hi, (E, G)).astype(np.uint32)
    return ids, rs


@pytest.mark.parametrize("seed", range(6))
def test_unbounded_capacity_is_the_argmax(orc, seed):
    rng = np.random.default_rng(seed)
    ids, rs = _case(rng, 300, 16, 3, 8, 50)
    assert (orc.shuffle_balanced(ids, 16, 8, rs, 300) == orc.shuffle_targets(ids, 16, 8, rs)).all()


@pytest.mark.parametrize("seed,T,E,k,G,hi,cap", [(0, 48, 8, 2, 4, 4, 12), (1, 50, 12, 3, 6, 3, 9),
                                                 (2, 64, 16, 4, 8, 100, 8), (3, 31, 8, 1, 4, 2, 8),
                                                 (4, 40, 10, 2, 5, 1, 8), (5, 60, 16, 2, 4, 6, 20),
                                                 (6, 1, 4, 2, 2, 3, 1), (7, 24, 6, 6, 3, 5, 8)])
def test_greedy_equals_deferred_acceptance(orc, seed, T, E, k, G, hi, cap):
    rng = np.random.default_rng(seed)
    ids, rs = _case(rng, T, E, k, G, hi)
    got = orc.shuffle_balanced(ids, E, G, rs, cap)
    assert got.tolist() == brute.shuffle_balanced_da(ids, G, rs, cap)
    assert brute.blocking_pairs(ids, G, rs, cap, got.tolist()) == []
    counts = np.bincount(got, minlength=G)
    assert (counts <= cap).all() and counts.sum() == T
    if T == G * cap:
        assert (counts == cap).all()


def test_planted_balanced_preferences_keep_the_argmax(orc):
    # every token's best rank is its planted rank and the planted ranks are
    # already balanced: the capacity binds nowhere
    G, E, k, C = 4, 8, 2, 10
    rs = np.zeros((E, G), np.uint32)
    for e in range(E):
        rs[e, e // 2] = 7
    rng = np.random.default_rng(3)
    ids = np.stack([rng.permutation(np.arange(2 * (t % G), 2 * (t % G) + 2)) for t in range(G * C)]).astype(np.int32)
    got = orc.shuffle_balanced(ids, E, G, rs, C)
    assert (got == np.arange(G * C) % G).all()


def test_hand_worked_example(orc):
    # 2 ranks, capacity 2, one pick per token; expert e's scores for ranks 0/1:
    #   e0: 5/1  e1: 5/1  e2: 5/4  e3: 3/3
    # pairs in order: (t0,r0,5) (t1,r0,5) (t2,r0,5) (t2,r1,4) (t3,r0,3) (t3,r1,3) ...
    # t0 -> 0, t1 -> 0 (rank 0 full), t2 -> 1, t3 -> 1 (rank 0 full; tie at 3
    # would otherwise pick rank 0)
    rs = np.array([[5, 1], [5, 1], [5, 4], [3, 3]], np.uint32)
    ids = np.array([[0], [1], [2], [3]], np.int32)
    assert orc.shuffle_balanced(ids, 4, 2, rs, 2).tolist() == [0, 0, 1, 1]
    # listing the tokens the other way round: equal scores go to the lower token id
    ids2 = np.array([[3], [2], [1], [0]], np.int32)
    # pairs: (t1,r0,5) (t2,r0,5) (t3,r0,5) (t1,r1,4) (t0,r0,3) (t0,r1,3)
    assert orc.shuffle_balanced(ids2, 4, 2, rs, 2).tolist() == [1, 0, 0, 1]


def test_capacity_below_shard_is_an_error(orc):
    ids = np.zeros((9, 1), np.int32)
    with pytest.raises(orc.OracleError):
        orc.shuffle_balanced(ids, 1, 4, np.ones((1, 4), np.uint32), 2)


def test_empty_batch(orc):
    assert orc.shuffle_balanced(np.zeros((0, 2), np.int32), 4, 2, np.ones((4, 2), np.uint32), 0).size == 0

"""Pins for the load-capped correlated placement ("Cobalt", "Problem
Formulation": every rank's load within a tolerance of the average; the
grouping itself is a greedy of our own reading).  eps < 0 and a huge eps reduce to the
plain correlated greedy; a hand-worked case; the pure-Python restatement; a
group overshoots its cap by less than one expert's load."""
import numpy as np
import pytest

from oracle import brute


def _coact(rng, E, T=400, k=3, skew=1.0):
    w = rng.random(E) ** skew
    ids = np.stack([rng.choice(E, size=k, replace=False, p=w / w.sum()) for _ in range(T)]).astype(np.int32)
    return ids


def test_no_cap_is_the_plain_greedy(orc):
    rng = np.random.default_rng(0)
    for E, G, rpn in [(16, 4, 2), (32, 8, 8), (24, 6, 3)]:
        ids = _coact(rng, E)
        C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
        plain = orc.place_correlated(C, G, rpn)
        assert (orc.place_correlated_capped(C, G, rpn, -1.0) == plain).all()
        assert (orc.place_correlated_capped(C, G, rpn, 1e9) == plain).all()


def test_hand_worked_case(orc):
    # 4 experts, 2 ranks on one node; loads 10, 9, 1, 1; experts 0 and 1 always together
    C = np.array([[10, 9, 1, 0], [9, 9, 0, 0], [1, 0, 1, 0], [0, 0, 0, 1]], np.uint32)
    # uncapped: {0, 1} (load 19) and {2, 3}
    assert orc.place_correlated(C, 2, 2).tolist() == [0, 0, 1, 1]
    # eps = 0.2: cap 1.2 * 21 / 2 = 12.6, so 1 cannot join 0; of 2 and 3, 2 has the
    # larger Ochiai with 0 (1 / sqrt(10)); group 1 = {1, 3}
    assert orc.place_correlated_capped(C, 2, 2, 0.2).tolist() == [0, 1, 0, 1]


@pytest.mark.parametrize("seed,E,G,rpn,eps", [(1, 16, 4, 2, 0.1), (2, 16, 8, 4, 0.0), (3, 24, 6, 3, 0.3),
                                              (4, 32, 8, 2, 0.05), (5, 12, 4, 4, 0.5)])
def test_equals_restatement(orc, seed, E, G, rpn, eps):
    rng = np.random.default_rng(seed)
    C = orc.coact(_coact(rng, E, skew=3.0)[None], E, want=("coact",))["coact"][0]
    got = orc.place_correlated_capped(C, G, rpn, eps)
    assert got.tolist() == brute.place_correlated(C.tolist(), G, rpn, eps)
    assert np.bincount(got, minlength=G).tolist() == [E // G] * G


def test_cap_overshoot_is_at_most_one_expert(orc):
    # the greedy fills groups in turn; a group exceeds the cap only through an
    # expert it had to take when none fitted, so by less than the heaviest load
    rng = np.random.default_rng(7)
    E, G, rpn, eps = 32, 4, 4, 0.25
    C = orc.coact(_coact(rng, E, T=2000)[None], E, want=("coact",))["coact"][0]
    n = np.diag(C).astype(np.float64)
    e2r = orc.place_correlated_capped(C, G, rpn, eps)
    loads = np.bincount(e2r, weights=n, minlength=G)
    assert loads.max() <= (1 + eps) * n.sum() / G + n.max()
    plain = np.bincount(orc.place_correlated(C, G, rpn), weights=n, minlength=G)
    assert loads.max() < plain.max()

"""Property-based checks of the oracle against the pure-Python brute force.

Hypothesis draws small shapes (T tokens, E experts, k picks, G ranks, rpn,
explicit or contiguous source ranks, W devices) and routing with heavy
overlap; for each draw the C oracle's counts, Ochiai, transitions, plan and
shuffle targets equal the brute force's, and its route tables move every
device's rows onto the one-device rows exactly once.  Derandomised, so the
draws are the same on every run."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import brute

SETTINGS = settings(max_examples=200, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])


@st.composite
def shapes(draw):
    G = draw(st.sampled_from([1, 2, 3, 4, 6, 8]))
    rpn = draw(st.sampled_from([r for r in range(1, G + 1) if G % r == 0]))
    E = G * draw(st.integers(1, 4))
    k = draw(st.integers(1, min(E, 6)))
    W = draw(st.sampled_from([w for w in range(1, G + 1) if G % w == 0]))
    T = G * W * draw(st.integers(1, 4)) if draw(st.booleans()) else draw(st.integers(1, 40))
    with_src = draw(st.booleans()) or T % G != 0
    seed = draw(st.integers(0, 2 ** 31))
    return T, E, k, G, rpn, W, with_src, seed


def _routing(rng, L, T, E, k):
    out = np.empty((L, T, k), np.int32)
    for l in range(L):
        for t in range(T):
            pool = np.arange(min(E, k + 1)) if rng.random() < 0.6 else np.arange(E)
            out[l, t] = rng.permutation(pool)[:k]
    return out


@SETTINGS
@given(shapes())
def test_stats_plan_shuffle_match_brute(orc, shape):
    T, E, k, G, rpn, W, with_src, seed = shape
    rng = np.random.default_rng(seed)
    ids = _routing(rng, 2, T, E, k)
    s = orc.coact(ids, E)
    assert s["coact"].tolist() == brute.coact(ids.tolist(), E)
    assert s["trans"].tolist() == brute.trans(ids.tolist(), E)
    assert s["ochiai"].tolist() == brute.ochiai(ids.tolist(), E)
    e2r = rng.permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    p = orc.plan(ids[0], E, G, rpn, e2r, src_rank=src)
    b = brute.plan(ids[0].tolist(), E, G, rpn, e2r.tolist(), None if src is None else src.tolist())
    assert p["row_token"].tolist() == b["row_token"] and p["row_of"].tolist() == b["row_of"]
    assert p["row_jmask"].tolist() == b["row_jmask"] and p["offsets"].tolist() == b["offsets"]
    assert (p["R"], p["R_remote"], p["local"], p["V"]) == (b["R"], b["R_remote"], b["local"], b["V"])
    rs = orc.rank_score(s["trans"][0], e2r, G)
    assert orc.shuffle_targets(ids[0], E, G, rs).tolist() == brute.shuffle_targets(ids[0].tolist(), G, rs.tolist())


@SETTINGS
@given(shapes())
def test_routes_cover_the_one_device_rows(orc, shape):
    T, E, k, G, rpn, W, _, seed = shape
    Gl = G // W
    T = G * W * max(1, T // (G * W))                     # every device's tokens split over its ranks
    rng = np.random.default_rng(seed)
    ids = _routing(rng, 1, T, E, k)[0]
    e2r = rng.permutation(np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
    o = orc.plan(ids, E, G, rpn, e2r)
    off = o["offsets"].astype(np.int64)
    Tl, P = T // W, G * Gl
    plans = []
    for h in range(W):
        src = (h * Gl + np.arange(Tl) // (Tl // Gl)).astype(np.int32)
        plans.append(orc.plan(ids[h * Tl:(h + 1) * Tl], E, G, rpn, e2r, src_rank=src))
    counts_all = np.concatenate([plans[h]["counts"][h * Gl:(h + 1) * Gl] for h in range(W)])
    seen = np.zeros(o["R"], np.int64)
    for h, lo in enumerate(plans):
        route = orc.ep_routes(counts_all, lo["offsets"], G, W, h)
        start = route[1:P + 2]
        for x in range(lo["R"]):
            i = int(np.searchsorted(start, x, side="right")) - 1
            r = i // Gl
            g = off[(r // Gl) * Gl * G] + x + route[P + 2 + i]
            assert o["row_token"][g] == h * Tl + lo["row_token"][x]
            seen[g] += 1
        assert route[0] == sum(int(o["counts"][s_, r_]) for s_ in range(G) for r_ in range(h * Gl, (h + 1) * Gl))
    assert (seen == 1).all()


@SETTINGS
@given(shapes(), st.integers(0, 3))
def test_balanced_shuffle_matches_deferred_acceptance(orc, shape, slack):
    """The greedy over one pair order (the oracle) and token-proposing
    deferred acceptance (the brute force) reach the same, stable assignment
    for any capacity that can hold all tokens."""
    T, E, k, G, rpn, W, _, seed = shape
    rng = np.random.default_rng(seed)
    ids = _routing(rng, 1, T, E, k)[0]
    rs = rng.integers(0, 4, (E, G)).astype(np.uint32)          # small scores: many ties
    capacity = -(-T // G) + slack
    got = orc.shuffle_balanced(ids, E, G, rs, capacity).tolist()
    assert got == brute.shuffle_balanced_da(ids.tolist(), G, rs.tolist(), capacity)
    assert brute.blocking_pairs(ids.tolist(), G, rs.tolist(), capacity, got) == []
    assert max(np.bincount(np.array(got), minlength=G)) <= capacity


@SETTINGS
@given(st.sampled_from([(4, 2, 1), (8, 4, 2), (12, 6, 3), (16, 8, 4), (12, 4, 4), (16, 4, 1)]),
       st.integers(0, 2 ** 31), st.sampled_from([-1.0, 0.0, 0.1, 0.5]))
def test_correlated_placement_matches_brute(orc, egr, seed, eps):
    """The greedy grouping (with and without a load tolerance) equals its
    pure-Python restatement on random symmetric co-activation counts."""
    E, G, rpn = egr
    rng = np.random.default_rng(seed)
    ids = _routing(rng, 1, 200, E, min(4, E))
    C = orc.coact(ids, E)["coact"][0]
    want = brute.place_correlated(C.tolist(), G, rpn, eps)
    got = orc.place_correlated_capped(C, G, rpn, eps) if eps >= 0 else orc.place_correlated(C, G, rpn)
    assert got.tolist() == list(want)

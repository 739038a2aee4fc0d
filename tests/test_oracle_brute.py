"""The C oracle against the pure-Python brute force (token sets, dicts of rows,
exact rationals) on tiny random inputs, including ragged sizes, k = 1, k = E,
G = 1, G = E and one rank per node."""
import numpy as np
import pytest

from oracle import brute

CASES = [
    # T, E, k, G, rpn, L
    (8, 4, 1, 2, 1, 2),
    (24, 8, 2, 4, 2, 3),
    (30, 6, 6, 3, 3, 2),
    (40, 16, 3, 8, 4, 2),
    (64, 32, 8, 8, 8, 2),
    (36, 12, 4, 12, 3, 2),
    (20, 10, 3, 1, 1, 2),
]


def _ids(rng, L, T, E, k, clustered):
    if not clustered:
        return np.stack([np.stack([rng.permutation(E)[:k] for _ in range(T)]) for _ in range(L)]).astype(np.int32)
    # heavy overlap: most tokens draw from the first k+1 experts
    out = np.empty((L, T, k), np.int32)
    for l in range(L):
        for t in range(T):
            pool = np.arange(min(E, k + 1)) if rng.random() < 0.7 else np.arange(E)
            out[l, t] = rng.permutation(pool)[:k]
    return out


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("clustered", [False, True])
def test_stats_vs_brute(orc, case, clustered):
    T, E, k, G, rpn, L = case
    rng = np.random.default_rng(hash((case, clustered)) % 2 ** 32)
    ids = _ids(rng, L, T, E, k, clustered)
    out = orc.coact(ids, E)
    assert out["coact"].tolist() == brute.coact(ids.tolist(), E)
    assert out["trans"].tolist() == brute.trans(ids.tolist(), E)
    assert out["ochiai"].tolist() == brute.ochiai(ids.tolist(), E)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("with_src", [False, True])
def test_plan_vs_brute(orc, case, with_src):
    T, E, k, G, rpn, L = case
    rng = np.random.default_rng(hash((case, with_src, 1)) % 2 ** 32)
    ids = _ids(rng, 1, T, E, k, clustered=True)[0]
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    src = rng.integers(0, G, T).astype(np.int32) if with_src else None
    if not with_src and T % G:
        pytest.skip("contiguous shards need G | T")
    p = orc.plan(ids, E, G, rpn, e2r, src_rank=src)
    b = brute.plan(ids.tolist(), E, G, rpn, e2r.tolist(), None if src is None else src.tolist())
    assert p["row_token"].tolist() == b["row_token"]
    assert p["row_jmask"].tolist() == b["row_jmask"]
    assert p["row_of"].tolist() == b["row_of"]
    assert p["counts"].tolist() == b["counts"]
    assert p["offsets"].tolist() == b["offsets"]
    assert (p["R"], p["R_remote"], p["local"], p["V"]) == (b["R"], b["R_remote"], b["local"], b["V"])
    assert [sorted(int(r) for r in range(G) if int(m) >> r & 1) for m in p["dest_mask"]] == \
        [sorted(s) for s in b["dest"]]


@pytest.mark.parametrize("case", CASES)
def test_shuffle_and_placement_vs_brute(orc, case):
    T, E, k, G, rpn, L = case
    rng = np.random.default_rng(hash((case, 2)) % 2 ** 32)
    ids = _ids(rng, 2, T, E, k, clustered=True)
    stats = orc.coact(ids, E)
    e2r = orc.place_correlated(stats["coact"][0], G, rpn)
    assert e2r.tolist() == brute.place_correlated(stats["coact"][0].tolist(), G, rpn)
    rs = orc.rank_score(stats["trans"][0], e2r, G)
    assert orc.shuffle_targets(ids[0], E, G, rs).tolist() == brute.shuffle_targets(ids[0].tolist(), G, rs.tolist())


def test_placement_vs_brute_random_counts(orc):
    rng = np.random.default_rng(77)
    for E, G, rpn in [(16, 4, 2), (24, 6, 3), (32, 8, 8), (48, 12, 4)]:
        A = rng.random((E, E)) < 0.2
        C = rng.integers(0, 50, (E, E)) * A
        C = np.triu(C, 1)
        C = C + C.T
        np.fill_diagonal(C, C.sum(1) // 2 + rng.integers(0, 5, E))
        C = C.astype(np.uint32)
        assert orc.place_correlated(C, G, rpn).tolist() == brute.place_correlated(C.tolist(), G, rpn)

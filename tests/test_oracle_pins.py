"""Pins for the CPU oracle: page-printed examples, closed forms, invariants and
special cases that reduce to a library routine.  None of these call the CUDA
path.  Each check is chosen so that a plausible slip in the oracle (a dropped
term, a swapped index, a transposed operand, a wrong tie-break) fails it."""
import math

import numpy as np
import pytest

from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ---------------------------------------------------------------- placement

def test_uniform_placement_worked_example(orc):
    rows = read_golden("uniform_placement_64x8.txt")
    E = int(rows[0][1]); G = int(rows[1][1])
    e2r = orc.place_uniform(E, G)
    for dev, lo, hi in (map(int, r) for r in rows[2:]):
        assert sorted(np.nonzero(e2r == dev)[0].tolist()) == list(range(lo, hi + 1))


def test_uniform_placement_rejects_uneven(orc):
    with pytest.raises(orc.OracleError) as ei:
        orc.place_uniform(10, 4)
    assert ei.value.code == orc.ERR_ARG


def test_capacity_placement_printed_variances(orc):
    torch = pytest.importorskip("torch")
    kv = {r[0]: r[1] for r in read_golden("capacity_placement_variance.txt")}
    torch.manual_seed(int(kv["seed"]))
    E, G = int(kv["E"]), int(kv["G"])
    loads = (torch.softmax(torch.randn(E), dim=0) * E).numpy().astype(np.float64)
    e2r, dev = orc.place_capacity(loads, G)
    assert np.bincount(e2r, minlength=G).sum() == E
    np.testing.assert_allclose(dev, np.bincount(e2r, weights=loads, minlength=G), rtol=1e-12)
    assert f"{np.var(dev, ddof=1):.4f}" == kv["capacity_variance"]
    uni = np.bincount(orc.place_uniform(E, G), weights=loads, minlength=G)
    assert f"{np.var(uni, ddof=1):.4f}" == kv["uniform_variance"]


def _planted_routing(E, G, T, seed, k=None):
    """Every token picks k experts from one cluster of E/G experts; clusters are
    scattered (non-contiguous) id sets."""
    rng = np.random.default_rng(seed)
    size = E // G
    k = size if k is None else k
    perm = rng.permutation(E)
    clusters = perm.reshape(G, size)
    c = rng.integers(0, G, T)
    ids = np.stack([rng.permutation(clusters[ci])[:k] for ci in c]).astype(np.int32)
    return ids, clusters, c


@pytest.mark.parametrize("E,G,rpn", [(16, 4, 4), (32, 8, 2), (64, 8, 8), (64, 16, 4), (24, 6, 1)])
def test_correlated_placement_recovers_planted_clusters(orc, E, G, rpn):
    ids, clusters, _ = _planted_routing(E, G, 4000, seed=E + G + rpn, k=max(2, E // G - 1))
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    groups = {frozenset(np.nonzero(e2r == r)[0].tolist()) for r in range(G)}
    assert groups == {frozenset(c.tolist()) for c in clusters}
    assert (np.bincount(e2r, minlength=G) == E // G).all()


def test_correlated_placement_node_level_first(orc):
    # Two super-clusters of 8 experts; inside each, two tight pairs of 4.  With
    # 2 nodes of 2 ranks the node split must follow the super-clusters.
    E, G, rpn = 16, 4, 2
    rng = np.random.default_rng(3)
    perm = rng.permutation(E)
    sub = perm.reshape(4, 4)               # rank-level clusters
    sup = [np.concatenate([sub[0], sub[1]]), np.concatenate([sub[2], sub[3]])]
    rows = []
    for _ in range(3000):
        s = rng.integers(0, 2)
        q = rng.integers(0, 2)
        a = rng.permutation(sub[2 * s + q])[:3]
        b = rng.permutation(sup[s][~np.isin(sup[s], a)])[:1]
        rows.append(np.concatenate([a, b]))
    ids = np.stack(rows).astype(np.int32)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    node = e2r // rpn
    for s in range(2):
        assert len(set(node[sup[s]].tolist())) == 1
    assert {frozenset(np.nonzero(e2r == r)[0].tolist()) for r in range(G)} == {frozenset(x.tolist()) for x in sub}


def test_correlated_placement_ties_go_to_lowest_id(orc):
    # No co-activation at all (every C is zero): seeds and growth fall back to
    # the lowest ids, i.e. the uniform contiguous map.
    E, G = 12, 3
    C = np.zeros((E, E), np.uint32)
    assert (orc.place_correlated(C, G, G) == orc.place_uniform(E, G)).all()


# ---------------------------------------------------------------- counts

def test_counts_hand_example(orc):
    # tokens: {0,1}, {0,1}, {1,2}, {0,3}   (E=4, k=2)
    ids = np.array([[[0, 1], [1, 0], [2, 1], [3, 0]]], np.int32)
    C = orc.coact(ids, 4)["coact"][0]
    want = np.array([[3, 2, 0, 1],
                     [2, 3, 1, 0],
                     [0, 1, 1, 0],
                     [1, 0, 0, 1]], np.uint32)
    assert (C == want).all()


@pytest.mark.parametrize("T,E,k", [(100, 8, 1), (257, 16, 3), (300, 32, 8), (64, 8, 8)])
def test_counts_invariants(orc, T, E, k):
    rng = np.random.default_rng(T + E + k)
    ids = np.stack([np.stack([rng.permutation(E)[:k] for _ in range(T)]) for _ in range(2)]).astype(np.int32)
    out = orc.coact(ids, E)
    for l in range(2):
        C = out["coact"][l].astype(np.int64)
        n = np.bincount(ids[l].ravel(), minlength=E)
        assert (C == C.T).all()
        assert (np.diag(C) == n).all()
        assert np.trace(C) == T * k
        assert C.sum() - np.trace(C) == T * k * (k - 1)
        assert (C.sum(axis=1) == k * n).all()
        if k == 1:
            assert (C == np.diag(np.diag(C))).all()
    M = out["trans"][0].astype(np.int64)
    n0 = np.bincount(ids[0].ravel(), minlength=E)
    n1 = np.bincount(ids[1].ravel(), minlength=E)
    assert (M.sum(axis=1) == k * n0).all()
    assert (M.sum(axis=0) == k * n1).all()
    assert M.sum() == T * k * k


def test_counts_reduce_to_one_hot_product(orc):
    # C = A^T A and M = A0^T A1 for the one-hot token x expert matrices A:
    # a textbook identity, evaluated here with numpy's matmul.
    rng = np.random.default_rng(7)
    T, E, k, L = 500, 24, 5, 3
    ids = np.stack([np.stack([rng.permutation(E)[:k] for _ in range(T)]) for _ in range(L)]).astype(np.int32)
    A = np.zeros((L, T, E), np.int64)
    for l in range(L):
        np.put_along_axis(A[l], ids[l].astype(np.int64), 1, axis=1)
    out = orc.coact(ids, E)
    for l in range(L):
        assert (out["coact"][l] == A[l].T @ A[l]).all()
    for l in range(L - 1):
        assert (out["trans"][l] == A[l].T @ A[l + 1]).all()


def test_transitions_identical_layers(orc):
    rng = np.random.default_rng(11)
    T, E = 200, 16
    one = np.stack([rng.permutation(E)[:1] for _ in range(T)]).astype(np.int32)
    M = orc.coact(np.stack([one, one]), E)["trans"][0]
    assert (M == np.diag(np.diag(M))).all()
    many = np.stack([rng.permutation(E)[:4] for _ in range(T)]).astype(np.int32)
    out = orc.coact(np.stack([many, many[:, ::-1].copy()]), E)
    assert (out["trans"][0] == out["coact"][0]).all()


def test_counts_reject_bad_ids(orc):
    bad = np.array([[[0, 0]]], np.int32)
    with pytest.raises(orc.OracleError) as ei:
        orc.coact(bad, 4)
    assert ei.value.code == orc.ERR_DATA
    with pytest.raises(orc.OracleError):
        orc.coact(np.array([[[0, 4]]], np.int32), 4)
    with pytest.raises(orc.OracleError):
        orc.coact(np.array([[[-1, 2]]], np.int32), 4)


# ---------------------------------------------------------------- Ochiai

def test_ochiai_hand_example(orc):
    # |A0| = 4, |A1| = 9, |A0 & A1| = 3  ->  3 / sqrt(36) = 0.5
    ids = [[0, 1]] * 3 + [[0, 2]] + [[1, 2]] * 6
    S = orc.coact(np.array([ids], np.int32), 3)["ochiai"][0]
    assert S[0, 1] == np.float32(0.5) and S[1, 0] == np.float32(0.5)
    assert S[0, 2] == np.float32(1.0 / math.sqrt(4 * 7))
    assert S[1, 2] == np.float32(6.0 / math.sqrt(9 * 7))


def test_ochiai_special_cases(orc):
    # experts 0,1 always together (identical token sets -> 1); expert 2 and 3
    # never together (disjoint -> 0); expert 4 unused (-> 0, diagonal 0)
    ids = [[0, 1, 2]] * 5 + [[0, 1, 3]] * 4
    S = orc.coact(np.array([ids], np.int32), 5)["ochiai"][0]
    assert S[0, 1] == 1.0 and S[1, 0] == 1.0
    assert S[2, 3] == 0.0
    assert S[4, 4] == 0.0 and (S[4] == 0).all()
    for e in range(4):
        assert S[e, e] == 1.0
    rng = np.random.default_rng(5)
    ids = np.stack([rng.permutation(32)[:6] for _ in range(400)]).astype(np.int32)
    S = orc.coact(ids[None], 32)["ochiai"][0]
    assert (S >= 0).all() and (S <= 1).all() and (S == S.T).all()


# ---------------------------------------------------------------- plan

def _uniform_ids(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k,G,rpn", [(64, 8, 2, 4, 2), (96, 16, 3, 8, 8), (128, 32, 8, 8, 1),
                                         (120, 12, 4, 6, 3), (64, 64, 8, 64, 8)])
def test_plan_invariants(orc, T, E, k, G, rpn):
    rng = np.random.default_rng(T * 7 + G)
    ids = _uniform_ids(rng, T, E, k)
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    p = orc.plan(ids, E, G, rpn, e2r)
    R = p["R"]
    assert T <= R <= T * k
    assert p["counts"].sum() == R
    off = p["offsets"]
    assert off[0] == 0 and off[-1] == R and (np.diff(off) >= 0).all()
    src = np.arange(T) // (T // G)
    # each (token, destination) pair appears exactly once, in (dst, src, t) order
    rt = p["row_token"]
    dst_of_row = np.repeat(np.arange(G), [p["counts"][:, r].sum() for r in range(G)])
    keys = list(zip(dst_of_row.tolist(), src[rt].tolist(), rt.tolist()))
    assert keys == sorted(keys) and len(set(keys)) == R
    want = {(int(e2r[e]), t) for t in range(T) for e in ids[t]}
    assert {(d, t) for d, _, t in keys} == want
    for t in range(T):
        for j in range(k):
            r = p["row_of"][t, j]
            assert rt[r] == t and dst_of_row[r] == e2r[ids[t, j]]
            assert p["row_jmask"][r] >> j & 1
        assert int(p["dest_mask"][t]) == sum(1 << int(x) for x in set(e2r[ids[t]].tolist()))
    assert p["R_remote"] == sum(1 for d, s, t in keys if d != s)
    if rpn == G:
        assert p["V"] == 0
    if rpn == 1:
        assert p["V"] == p["R_remote"]


def test_plan_k1_is_stable_counting_sort(orc):
    rng = np.random.default_rng(1)
    T, E, G = 400, 16, 4
    ids = rng.integers(0, E, (T, 1)).astype(np.int32)
    e2r = orc.place_uniform(E, G)
    p = orc.plan(ids, E, G, 2, e2r)
    assert p["R"] == T
    assert (p["row_token"] == np.argsort(e2r[ids[:, 0]], kind="stable")).all()


def test_plan_single_rank(orc):
    rng = np.random.default_rng(2)
    T, E, k = 77, 8, 3
    ids = _uniform_ids(rng, T, E, k)
    p = orc.plan(ids, E, 1, 1, np.zeros(E, np.int32))
    assert p["R"] == T and (p["row_token"] == np.arange(T)).all()
    assert p["R_remote"] == 0 and p["V"] == 0 and p["local"] == T * k


def test_plan_src_rank_order(orc):
    rng = np.random.default_rng(4)
    T, E, k, G = 90, 12, 3, 6
    ids = _uniform_ids(rng, T, E, k)
    e2r = orc.place_uniform(E, G)
    src = rng.integers(0, G, T).astype(np.int32)
    p = orc.plan(ids, E, G, 3, e2r, src_rank=src)
    # (dst, src, t) order with explicit source ranks: a lexsort by numpy
    pairs = [(int(e2r[e]), int(src[t]), t) for t in range(T) for e in set(ids[t].tolist())]
    pairs = sorted(set((d, s, t) for d, s, t in pairs))
    assert p["row_token"].tolist() == [t for _, _, t in pairs]
    local = sum(1 for t in range(T) for e in ids[t] if e2r[e] == src[t])
    assert p["local"] == local


def test_local_share_uniform_routing(orc):
    kv = {r[0]: r[1] for r in read_golden("local_share_uniform.txt")}
    G, share = int(kv["G"]), float(kv["share"])
    rng = np.random.default_rng(9)
    T, E, k = 4096, 64, 2
    ids = _uniform_ids(rng, T, E, k)
    p = orc.plan(ids, E, G, G, orc.place_uniform(E, G))
    got = p["local"] / (T * k)
    sigma = math.sqrt(share * (1 - share) / (T * k))
    assert abs(got - share) < 4 * sigma
    # exact variant: every token picks one expert on every rank -> exactly 1/G
    per = E // G
    ids = np.stack([np.array([r * per + rng.integers(per) for r in range(G)]) for _ in range(T)]).astype(np.int32)
    p = orc.plan(ids, E, G, G, orc.place_uniform(E, G))
    assert p["local"] == T and p["local"] / (T * G) == share
    assert p["R"] == T * G


def test_plan_rejects_bad_input(orc):
    ids = np.array([[0, 1], [2, 2]], np.int32)
    with pytest.raises(orc.OracleError):
        orc.plan(ids, 4, 2, 2, orc.place_uniform(4, 2))
    ids = np.array([[0, 1], [2, 3]], np.int32)
    with pytest.raises(orc.OracleError):
        orc.plan(ids, 4, 2, 2, np.array([0, 0, 1, 2], np.int32))
    with pytest.raises(orc.OracleError):
        orc.plan(ids, 4, 2, 2, orc.place_uniform(4, 2), src_rank=np.array([0, 5], np.int32))


# ---------------------------------------------------------------- permute / combine

def test_permute_gathers_rows(orc):
    rng = np.random.default_rng(6)
    T, E, k, G, d = 50, 8, 3, 4, 5
    ids = _uniform_ids(rng, 52, E, k)[:T + 2]
    x = rng.standard_normal((52, d)).astype(np.float32)
    p = orc.plan(ids, E, G, 2, orc.place_uniform(E, G))
    send = orc.permute(x, p["row_token"])
    assert (send == x[p["row_token"]]).all()


def test_combine_identity_round_trip(orc):
    from synth import f32_to_bf16_bits, bf16_bits_to_f32
    rng = np.random.default_rng(8)
    T, E, k, G, d = 64, 16, 4, 4, 24
    ids = _uniform_ids(rng, T, E, k)
    z = rng.standard_normal((T, k)).astype(np.float32)
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    xb = f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    p = orc.plan(ids, E, G, 2, orc.place_uniform(E, G))
    Y = orc.permute(xb, p["row_token"])
    out = orc.combine(Y, p["row_of"], w, y_is_bf16=True)
    x = bf16_bits_to_f32(xb).astype(np.float64)
    np.testing.assert_allclose(out, x * w.astype(np.float64).sum(1, keepdims=True), rtol=1e-15, atol=0)
    # weights sum to 1 within fp32 rounding, so rounding back to bf16 returns x exactly
    assert (f32_to_bf16_bits(out.astype(np.float32)) == xb).all()


def test_combine_matches_einsum_and_exact(orc):
    from oracle import brute
    rng = np.random.default_rng(10)
    T, k, d, Rm = 12, 3, 7, 20
    Y = rng.standard_normal((Rm, d)).astype(np.float32)
    idx = rng.integers(0, Rm, (T, k)).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    out = orc.combine(Y, idx, w, y_is_bf16=False)
    ref = np.einsum("tj,tjc->tc", w.astype(np.float64), Y[idx].astype(np.float64))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-14)
    exact = brute.combine_exact(Y.tolist(), idx.tolist(), w.tolist())
    mag = np.einsum("tj,tjc->tc", np.abs(w.astype(np.float64)), np.abs(Y[idx].astype(np.float64)))
    for t in range(T):
        for c in range(d):
            assert abs(out[t, c] - float(exact[t][c])) <= k * 2.0 ** -53 * mag[t, c] * 1.0001
    bad = idx.copy(); bad[0, 0] = Rm
    with pytest.raises(orc.OracleError):
        orc.combine(Y, bad, w, y_is_bf16=False)


# ---------------------------------------------------------------- shuffle

def test_shuffle_planted_clusters(orc):
    E, G, T = 32, 4, 3000
    ids, clusters, c = _planted_routing(E, G, T, seed=21, k=3)
    stats = orc.coact(np.stack([ids, ids]), E)
    e2r = orc.place_correlated(stats["coact"][0], G, G)
    rs = orc.rank_score(stats["trans"][0], e2r, G)
    tgt = orc.shuffle_targets(ids, E, G, rs)
    assert (tgt == e2r[clusters[c, 0]]).all()
    p = orc.plan(ids, E, G, G, e2r, src_rank=tgt)
    assert p["R"] == T and p["R_remote"] == 0 and p["local"] == T * 3


def test_shuffle_ties_lowest_rank(orc):
    rs = np.zeros((4, 3), np.uint32)
    rs[0] = [5, 7, 7]
    rs[1] = [2, 0, 0]
    ids = np.array([[0, 1], [2, 3]], np.int32)
    tgt = orc.shuffle_targets(ids, 4, 3, rs)
    assert tgt.tolist() == [0, 0]   # [7, 7, 7] -> 0 ; [0, 0, 0] -> 0
    rs[1] = [0, 0, 1]
    assert orc.shuffle_targets(ids, 4, 3, rs).tolist() == [2, 0]


def test_rank_score_definition(orc):
    rng = np.random.default_rng(12)
    E, G = 16, 4
    M = rng.integers(0, 1000, (E, E)).astype(np.uint32)
    e2r = rng.permutation(orc.place_uniform(E, G)).astype(np.int32)
    rs = orc.rank_score(M, e2r, G)
    onehot = np.zeros((E, G), np.int64)
    onehot[np.arange(E), e2r] = 1
    assert (rs == M.astype(np.int64) @ onehot).all()


def test_capacity_placement_hand_example(orc):
    # loads 5, 4, 3, 2 on 2 devices, largest first onto the least-loaded device
    # (equal loads: the lower device): 5 -> d0 ; 4 -> d1 ; 3 -> d1 (4 < 5) ;
    # 2 -> d0 (5 < 7)  =>  device loads 7, 7
    e2r, dev = orc.place_capacity(np.array([2.0, 5.0, 3.0, 4.0]), 2)
    assert e2r.tolist() == [0, 0, 1, 1] and dev.tolist() == [7.0, 7.0]
    # all loads equal: experts in id order, each onto the lowest least-loaded device
    e2r, _ = orc.place_capacity(np.ones(6), 3)
    assert e2r.tolist() == [0, 1, 2, 0, 1, 2]

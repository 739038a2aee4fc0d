"""Parity of the replica assignment and of the plan over per-pick serving
ranks with the oracle ("Cobalt ...", "Problem Formulation": tasks run on a
replica of their expert; the assignment reaches the fewest remote nodes).
Integers throughout: bit-exact."""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import WORKLOADS, make_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cap():
    from co_activation_placement_b200 import build
    build.build()
    import co_activation_placement_b200 as cap
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    cap.lib()
    return cap


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def check_plan(p, o, T):
    R = o["R"]
    assert int(host(p.err)[0]) == 0
    assert host(p.summary).tolist() == o["summary"].tolist()
    assert (host(p.counts) == o["counts"]).all() and (host(p.offsets) == o["offsets"]).all()
    assert (host(p.row_token)[:R] == o["row_token"]).all()
    assert (host(p.row_jmask)[:R] == o["row_jmask"]).all()
    assert (host(p.row_of)[:T] == o["row_of"]).all()


@pytest.mark.parametrize("name,extra,with_src", [("one_node", 2, False), ("ep32", 1, True), ("ep32", 2, False),
                                                 ("large_ep64", 1, True), ("large_ep64", 2, False)])
def test_replica_assignment_and_plan(cap, name, extra, with_src):
    w = WORKLOADS[name]
    ids = make_routing(w)[0]
    cal = make_routing(w, seed=1)[0]
    C = orc.coact(cal[None], w.E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, w.G, w.rpn)
    rr, nr = cap.place_replicas(C, w.G, w.rpn, e2r, extra)
    rr_o, nr_o = orc.place_replicas(C, w.G, w.rpn, e2r, extra)
    assert (rr == rr_o).all() and (nr == nr_o).all()
    rng = np.random.default_rng(7)
    src = rng.integers(0, w.G, w.T).astype(np.int32) if with_src else None
    pr, nrem = cap.assign_replicas(dev(ids), w.E, w.G, w.rpn, dev(rr), dev(nr),
                                   src_rank=None if src is None else dev(src))
    pr_o, nrem_o = orc.assign_replicas(ids, w.E, w.G, w.rpn, rr_o, nr_o, src_rank=src)
    assert (host(pr)[: w.T] == pr_o).all() and (host(nrem)[: w.T] == nrem_o).all()
    p = cap.plan_dispatch_ranks(dev(ids), w.E, w.G, w.rpn, pr, src_rank=None if src is None else dev(src))
    o = orc.plan(ids, w.E, w.G, w.rpn, None, src_rank=src, pick_rank=pr_o)
    check_plan(p, o, w.T)
    assert o["V"] == int(nrem_o.sum())
    # replicas never add remote nodes compared with the single placement
    base = orc.plan(ids, w.E, w.G, w.rpn, e2r, src_rank=src)
    assert o["V"] <= base["V"]


def test_replica_assignment_small_and_errors(cap):
    rng = np.random.default_rng(3)
    T, E, k, G, rpn = 999, 16, 3, 8, 2
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    rr, nr = orc.place_replicas(C, G, rpn, e2r, 2)
    src = rng.integers(0, G, T).astype(np.int32)
    pr, nrem = cap.assign_replicas(dev(ids), E, G, rpn, dev(rr), dev(nr), src_rank=dev(src))
    pr_o, nrem_o = orc.assign_replicas(ids, E, G, rpn, rr, nr, src_rank=src)
    assert (host(pr)[:T] == pr_o).all() and (host(nrem)[:T] == nrem_o).all()
    # an out-of-range id is reported and its token gets -1
    bad = ids.copy()
    bad[5, 1] = E + 3
    err = cap.new_err("cuda")
    pr2, nrem2 = cap.assign_replicas(dev(bad), E, G, rpn, dev(rr), dev(nr), src_rank=dev(src), err=err)
    assert int(host(err)[0]) == cap.DERR_ID_RANGE and (host(pr2)[5] == -1).all()
    # pick ranks out of range are reported by the plan
    prb = host(pr).copy()
    prb[7, 0] = G
    p = cap.plan_dispatch_ranks(dev(ids), E, G, rpn, dev(prb[:T]), src_rank=dev(src))
    assert int(host(p.err)[0]) == cap.DERR_RANK_RANGE
    with pytest.raises(cap.MoeError):
        cap.assign_replicas(dev(ids), E, 16, 1, dev(rr), dev(nr), src_rank=dev(src))   # 16 nodes > 8


# ------------------------------------------------- load-capped assignment

@pytest.mark.parametrize("name,extra,eps,with_src", [("one_node", 2, 0.0, False), ("one_node", 2, 0.1, True),
                                                     ("ep32", 2, 0.05, False), ("ep32", 1, 0.2, True),
                                                     ("large_ep64", 1, 0.1, False), ("large_ep64", 2, 0.0, True),
                                                     ("large_ep64", 2, float("inf"), False)])
def test_capped_assignment_full_size(cap, name, extra, eps, with_src):
    """The load-capped assignment ("Cobalt", "Problem Formulation": sum_e w_r^e
    <= (1 + eps) K T / G) bit for bit against the oracle's token-order greedy
    at the workloads' full sizes: picks, remote nodes per token, rank loads;
    eps = inf equals the uncapped assignment; the plan over the picks too."""
    w = WORKLOADS[name]
    ids = make_routing(w)[0]
    cal = make_routing(w, seed=1)[0]
    C = orc.coact(cal[None], w.E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, w.G, w.rpn)
    rr, nr = orc.place_replicas(C, w.G, w.rpn, e2r, extra)
    rng = np.random.default_rng(11)
    src = rng.integers(0, w.G, w.T).astype(np.int32) if with_src else None
    err = cap.new_err("cuda")
    pr, nrem, load = cap.assign_replicas_capped(dev(ids), w.E, w.G, w.rpn, dev(rr), dev(nr), eps,
                                                src_rank=None if src is None else dev(src), err=err)
    pr_o, nrem_o, load_o = orc.assign_replicas_capped(ids, w.E, w.G, w.rpn, rr, nr, eps, src_rank=src)
    assert int(host(err)[0]) == 0
    assert (host(pr)[: w.T] == pr_o).all()
    assert (host(nrem)[: w.T] == nrem_o).all()
    assert host(load).tolist() == load_o.tolist()
    if eps == float("inf"):
        pu, nu = orc.assign_replicas(ids, w.E, w.G, w.rpn, rr, nr, src_rank=src)
        assert (pr_o == pu).all() and (nrem_o == nu).all()
    p = cap.plan_dispatch_ranks(dev(ids), w.E, w.G, w.rpn, pr, src_rank=None if src is None else dev(src))
    check_plan(p, orc.plan(ids, w.E, w.G, w.rpn, None, src_rank=src, pick_rank=pr_o), w.T)


@pytest.mark.parametrize("T,E,k,G,rpn,eps", [(999, 16, 3, 8, 2, 0.0), (5000, 32, 4, 8, 4, 0.03),
                                             (1, 16, 3, 8, 2, 0.0), (130, 64, 8, 64, 8, 0.0),
                                             (4096, 16, 2, 4, 1, 0.5), (777, 24, 6, 8, 1, 0.01)])
def test_capped_assignment_shapes(cap, T, E, k, G, rpn, eps):
    """Ragged token counts, one token, tight caps (many closing rounds), every
    rank its own node, explicit source ranks."""
    rng = np.random.default_rng(T + E + G)
    hot = rng.permutation(E)[: k + 2]
    ids = np.where((rng.random(T) < 0.8)[:, None], hot[np.argsort(rng.random((T, hot.size)), axis=1)[:, :k]],
                   np.argsort(rng.random((T, E)), axis=1)[:, :k]).astype(np.int32)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    rr, nr = orc.place_replicas(C, G, rpn, e2r, 2)
    src = rng.integers(0, G, T).astype(np.int32)
    pr, nrem, load = cap.assign_replicas_capped(dev(ids), E, G, rpn, dev(rr), dev(nr), eps, src_rank=dev(src))
    pr_o, nrem_o, load_o = orc.assign_replicas_capped(ids, E, G, rpn, rr, nr, eps, src_rank=src)
    assert (host(pr)[:T] == pr_o).all() and (host(nrem)[:T] == nrem_o).all()
    assert host(load).tolist() == load_o.tolist()


def test_capped_assignment_errors(cap):
    rng = np.random.default_rng(4)
    T, E, k, G, rpn = 600, 16, 3, 8, 2
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    rr, nr = orc.place_replicas(C, G, rpn, orc.place_correlated(C, G, rpn), 1)
    bad = ids.copy()
    bad[9, 2] = E + 1
    err = cap.new_err("cuda")
    pr, nrem, load = cap.assign_replicas_capped(dev(bad), E, G, rpn, dev(rr), dev(nr), 0.1, err=err)
    assert int(host(err)[0]) == cap.DERR_ID_RANGE and (host(pr)[9] == -1).all()
    assert int(host(load).sum()) == (T - 1) * k          # the invalid token counts for no rank
    for eps in (-0.5, float("nan")):
        with pytest.raises(cap.MoeError):
            cap.assign_replicas_capped(dev(ids), E, G, rpn, dev(rr), dev(nr), eps)
    # the context stays usable
    pr, _, _ = cap.assign_replicas_capped(dev(ids), E, G, rpn, dev(rr), dev(nr), 0.1)
    assert (host(pr)[:T] == orc.assign_replicas_capped(ids, E, G, rpn, rr, nr, 0.1)[0]).all()


@pytest.mark.parametrize("seed", range(10))
def test_capped_assignment_random(cap, seed):
    """Random shapes, replica budgets and tolerances, with skewed expert
    popularity so that many ranks reach the cap at scattered tokens: every
    round re-evaluates only the tokens whose options changed."""
    rng = np.random.default_rng(900 + seed)
    rpn = int(rng.choice([1, 2, 4, 8]))
    G = rpn * int(rng.integers(1, min(8, 64 // rpn) + 1))
    E = G * int(rng.integers(1, 9))
    k = int(rng.integers(1, min(8, E) + 1))
    T = int(rng.integers(1, 20000))
    if rng.random() < 0.5:
        T = T // G * G or G
    eps = float(rng.choice([0.0, 0.01, 0.05, 0.3]))
    extra = int(rng.integers(1, 4))
    pop = rng.zipf(1.3, E).astype(np.float64)
    pop /= pop.sum()
    ids = np.stack([rng.choice(E, k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)
    C = orc.coact(ids[None], E, want=("coact",))["coact"][0]
    e2r = orc.place_correlated(C, G, rpn)
    rr, nr = orc.place_replicas(C, G, rpn, e2r, extra)
    src = rng.integers(0, G, T).astype(np.int32) if (T % G or rng.random() < 0.5) else None
    err = cap.new_err("cuda")
    pr, nrem, load = cap.assign_replicas_capped(dev(ids), E, G, rpn, dev(rr), dev(nr), eps,
                                                src_rank=None if src is None else dev(src), err=err)
    pr_o, nrem_o, load_o = orc.assign_replicas_capped(ids, E, G, rpn, rr, nr, eps, src_rank=src)
    assert int(host(err)[0]) == 0
    assert (host(pr)[:T] == pr_o).all() and (host(nrem)[:T] == nrem_o).all()
    assert host(load).tolist() == load_o.tolist()


@pytest.mark.parametrize("blocks", [1, 3, 64, 0])
def test_capped_assignment_grid_sizes(cap, blocks):
    """The result does not depend on the cooperative grid (moe_cooperative_blocks):
    one block, a few, one per rank, one per SM.  With 1 and 3 blocks a block's
    131,072 / B tokens are too many for their pick-rank sets to sit in shared
    memory, so those grids also cover the kernel without them."""
    w = WORKLOADS["large_ep64"]
    ids = make_routing(w)[0]
    cal = make_routing(w, seed=1)[0]
    C = orc.coact(cal[None], w.E, want=("coact",))["coact"][0]
    rr, nr = orc.place_replicas(C, w.G, w.rpn, orc.place_correlated(C, w.G, w.rpn), 1)
    prev = cap.cooperative_blocks(blocks)
    try:
        err = cap.new_err("cuda")
        pr, nrem, load = cap.assign_replicas_capped(dev(ids), w.E, w.G, w.rpn, dev(rr), dev(nr), 0.1, err=err)
        torch.cuda.synchronize()
    finally:
        cap.cooperative_blocks(prev)
    pr_o, nrem_o, load_o = orc.assign_replicas_capped(ids, w.E, w.G, w.rpn, rr, nr, 0.1)
    assert int(host(err)[0]) == 0
    assert (host(pr)[: w.T] == pr_o).all() and (host(nrem)[: w.T] == nrem_o).all()
    assert host(load).tolist() == load_o.tolist()


@pytest.mark.parametrize("name,overlap", [("ep32", True), ("ep32", False), ("large_ep64", True)])
def test_pipeline_with_capped_replicas(cap, name, overlap):
    """A whole step with the load-capped assignment (eps = 0.1): every layer's
    plan over the picks the oracle's token-order greedy makes, with the
    previous layer's shuffle targets as source ranks; beside the row traffic
    (one block per rank) or in line."""
    from co_activation_placement_b200 import pipeline
    from synth import make_gates, make_hidden
    w = WORKLOADS[name]
    ids = make_routing(w)
    ids_cal = make_routing(w, seed=w.seed + 1)
    hp = pipeline.prepare(w.E, w.G, w.rpn, ids, make_gates(w), make_hidden(w), w.dtype, ids_cal,
                          shuffle=True, out_dtype=torch.float32, replica_extra=1, replica_eps=0.1,
                          overlap=overlap)
    hp.step()
    torch.cuda.synchronize()
    assert int(host(hp.err)[0]) == 0
    oc = orc.coact(ids_cal, w.E, want=("coact", "trans"))
    e2r = [orc.place_correlated(oc["coact"][l], w.G, w.rpn) for l in range(w.L)]
    src = None
    for l in range(w.L):
        rr, nr = orc.place_replicas(oc["coact"][l], w.G, w.rpn, e2r[l], 1)
        pr, _, load = orc.assign_replicas_capped(ids[l], w.E, w.G, w.rpn, rr, nr, 0.1, src_rank=src)
        assert host(hp.rank_load[l]).tolist() == load.tolist()
        op = orc.plan(ids[l], w.E, w.G, w.rpn, None, src_rank=src, pick_rank=pr)
        assert host(hp.plans[l].summary).tolist() == op["summary"].tolist()
        assert (host(hp.plans[l].row_of)[: w.T] == op["row_of"]).all()
        if l + 1 < w.L:
            src = orc.shuffle_targets(ids[l], w.E, w.G, orc.rank_score(oc["trans"][l], e2r[l + 1], w.G))

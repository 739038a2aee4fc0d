"""The capacity-balanced shuffle on the GPU against the oracle: random
shapes with many equal scores, exact and loose capacities, the
unconstrained limit, the workloads at full size, a CUDA graph replay, and
data errors reported in the error word."""
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


def run(cap, ids, E, G, rs, capacity):
    info = torch.zeros(6, dtype=torch.int64, device="cuda")
    err = cap.new_err("cuda")
    tg = cap.shuffle_balanced(dev(ids), E, G, dev(rs), capacity, info=info, err=err)
    return host(tg)[: ids.shape[0]], host(info), int(host(err)[0])


@pytest.mark.parametrize("seed", range(16))
def test_random_shapes(cap, seed):
    rng = np.random.default_rng(500 + seed)
    G = int(rng.choice([1, 2, 3, 8, 16, 33, 64]))
    E = G * int(rng.integers(1, max(2, 256 // G) + 1))
    k = int(rng.integers(1, min(8, E) + 1))
    T = int(rng.integers(1, 6000))
    capacity = -(-T // G) + int(rng.choice([0, 0, 1, 7]))
    hi = int(rng.choice([2, 4, 50, 2 ** 20, 2 ** 32 - 1]))          # small ranges: many equal scores
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    rs = rng.integers(0, hi, (E, G), dtype=np.uint64).astype(np.uint32)
    got, info, err = run(cap, ids, E, G, rs, capacity)
    assert err == 0
    assert (got == orc.shuffle_balanced(ids, E, G, rs, capacity)).all()
    assert info[0] >= 1 and info[1] >= T
    assert np.bincount(got, minlength=G).max() <= capacity


def test_unbounded_capacity_equals_argmax(cap):
    rng = np.random.default_rng(7)
    T, E, k, G = 3000, 64, 4, 16
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    rs = rng.integers(0, 30, (E, G)).astype(np.uint32)
    got, info, err = run(cap, ids, E, G, rs, T)
    assert err == 0 and info[0] == 1
    assert (got == host(cap.shuffle_targets(dev(ids), E, G, dev(rs)))[:T]).all()


@pytest.mark.parametrize("name", ["one_node", "ep32", "large_ep64"])
def test_workloads_full_size(cap, name):
    w = WORKLOADS[name]
    ids = make_routing(w, seed=0)
    cal = make_routing(w, seed=1)
    oc = orc.coact(cal, w.E, want=("coact", "trans"))
    e2r1 = orc.place_correlated(oc["coact"][1], w.G, w.rpn)
    rs = orc.rank_score(oc["trans"][0], e2r1, w.G)
    capacity = w.T // w.G
    got, info, err = run(cap, ids[0], w.E, w.G, rs, capacity)
    assert err == 0
    want = orc.shuffle_balanced(ids[0], w.E, w.G, rs, capacity)
    assert (got == want).all()
    assert (np.bincount(got, minlength=w.G) == capacity).all()


def test_repeat_and_graph_replay(cap):
    rng = np.random.default_rng(9)
    T, E, k, G = 8192, 128, 6, 32
    ids = dev(np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32))
    rs = dev(rng.integers(0, 8, (E, G)).astype(np.uint32))
    a = host(cap.shuffle_balanced(ids, E, G, rs, T // G))[:T].copy()
    b = host(cap.shuffle_balanced(ids, E, G, rs, T // G))[:T].copy()
    assert (a == b).all()
    tg = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    err = cap.new_err("cuda")
    ws = torch.empty(cap.shuffle_balanced_workspace(T, G, T // G), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        cap.shuffle_balanced(ids, E, G, rs, T // G, target=tg, err=err, ws=ws)     # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    tg.fill_(-1)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cap.shuffle_balanced(ids, E, G, rs, T // G, target=tg, err=err, ws=ws)
    g.replay()
    g.replay()
    assert int(host(err)[0]) == 0
    assert (host(tg) == a).all()


def test_id_out_of_range_is_reported(cap):
    rng = np.random.default_rng(3)
    T, E, k, G = 512, 16, 2, 4
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    ids[17, 1] = E + 3
    rs = rng.integers(0, 10, (E, G)).astype(np.uint32)
    got, info, err = run(cap, ids, E, G, rs, T // G)
    assert err == cap.DERR_ID_RANGE
    assert (np.bincount(got, minlength=G) == T // G).all()    # every token still placed


def test_empty_and_argument_errors(cap):
    info = torch.full((6,), 9, dtype=torch.int64, device="cuda")
    cap.shuffle_balanced(torch.zeros((0, 2), dtype=torch.int32, device="cuda"), 4, 2,
                         torch.ones((4, 2), dtype=torch.uint32, device="cuda"), 0, info=info)
    assert host(info).tolist() == [0] * 6
    with pytest.raises(cap.MoeError) as ei:
        cap.shuffle_balanced(torch.zeros((9, 1), dtype=torch.int32, device="cuda"), 1, 4,
                             torch.ones((1, 4), dtype=torch.uint32, device="cuda"), 2)
    assert ei.value.status == cap.MOE_ERR_ARG


@pytest.mark.parametrize("blocks", [1, 5, 64])
def test_grid_sizes(cap, blocks):
    """The result does not depend on the cooperative grid (moe_cooperative_blocks):
    blocks that own several ranks, or none."""
    w = WORKLOADS["large_ep64"]
    ids = make_routing(w)[0]
    cal = make_routing(w, seed=w.seed + 1)
    oc = orc.coact(cal[:2], w.E, want=("coact", "trans"))
    rs = orc.rank_score(oc["trans"][0], orc.place_correlated(oc["coact"][1], w.G, w.rpn), w.G)
    prev = cap.cooperative_blocks(blocks)
    try:
        got, info, err = run(cap, ids, w.E, w.G, rs, w.T // w.G)
    finally:
        cap.cooperative_blocks(prev)
    assert err == 0
    assert (got == orc.shuffle_balanced(ids, w.E, w.G, rs, w.T // w.G)).all()


@pytest.mark.parametrize("name,overlap", [("one_node", True), ("one_node", False), ("large_ep64", True),
                                          ("large_ep64", False)])
def test_pipeline_with_balanced_shuffle(cap, name, overlap):
    """A whole step with capped shards: every layer's plan uses the previous
    layer's balanced targets as source ranks, as the oracle does; the shuffle
    beside the row traffic (one block per rank) or in line."""
    from co_activation_placement_b200 import pipeline
    from synth import make_gates, make_hidden
    w = WORKLOADS[name]
    ids = make_routing(w)
    ids_cal = make_routing(w, seed=w.seed + 1)
    hp = pipeline.prepare(w.E, w.G, w.rpn, ids, make_gates(w), make_hidden(w), w.dtype, ids_cal,
                          shuffle=True, out_dtype=torch.float32, shuffle_capacity=w.T // w.G,
                          overlap=overlap)
    hp.step()
    torch.cuda.synchronize()
    assert int(host(hp.err)[0]) == 0
    oc = orc.coact(ids_cal, w.E, want=("coact", "trans"))
    e2r = [orc.place_correlated(oc["coact"][l], w.G, w.rpn) for l in range(w.L)]
    src = None
    for l in range(w.L):
        op = orc.plan(ids[l], w.E, w.G, w.rpn, e2r[l], src_rank=src)
        assert host(hp.plans[l].summary).tolist() == op["summary"].tolist()
        assert (host(hp.plans[l].row_of)[: w.T] == op["row_of"]).all()
        if l + 1 < w.L:
            rs = orc.rank_score(oc["trans"][l], e2r[l + 1], w.G)
            src = orc.shuffle_balanced(ids[l], w.E, w.G, rs, w.T // w.G)
            assert (host(hp.targets[l]) == src).all()
            assert int(host(hp.shuffle_info)[l][0]) >= 1

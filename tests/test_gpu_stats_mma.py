"""Co-activation statistics on the tensor cores (C_l = X_l X_l^T and
M_l = X_l X_{l+1}^T with tcgen05.mma kind::i8) against the oracle, and
against the shared-memory histogram path on the same inputs: every count
bit-exact, Ochiai bit-exact."""
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
    yield cap
    cap.coact_stats_method(0)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def check(cap, ids, E, method):
    cap.coact_stats_method(method)
    try:
        g = cap.coact_stats(dev(ids), E)
        torch.cuda.synchronize()
    finally:
        cap.coact_stats_method(0)
    o = orc.coact(ids, E)
    assert int(host(g["err"])[0]) == 0
    assert (host(g["coact"]) == o["coact"]).all()
    assert (host(g["ochiai"]).view(np.uint32) == o["ochiai"].view(np.uint32)).all()
    if ids.shape[0] > 1:
        assert (host(g["trans"]) == o["trans"]).all()


def test_one_block_first(cap):
    # the smallest launch of the tensor-core path: one product, one slice, one stage
    rng = np.random.default_rng(0)
    ids = np.argsort(rng.random((1, 100, 32)), axis=2)[:, :, :2].astype(np.int32)
    check(cap, ids, 32, 2)


@pytest.mark.parametrize("L,T,k,E", [(2, 300, 3, 32), (3, 1000, 2, 48), (2, 129, 8, 160), (1, 5000, 4, 64),
                                     (4, 4097, 8, 256), (2, 128, 1, 128), (3, 20000, 6, 96), (2, 1, 2, 32),
                                     # two layers per block: odd L (a last block with one tile), E < 128,
                                     # slices of one ragged stage and empty slices
                                     (5, 3001, 8, 128), (8, 2000, 4, 64), (4, 777, 5, 112), (7, 40000, 8, 128),
                                     (6, 90, 3, 80)])
def test_shapes(cap, L, T, k, E):
    rng = np.random.default_rng(L * 1000 + T + E)
    ids = np.stack([np.argsort(rng.random((T, E)), axis=1)[:, :k] for _ in range(L)]).astype(np.int32)
    check(cap, ids, E, 2)


@pytest.mark.parametrize("name", ["one_node", "ep32", "large_ep64"])
def test_workloads_both_methods(cap, name):
    w = WORKLOADS[name]
    ids = make_routing(w)
    check(cap, ids, w.E, 2)
    check(cap, ids, w.E, 1)


def test_sweep_sample_both_methods(cap):
    w = WORKLOADS["stats_sweep"]
    ids = make_routing(w, T=131072)
    check(cap, ids, w.E, 2)


def test_partial_outputs_and_errors(cap):
    rng = np.random.default_rng(5)
    L, T, k, E = 3, 9000, 4, 128
    ids = np.stack([np.argsort(rng.random((T, E)), axis=1)[:, :k] for _ in range(L)]).astype(np.int32)
    o = orc.coact(ids, E)
    cap.coact_stats_method(2)
    try:
        g = cap.coact_stats(dev(ids), E, want=("trans",))
        assert (host(g["trans"]) == o["trans"]).all()
        g = cap.coact_stats(dev(ids), E, want=("coact",))
        assert (host(g["coact"]) == o["coact"]).all()
        bad = ids.copy()
        bad[1, 77, 2] = E + 5
        assert int(host(cap.coact_stats(dev(bad), E)["err"])[0]) == cap.DERR_ID_RANGE
        bad = ids.copy()
        bad[0, 12, 1] = bad[0, 12, 0]
        assert int(host(cap.coact_stats(dev(bad), E)["err"])[0]) == cap.DERR_ID_REPEAT
        # the context stays usable
        g = cap.coact_stats(dev(ids), E)
        assert int(host(g["err"])[0]) == 0 and (host(g["coact"]) == o["coact"]).all()
    finally:
        cap.coact_stats_method(0)

"""EMA co-activation statistics on the GPU against the oracle: three batches
of counts, bit-exact averages and Ochiai."""
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


@pytest.mark.parametrize("name,alpha", [("one_node", 0.1), ("ep32", 0.5), ("large_ep64", 0.03)])
def test_three_batches(cap, name, alpha):
    w = WORKLOADS[name]
    ema_h = None
    ema_d = None
    for seed in (0, 1, 2):
        ids = make_routing(w, seed=seed)
        c = cap.coact_stats(torch.from_numpy(ids).cuda(), w.E, want=("coact",))["coact"]
        ema_d, och_d = cap.coact_ema(c, alpha, ema_in=ema_d)
        ema_h, och_h = orc.coact_ema(orc.coact(ids, w.E, want=("coact",))["coact"], alpha, ema_h)
        torch.cuda.synchronize()
        assert (ema_d.cpu().numpy().view(np.uint64) == ema_h.view(np.uint64)).all()
        assert (och_d.cpu().numpy().view(np.uint32) == och_h.view(np.uint32)).all()


def test_in_place_is_rejected(cap):
    c = torch.zeros((1, 4, 4), dtype=torch.uint32, device="cuda")
    e = torch.zeros((1, 4, 4), dtype=torch.float64, device="cuda")
    with pytest.raises(cap.MoeError):
        cap.coact_ema(c, 0.5, ema_in=e, ema_out=e)
